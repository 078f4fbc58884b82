"""The give-up path of the bounded device waits, on the GPU.

With the wait limit at 0 every ordinary mbarrier wait of the tensor-core
kernels gives up at its first poll: select with one query head per KV head
and with G = 4 grouped heads, prefill attention for head dim 64 (the
row-owner kernel) and 128 (the chunk-major kernel).  The kernel then records
HILS_ERR_DEVICE_TIMEOUT in the workspace's error word, waits for the copies
and MMAs it already issued, releases its tensor memory and returns.  The test
checks that status and that the next calls on the same context, with the
default limit, give the results of a normal run (bit for bit: the kernels
have a fixed accumulation order) and the oracle's output.
"""
import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_b200 as hils
from chunk_wise_hierarchical_b200._abi import HILS_BF16, make_shape
from hils_inputs import prefill_inputs
from oracle import hils_oracle as O
from parity_util import check_close

pytestmark = pytest.mark.gpu

HILS_OK, HILS_ERR_DEVICE_TIMEOUT = 0, 6


@pytest.mark.parametrize("d,h,g,n", [(64, 2, 2, 64 * 6 + 10), (128, 2, 2, 64 * 6 + 10), (128, 8, 2, 64 * 65 + 3)])
def test_forced_give_up_then_a_normal_call(d, h, g, n):
    b, K = 1, 2
    inp = prefill_inputs(batch=b, heads_q=h, heads_kv=g, seq_len=n, head_dim=d, top_k=K, dtype="bf16", seed=5)
    q, k, v, lm = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.landmark))
    sh = make_shape(b, h, g, d, n, K, HILS_BF16)
    ws_sel = hils.new_workspace(sh, hils.OP_SELECT, q.device)
    ws_att = hils.new_workspace(sh, hils.OP_ATTEND_SELECTED, q.device)

    kbar, hb = hils.summarize(k, lm)
    idx0, sc0 = hils.select(q, kbar, hb, K, g, ws=ws_sel)
    out0 = hils.attend_selected(q, k, v, idx0, sc0, ws=ws_att)
    assert hils.device_status(ws_sel) == HILS_OK and hils.device_status(ws_att) == HILS_OK

    prev = hils.set_wait_limit(0)
    try:
        assert prev == hils.DEFAULT_WAIT_LIMIT
        hils.select(q, kbar, hb, K, g, ws=ws_sel)
        assert hils.device_status(ws_sel) == HILS_ERR_DEVICE_TIMEOUT
        out_fail = torch.zeros_like(q)
        hils.attend_selected(q, k, v, idx0, sc0, out=out_fail, ws=ws_att)
        assert hils.device_status(ws_att) == HILS_ERR_DEVICE_TIMEOUT
        # a kernel that gave up writes no output
        assert not out_fail.any()
    finally:
        hils.set_wait_limit(prev)

    # the following calls, same context and workspaces, default limit
    idx1, sc1 = hils.select(q, kbar, hb, K, g, ws=ws_sel)
    out1 = hils.attend_selected(q, k, v, idx1, sc1, ws=ws_att)
    out2, idx2 = hils.attend(q, k, v, lm, K, return_idx=True)
    torch.cuda.synchronize()
    assert hils.device_status(ws_sel) == HILS_OK and hils.device_status(ws_att) == HILS_OK
    assert torch.equal(idx1, idx0) and torch.equal(sc1, sc0)
    assert torch.equal(out1, out0)
    assert torch.equal(idx2, idx0) and torch.equal(out2, out0)
    ref = O.forward(inp.q, inp.k, inp.v, inp.landmark, 64, K, forced_idx=idx0.cpu().numpy())
    check_close(out0.float().cpu().numpy(), ref["out"], True)
