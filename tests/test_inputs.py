"""The seeded workload generator: determinism, shapes and needle planting."""
import torch

from hils_inputs import prefill_inputs, decode_inputs


def test_prefill_inputs_deterministic_and_needles():
    a = prefill_inputs(2, 4, 2, 512, 32, chunk=64, top_k=4, dtype="bf16", needles=3, seed=5)
    b = prefill_inputs(2, 4, 2, 512, 32, chunk=64, top_k=4, dtype="bf16", needles=3, seed=5)
    assert torch.equal(a.k, b.k) and torch.equal(a.q, b.q) and a.needles == b.needles
    assert a.q.shape == (2, 4, 512, 32) and a.k.shape == (2, 2, 512, 32)
    assert a.landmark.shape == (2, 4, 8, 32)
    assert len(a.needles) == 2 * 4 * 3
    for (bi, hi, c, j, i) in a.needles:
        assert i >= (c + 1) * 64
        key = a.k[bi, hi // 2, c * 64 + j].float()
        # a later needle may overwrite an earlier one at the same slot
        assert abs(key.norm().item() - 4.0) < 0.05


def test_decode_inputs_pages_are_a_permutation():
    di = decode_inputs(3, 4, 2, 0, 16, chunk=64, top_k=4, seq_lens=[1, 130, 64], seed=1)
    bt = di.block_table
    used = bt[bt >= 0].tolist()
    assert sorted(used) == list(range(di.k_pages.shape[0]))
    assert (bt[0] >= 0).sum() == 1 and (bt[1] >= 0).sum() == 3 and (bt[2] >= 0).sum() == 1
    assert all(c < (L - 1) // 64 for (b, h, c, j), L in
               [(n, [1, 130, 64][n[0]]) for n in di.needles])
