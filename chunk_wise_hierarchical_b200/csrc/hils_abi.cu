// C ABI of libhils.so: argument validation, workspace layout and dispatch.
// Every entry point checks its arguments on the host, then enqueues kernels on
// the caller's stream; nothing here allocates device memory or synchronises
// (except hils_device_status).
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/hils.h"
#include "common.cuh"
#include "kernels.cuh"

namespace {

// Polls of an ordinary bounded wait in the tensor-core kernels (hils_set_wait_limit).
std::atomic<uint32_t> g_wait_limit{HILS_DEFAULT_WAIT_LIMIT};

constexpr size_t kAlign = 256;
constexpr size_t kHeader = 256;  // error word + reserved
constexpr int kMaxWindow = 64 * 128;  // local branch of at most 128 chunks
constexpr int kMaxDecodeLocal = 16;   // ... and of at most 16 in a decode step

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hils_status check_shape(const hils_shape* s, bool need_seq) {
  if (!s) return HILS_ERR_INVALID_ARG;
  if (s->batch < 0 || s->heads_q <= 0 || s->heads_kv <= 0 || s->head_dim <= 0 || s->seq_len < 0 ||
      s->chunk <= 0 || s->top_k < 0)
    return HILS_ERR_INVALID_ARG;
  if (s->heads_q % s->heads_kv != 0) return HILS_ERR_INVALID_ARG;
  if (!std::isfinite(s->scale)) return HILS_ERR_INVALID_ARG;
  if (s->dtype != HILS_F32 && s->dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
  const int grp = s->heads_q / s->heads_kv;
  if (grp != 1 && grp != 2 && grp != 4 && grp != 8) return HILS_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return HILS_ERR_UNSUPPORTED;
  if (s->chunk != hils::kChunk) return HILS_ERR_UNSUPPORTED;
  if (s->top_k > hils::kMaxTopK) return HILS_ERR_UNSUPPORTED;
  if (s->window < 0 || s->window % s->chunk != 0) return HILS_ERR_INVALID_ARG;
  if (s->window > kMaxWindow) return HILS_ERR_UNSUPPORTED;
  (void)need_seq;
  return HILS_OK;
}

// Chunks in the local branch: the own chunk (window 0 or B) or window / B.
int n_local(const hils_shape* s) { return s->window <= s->chunk ? 1 : s->window / s->chunk; }

float eff_scale(const hils_shape* s) {
  return s->scale == 0.f ? 1.0f / std::sqrt((float)s->head_dim) : s->scale;
}

// Whether prefill attention takes the chunk-major tensor-core path for this shape (its
// scratch is then part of the workspace); the kernel's register check comes at launch.
bool cm_applies(const hils_shape* s) {
  if (s->dtype != HILS_BF16 || s->heads_kv <= 0) return false;
  const int G = s->heads_q / s->heads_kv;
  if (!hils::cm_shape_supported(s->head_dim, G, s->top_k, s->seq_len, n_local(s))) return false;
  const hils::CmScratch S = hils::cm_scratch(s->batch, s->heads_q, s->heads_kv, s->seq_len, s->head_dim,
                                             s->top_k, n_local(s));
  // partial rows and selection indices are 32-bit
  return ((size_t)S.n_lt + S.max_sel) * 128 < (1ull << 31) &&
         (size_t)s->batch * s->heads_kv * s->seq_len * s->top_k < (1ull << 31) &&
         (size_t)s->batch * s->heads_q * s->seq_len < (1ull << 31);
}
size_t cm_bytes(const hils_shape* s) {
  if (!cm_applies(s)) return 0;
  return hils::cm_scratch(s->batch, s->heads_q, s->heads_kv, s->seq_len, s->head_dim, s->top_k, n_local(s)).total;
}

// Whether selection takes the grouped tensor-core path (its split summaries are then
// part of the workspace): bf16, G in {2, 4, 8}, at least one full tile of chunks and of
// queries.
bool gtc_applies(const hils_shape* s) {
  if (s->dtype != HILS_BF16 || s->heads_kv <= 0) return false;
  const int G = s->heads_q / s->heads_kv;
  return hils::select_gtc_supported(s->head_dim, G, s->top_k, true) && s->seq_len / s->chunk >= 64 &&
         s->seq_len >= 128;
}
size_t gtc_bytes(const hils_shape* s) {
  if (!gtc_applies(s)) return 0;
  return 2 * align_up(hils::gtc_split_bytes(s->batch, s->heads_q, s->seq_len / s->chunk, s->head_dim));
}

struct AttendLayout {
  size_t kbar, hbias, idx, ssel, gtc, cm, total;
};
AttendLayout attend_layout(const hils_shape* s) {
  const size_t b = s->batch, h = s->heads_q, g = s->heads_kv, n = s->seq_len, d = s->head_dim;
  const size_t C = n / s->chunk, K = s->top_k;
  AttendLayout L;
  size_t off = kHeader;
  L.kbar = off; off = align_up(off + b * h * C * d * 4);
  L.hbias = off; off = align_up(off + b * h * C * 4);
  L.idx = off; off = align_up(off + b * g * n * K * 4);
  L.ssel = off; off = align_up(off + b * h * n * K * 4);
  L.gtc = off; off = align_up(off + gtc_bytes(s));
  L.cm = off; off = align_up(off + cm_bytes(s));
  L.total = off;
  return L;
}

struct BackwardLayout {
  size_t drow, list_off, list, total;
};
BackwardLayout backward_layout(const hils_shape* s) {
  const size_t b = s->batch, h = s->heads_q, g = s->heads_kv, n = s->seq_len, K = s->top_k;
  const size_t C = n / s->chunk;
  BackwardLayout L;
  size_t off = kHeader;
  L.drow = off; off = align_up(off + b * h * n * 4);
  L.list_off = off; off = align_up(off + b * g * (C + 1) * 4);
  L.list = off; off = align_up(off + b * g * n * K * 4);
  L.total = off;
  return L;
}

struct DecodeLayout {
  size_t part_keys, part_att, scan_ticket, att_ticket, idx, sel_page, ssel, total;
};
DecodeLayout decode_layout(const hils_shape* s) {
  const size_t b = s->batch, h = s->heads_q, g = s->heads_kv, K = s->top_k, d = s->head_dim;
  const size_t G = h / g;
  const int cmax = (s->seq_len + s->chunk - 1) / s->chunk;
  const size_t nsplit = hils::decode_splits(s->batch, cmax);
  DecodeLayout L;
  size_t off = kHeader;
  L.part_keys = off; off = align_up(off + b * g * nsplit * K * 8);
  L.part_att = off; off = align_up(off + b * g * 2 * (K + n_local(s)) * G * (d + 2) * 4);  // half-chunk partials
  L.scan_ticket = off; off = align_up(off + b * g * 4);
  L.att_ticket = off; off = align_up(off + b * g * 4);
  L.idx = off; off = align_up(off + b * g * K * 4);
  L.sel_page = off; off = align_up(off + b * g * K * 4);
  L.ssel = off; off = align_up(off + b * h * K * 4);
  L.total = off;
  return L;
}

hils_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA; }

// Prefill attention + fusion for a selection: the chunk-major tcgen05 path for bf16
// inputs (scratch at `cm_ws`, 256-byte aligned), else the row-owner tcgen05 kernels
// where they fit the shape, else the row kernel.
cudaError_t run_prefill_attention(const hils_shape* s, const void* q, const void* k, const void* v,
                                  const int32_t* idx, const float* ssel, void* out, float* lse,
                                  unsigned* err, void* cm_ws, cudaStream_t cs) {
  const bool bf16 = s->dtype == HILS_BF16;
  const int G = s->heads_q / s->heads_kv;
  // d = 64 with the own-chunk branch stays on the row-owner kernel, measured faster there;
  // every other bf16 shape the chunk-major path covers takes it
  const bool row_owner_d64 = bf16 && n_local(s) == 1 && s->head_dim == 64 &&
                             hils::attend_tc3_supported(64, G, s->top_k, s->seq_len);
  if (!row_owner_d64 && cm_ws && cm_applies(s) && hils::cm_kernel_ready(s->head_dim, G)) {
    const hils::CmScratch S = hils::cm_scratch(s->batch, s->heads_q, s->heads_kv, s->seq_len, s->head_dim,
                                               s->top_k, n_local(s));
    char* w = static_cast<char*>(cm_ws);
    hils::CmArgs a{};
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.idx = idx; a.ssel = ssel; a.out = static_cast<__nv_bfloat16*>(out); a.lse = lse; a.err = err;
    a.cnt = reinterpret_cast<int*>(w + S.cnt);
    a.cur = reinterpret_cast<int*>(w + S.cur);
    a.toff = reinterpret_cast<int*>(w + S.toff);
    a.n_sel = reinterpret_cast<int*>(w + S.n_sel);
    a.abort_flag = reinterpret_cast<int*>(w + S.abort_flag);
    a.desc = reinterpret_cast<int4*>(w + S.desc);
    a.ent_q = reinterpret_cast<int*>(w + S.ent_q);
    a.pos = reinterpret_cast<int*>(w + S.pos);
    a.part = reinterpret_cast<__nv_bfloat16*>(w + S.part);
    a.plse = reinterpret_cast<float*>(w + S.plse);
    a.b = s->batch; a.h = s->heads_q; a.g = s->heads_kv; a.n = s->seq_len; a.d = s->head_dim;
    a.top_k = s->top_k; a.n_local = n_local(s);
    a.c_sel = S.c_sel; a.c_all = S.c_all; a.tl = S.tl; a.n_lt = S.n_lt; a.max_sel = S.max_sel;
    a.scale = eff_scale(s);
    a.poll = g_wait_limit.load();
    return hils::run_attend_cm(a, cs);
  }
  if (bf16 && n_local(s) == 1 && hils::attend_tc_supported(s->head_dim, G, s->top_k, s->seq_len)) {
    hils::TcAttendArgs ta{};
    ta.q = static_cast<const __nv_bfloat16*>(q);
    ta.k = static_cast<const __nv_bfloat16*>(k);
    ta.v = static_cast<const __nv_bfloat16*>(v);
    ta.idx = idx; ta.ssel = ssel; ta.out = static_cast<__nv_bfloat16*>(out); ta.lse = lse; ta.err = err;
    ta.b = s->batch; ta.h = s->heads_q; ta.g = s->heads_kv; ta.n = s->seq_len; ta.top_k = s->top_k;
    ta.scale = eff_scale(s);
    ta.poll = g_wait_limit.load();
    return hils::run_attend_tc(ta, s->head_dim, cs);
  }
  hils::AttendRowsArgs ar{};
  ar.q = q; ar.k = k; ar.v = v; ar.idx = idx; ar.ssel = ssel; ar.out = out; ar.lse = lse;
  ar.block_table = nullptr; ar.seq_lens = nullptr; ar.err = err;
  ar.b = s->batch; ar.h = s->heads_q; ar.g = s->heads_kv; ar.n = s->seq_len; ar.d = s->head_dim;
  ar.top_k = s->top_k; ar.max_chunks = 0; ar.n_pages = 0; ar.scale = eff_scale(s); ar.bf16 = bf16;
  ar.paged = false; ar.n_local = n_local(s);
  return hils::run_attend_rows(ar, cs);
}

}  // namespace

extern "C" {

const char* hils_status_string(int status) {
  switch (status) {
    case HILS_OK: return "ok";
    case HILS_ERR_INVALID_ARG: return "invalid argument";
    case HILS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case HILS_ERR_WORKSPACE: return "workspace missing or too small";
    case HILS_ERR_CUDA: return "CUDA error";
    case HILS_ERR_DEVICE_CHECK: return "device-side index check failed";
    case HILS_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int32_t hils_abi_version(void) { return 3; }

uint32_t hils_set_wait_limit(uint32_t polls) { return g_wait_limit.exchange(polls); }

hils_status hils_workspace_size(const hils_shape* s, int32_t op, size_t* bytes) {
  if (!bytes) return HILS_ERR_INVALID_ARG;
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  switch (op) {
    case HILS_OP_SELECT: *bytes = kHeader + gtc_bytes(s); return HILS_OK;
    case HILS_OP_ATTEND: *bytes = attend_layout(s).total; return HILS_OK;
    case HILS_OP_DECODE: *bytes = decode_layout(s).total; return HILS_OK;
    case HILS_OP_ATTEND_SELECTED: *bytes = kHeader + cm_bytes(s); return HILS_OK;
    case HILS_OP_BACKWARD: *bytes = backward_layout(s).total; return HILS_OK;
  }
  return HILS_ERR_INVALID_ARG;
}

hils_status hils_summarize(const hils_shape* s, const void* k, const void* landmark_q, float* kbar,
                           float* hbias, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  const int C = s->seq_len / s->chunk;
  if ((size_t)s->batch * C == 0) return HILS_OK;
  if (!k || !landmark_q || !kbar || !hbias) return HILS_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(landmark_q) || !aligned16(kbar)) return HILS_ERR_INVALID_ARG;
  hils::SummarizeArgs a{};
  a.k = k; a.lm = landmark_q; a.kbar = kbar; a.hbias = hbias;
  a.b = s->batch; a.h = s->heads_q; a.g = s->heads_kv; a.n = s->seq_len; a.d = s->head_dim;
  a.n_chunks = C; a.scale = eff_scale(s); a.bf16 = s->dtype == HILS_BF16;
  a.page_ids = nullptr;
  return cuda_status(hils::run_summarize(a, (cudaStream_t)stream));
}

hils_status hils_summarize_paged(const hils_shape* s, const void* k_pages, const void* landmark_pages,
                                 const int32_t* page_ids, int32_t n_listed, int32_t n_pages,
                                 float* kbar_pages, float* hbias_pages, void* stream) {
  return hils_summarize_paged_ex(s, k_pages, landmark_pages, page_ids, n_listed, n_pages, kbar_pages, HILS_F32,
                                 hbias_pages, stream);
}

hils_status hils_summarize_paged_ex(const hils_shape* s, const void* k_pages, const void* landmark_pages,
                                    const int32_t* page_ids, int32_t n_listed, int32_t n_pages,
                                    void* kbar_pages, int32_t summary_dtype, float* hbias_pages, void* stream) {
  hils_status st = check_shape(s, false);
  if (st != HILS_OK) return st;
  if (summary_dtype != HILS_F32 && summary_dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
  if (summary_dtype == HILS_BF16 && s->dtype != HILS_BF16) return HILS_ERR_UNSUPPORTED;
  if (n_listed < 0 || n_pages < 0) return HILS_ERR_INVALID_ARG;
  if (n_listed == 0) return HILS_OK;
  if (!k_pages || !landmark_pages || !page_ids || !kbar_pages || !hbias_pages) return HILS_ERR_INVALID_ARG;
  if (!aligned16(k_pages) || !aligned16(landmark_pages) || !aligned16(kbar_pages)) return HILS_ERR_INVALID_ARG;
  hils::SummarizeArgs a{};
  a.k = k_pages; a.lm = landmark_pages; a.kbar = kbar_pages; a.hbias = hbias_pages;
  a.b = 0; a.h = s->heads_q; a.g = s->heads_kv; a.n = 0; a.d = s->head_dim; a.n_chunks = 0;
  a.scale = eff_scale(s); a.bf16 = s->dtype == HILS_BF16;
  a.page_ids = page_ids; a.n_listed = n_listed; a.n_pages = n_pages;
  a.kbar_bf16 = summary_dtype == HILS_BF16;
  return cuda_status(hils::run_summarize(a, (cudaStream_t)stream));
}

// Scores + Top-K: the tensor-core kernel where it applies (bf16, G = 1), else SIMT.
// gtc_ws: the split-summary scratch (gtc_bytes), or nullptr where the grouped path does
// not apply.
static cudaError_t run_select(const hils::SelectArgs& a, void* gtc_ws, cudaStream_t st) {
  if (hils::select_tc_supported(a.d, a.h / a.g, a.top_k, a.bf16)) {
    hils::SelectArgs t = a;
    t.poll = g_wait_limit.load();
    return hils::run_select_tc(t, st);
  }
  if (gtc_ws) {
    hils::GtcArgs g{};
    g.q = static_cast<const __nv_bfloat16*>(a.q);
    g.kbar = a.kbar; g.hbias = a.hbias; g.idx = a.idx; g.score = a.score; g.err = a.err;
    const size_t half = align_up(hils::gtc_split_bytes(a.b, a.h, a.n_chunks, a.d));
    g.kbar_hi = static_cast<__nv_bfloat16*>(gtc_ws);
    g.kbar_lo = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(gtc_ws) + half);
    g.b = a.b; g.h = a.h; g.g = a.g; g.n = a.n; g.d = a.d; g.n_chunks = a.n_chunks; g.top_k = a.top_k;
    g.n_local = a.n_local; g.scale = a.scale; g.poll = g_wait_limit.load();
    return hils::run_select_gtc(g, st);
  }
  return hils::run_select_simt(a, st);
}

hils_status hils_select(const hils_shape* s, const void* q, const float* kbar, const float* hbias,
                        int32_t* topk_idx, float* topk_score, void* ws, size_t ws_bytes, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if ((size_t)s->batch * s->seq_len * s->top_k == 0) return HILS_OK;
  const int C = s->seq_len / s->chunk;
  if (!q || !topk_idx || (C > 0 && (!kbar || !hbias))) return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || (C > 0 && !aligned16(kbar))) return HILS_ERR_INVALID_ARG;
  const size_t gb = gtc_bytes(s);
  if (!ws || ws_bytes < kHeader + gb || !aligned16(ws)) return HILS_ERR_WORKSPACE;
  hils::SelectArgs a{};
  a.q = q; a.kbar = kbar; a.hbias = hbias; a.idx = topk_idx; a.score = topk_score;
  a.err = static_cast<unsigned*>(ws);
  a.b = s->batch; a.h = s->heads_q; a.g = s->heads_kv; a.n = s->seq_len; a.d = s->head_dim;
  a.n_chunks = C; a.top_k = s->top_k; a.scale = eff_scale(s); a.bf16 = s->dtype == HILS_BF16;
  a.n_local = n_local(s);
  return cuda_status(run_select(a, gb ? static_cast<char*>(ws) + kHeader : nullptr, (cudaStream_t)stream));
}

hils_status hils_attend(const hils_shape* s, const void* q, const void* k, const void* v,
                        const void* landmark_q, void* out, float* lse_out, int32_t* topk_idx_out, void* ws,
                        size_t ws_bytes, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if ((size_t)s->batch * s->seq_len == 0) return HILS_OK;
  const int C = s->seq_len / s->chunk;
  if (!q || !k || !v || !out || (C > 0 && !landmark_q)) return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (C > 0 && !aligned16(landmark_q)))
    return HILS_ERR_INVALID_ARG;
  const AttendLayout L = attend_layout(s);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return HILS_ERR_WORKSPACE;
  cudaStream_t cs = (cudaStream_t)stream;
  char* w = static_cast<char*>(ws);
  float* kbar = reinterpret_cast<float*>(w + L.kbar);
  float* hbias = reinterpret_cast<float*>(w + L.hbias);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(w + L.idx);
  float* ssel = reinterpret_cast<float*>(w + L.ssel);
  const bool bf16 = s->dtype == HILS_BF16;
  const float scale = eff_scale(s);

  if (C > 0) {
    hils::SummarizeArgs sa{};
    sa.k = k; sa.lm = landmark_q; sa.kbar = kbar; sa.hbias = hbias;
    sa.b = s->batch; sa.h = s->heads_q; sa.g = s->heads_kv; sa.n = s->seq_len; sa.d = s->head_dim;
    sa.n_chunks = C; sa.scale = scale; sa.bf16 = bf16; sa.page_ids = nullptr;
    if (hils::run_summarize(sa, cs) != cudaSuccess) return HILS_ERR_CUDA;
  }
  if (s->top_k > 0) {
    hils::SelectArgs se{};
    se.q = q; se.kbar = kbar; se.hbias = hbias; se.idx = idx; se.score = ssel;
    se.b = s->batch; se.h = s->heads_q; se.g = s->heads_kv; se.n = s->seq_len; se.d = s->head_dim;
    se.n_chunks = C; se.top_k = s->top_k; se.scale = scale; se.bf16 = bf16; se.n_local = n_local(s);
    se.err = reinterpret_cast<unsigned*>(w);
    if (run_select(se, L.gtc != L.cm ? w + L.gtc : nullptr, cs) != cudaSuccess) return HILS_ERR_CUDA;
  }
  return cuda_status(run_prefill_attention(s, q, k, v, idx, ssel, out, lse_out, reinterpret_cast<unsigned*>(w),
                                           L.cm != L.total ? w + L.cm : nullptr, cs));
}

hils_status hils_attend_selected(const hils_shape* s, const void* q, const void* k, const void* v,
                                 const int32_t* topk_idx, const float* topk_score, void* out, float* lse_out,
                                 void* ws, size_t ws_bytes, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if ((size_t)s->batch * s->seq_len == 0) return HILS_OK;
  if (!q || !k || !v || !out || (s->top_k > 0 && (!topk_idx || !topk_score))) return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return HILS_ERR_INVALID_ARG;
  const size_t cmb = cm_bytes(s);
  if (!ws || ws_bytes < kHeader + cmb || !aligned16(ws)) return HILS_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  return cuda_status(run_prefill_attention(s, q, k, v, topk_idx, topk_score, out, lse_out,
                                           reinterpret_cast<unsigned*>(ws), cmb ? w + kHeader : nullptr,
                                           (cudaStream_t)stream));
}

hils_status hils_backward(const hils_shape* s, const void* q, const void* k, const void* v,
                          const void* landmark_q, const void* out, const float* lse, const int32_t* topk_idx,
                          const float* topk_score, const void* dout, float* dq, float* dk, float* dv,
                          float* dlandmark, void* ws, size_t ws_bytes, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if (s->dtype != HILS_BF16) return HILS_ERR_UNSUPPORTED;
  if ((size_t)s->batch * s->seq_len == 0) return HILS_OK;
  if ((long long)s->seq_len * s->top_k >= (1ll << 31) || s->seq_len >= (1 << 25)) return HILS_ERR_UNSUPPORTED;
  const int C = s->seq_len / s->chunk;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return HILS_ERR_INVALID_ARG;
  if (C > 0 && (!landmark_q || !dlandmark)) return HILS_ERR_INVALID_ARG;
  if (s->top_k > 0 && (!topk_idx || !topk_score)) return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (C > 0 && !aligned16(landmark_q)))
    return HILS_ERR_INVALID_ARG;
  const BackwardLayout L = backward_layout(s);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return HILS_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  hils::BwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.landmark = landmark_q; a.out = out; a.dout = dout; a.lse = lse;
  a.idx = topk_idx; a.ssel = topk_score; a.dq = dq; a.dk = dk; a.dv = dv; a.dlandmark = dlandmark;
  a.drow = reinterpret_cast<float*>(w + L.drow);
  a.list_off = reinterpret_cast<int*>(w + L.list_off);
  a.list = reinterpret_cast<int*>(w + L.list);
  a.err = reinterpret_cast<unsigned*>(w);
  a.b = s->batch; a.h = s->heads_q; a.g = s->heads_kv; a.n = s->seq_len; a.d = s->head_dim;
  a.top_k = s->top_k; a.n_local = n_local(s); a.scale = eff_scale(s);
  return cuda_status(hils::run_backward(a, (cudaStream_t)stream));
}

hils_status hils_decode(const hils_shape* s, const void* q, const void* k_pages, const void* v_pages,
                        const float* kbar_pages, const float* hbias_pages, const int32_t* block_table,
                        int32_t max_chunks, const int32_t* seq_lens, int32_t n_pages, void* out,
                        int32_t* topk_idx_out, void* ws, size_t ws_bytes, void* stream) {
  return hils_decode_ex(s, q, k_pages, v_pages, kbar_pages, HILS_F32, hbias_pages, block_table, max_chunks,
                        seq_lens, n_pages, out, topk_idx_out, ws, ws_bytes, stream);
}

hils_status hils_decode_ex(const hils_shape* s, const void* q, const void* k_pages, const void* v_pages,
                           const void* kbar_pages, int32_t summary_dtype, const float* hbias_pages,
                           const int32_t* block_table, int32_t max_chunks, const int32_t* seq_lens,
                           int32_t n_pages, void* out, int32_t* topk_idx_out, void* ws, size_t ws_bytes,
                           void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if (summary_dtype != HILS_F32 && summary_dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
  if (summary_dtype == HILS_BF16 && s->dtype != HILS_BF16) return HILS_ERR_UNSUPPORTED;
  if (s->batch == 0) return HILS_OK;
  if (!hils::decode_supported(s->heads_q, s->head_dim) || n_local(s) > kMaxDecodeLocal) return HILS_ERR_UNSUPPORTED;
  if (max_chunks <= 0 || n_pages <= 0) return HILS_ERR_INVALID_ARG;
  if ((long long)max_chunks > ((long long)s->seq_len + s->chunk - 1) / s->chunk) return HILS_ERR_INVALID_ARG;
  if (!hils::decode_merge_supported(s->batch, max_chunks, s->top_k)) return HILS_ERR_UNSUPPORTED;
  if (!q || !k_pages || !v_pages || !kbar_pages || !hbias_pages || !block_table || !seq_lens || !out)
    return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(kbar_pages) ||
      !aligned16(out))
    return HILS_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(s);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return HILS_ERR_WORKSPACE;
  cudaStream_t cs = (cudaStream_t)stream;
  char* w = static_cast<char*>(ws);
  unsigned* err = reinterpret_cast<unsigned*>(w);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(w + L.idx);
  hils::DecodeArgs da{};
  da.q = q; da.k_pages = k_pages; da.v_pages = v_pages; da.kbar_pages = kbar_pages;
  da.hbias_pages = hbias_pages; da.block_table = block_table; da.seq_lens = seq_lens; da.out = out;
  da.idx = idx;
  da.ssel = reinterpret_cast<float*>(w + L.ssel);
  da.sel_page = reinterpret_cast<int32_t*>(w + L.sel_page);
  da.part_keys = reinterpret_cast<unsigned long long*>(w + L.part_keys);
  da.part_att = reinterpret_cast<float*>(w + L.part_att);
  da.scan_ticket = reinterpret_cast<unsigned*>(w + L.scan_ticket);
  da.att_ticket = reinterpret_cast<unsigned*>(w + L.att_ticket);
  da.err = err;
  da.b = s->batch; da.h = s->heads_q; da.g = s->heads_kv; da.d = s->head_dim; da.top_k = s->top_k;
  da.max_chunks = max_chunks; da.n_pages = n_pages; da.scale = eff_scale(s);
  da.bf16 = s->dtype == HILS_BF16;
  da.kbar_bf16 = summary_dtype == HILS_BF16;
  da.n_local = n_local(s);
  return cuda_status(hils::run_decode(da, cs));
}

hils_status hils_device_status(void* ws, void* stream) {
  if (!ws) return HILS_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return HILS_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return HILS_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(word), cs) != cudaSuccess) return HILS_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return HILS_ERR_CUDA;
  }
  if (word & hils::kErrTimeout) return HILS_ERR_DEVICE_TIMEOUT;
  if (word & hils::kErrBadPage) return HILS_ERR_DEVICE_CHECK;
  return HILS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// hils_decode_static: decode whose scratch is a device array owned by this
// file, for callers that cannot hand the library a workspace (no counterpart
// in the HiLS notes).  Nothing here allocates or frees device memory.
namespace {

constexpr size_t kStaticScratchBytes = HILS_DECODE_STATIC_SCRATCH_BYTES;
constexpr size_t kStaticTicketSlots = 4096;  // batch * heads_kv limit
constexpr int kStaticMaxDevices = 64;

// Scratch of hils_decode_static.  Byte layout (fixed parts first, so the ticket
// counters never share bytes with the data of a call of another shape):
//   [0, 256)                 error word, when the caller passes no status word
//   [256, 256 + 16 KiB)      scan tickets, one per (sequence, KV head)
//   [.., + 16 KiB)           attention tickets
//   then, per call's shape: part_keys, part_att, idx, sel_page, ssel
// The ticket counters must be zero when a call starts: device memory of a
// __device__ array is zero when the module is loaded, and every call that
// completes leaves them at zero (the CTA that consumes a ticket resets it).
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

struct StaticLayout {
  size_t scan_ticket, att_ticket, part_keys, part_att, idx, sel_page, ssel, total;
};
StaticLayout static_decode_layout(const hils_shape* s) {
  const size_t b = s->batch, h = s->heads_q, g = s->heads_kv, K = s->top_k, d = s->head_dim;
  const size_t G = h / g;
  const int cmax = (s->seq_len + s->chunk - 1) / s->chunk;
  const size_t nsplit = hils::decode_splits(s->batch, cmax);
  StaticLayout L;
  size_t off = kHeader;
  L.scan_ticket = off; off += kStaticTicketSlots * 4;
  L.att_ticket = off; off += kStaticTicketSlots * 4;
  L.part_keys = off; off = align_up(off + b * g * nsplit * K * 8);
  L.part_att = off; off = align_up(off + b * g * 2 * (K + n_local(s)) * G * (d + 2) * 4);  // half-chunk partials
  L.idx = off; off = align_up(off + b * g * K * 4);
  L.sel_page = off; off = align_up(off + b * g * K * 4);
  L.ssel = off; off = align_up(off + b * h * K * 4);
  L.total = off;
  return L;
}

std::mutex g_static_mu;
unsigned char* g_static_ptr[kStaticMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device (the lookup may load this library's device code onto it).
cudaError_t static_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kStaticMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

hils_status hils_decode_static(const hils_shape* s, const void* q, const void* k_pages, const void* v_pages,
                               const float* kbar_pages, const float* hbias_pages, const int32_t* block_table,
                               int32_t max_chunks, const int32_t* seq_lens, int32_t n_pages, void* out,
                               int32_t* topk_idx_out, unsigned* status_word, void* stream) {
  hils_status st = check_shape(s, true);
  if (st != HILS_OK) return st;
  if (s->batch == 0) return HILS_OK;
  if (!hils::decode_supported(s->heads_q, s->head_dim) || n_local(s) > kMaxDecodeLocal) return HILS_ERR_UNSUPPORTED;
  if (max_chunks <= 0 || n_pages <= 0) return HILS_ERR_INVALID_ARG;
  if ((long long)max_chunks > ((long long)s->seq_len + s->chunk - 1) / s->chunk) return HILS_ERR_INVALID_ARG;
  if (!hils::decode_merge_supported(s->batch, max_chunks, s->top_k)) return HILS_ERR_UNSUPPORTED;
  if (!q || !k_pages || !v_pages || !kbar_pages || !hbias_pages || !block_table || !seq_lens || !out)
    return HILS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(kbar_pages) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(status_word) & 3u) != 0)
    return HILS_ERR_INVALID_ARG;
  if ((size_t)s->batch * s->heads_kv > kStaticTicketSlots) return HILS_ERR_WORKSPACE;
  const StaticLayout L = static_decode_layout(s);
  if (L.total > kStaticScratchBytes) return HILS_ERR_WORKSPACE;
  unsigned char* w = nullptr;
  if (static_scratch(&w) != cudaSuccess) return HILS_ERR_CUDA;
  hils::DecodeArgs da{};
  da.q = q; da.k_pages = k_pages; da.v_pages = v_pages; da.kbar_pages = kbar_pages;
  da.hbias_pages = hbias_pages; da.block_table = block_table; da.seq_lens = seq_lens; da.out = out;
  da.idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(w + L.idx);
  da.ssel = reinterpret_cast<float*>(w + L.ssel);
  da.sel_page = reinterpret_cast<int32_t*>(w + L.sel_page);
  da.part_keys = reinterpret_cast<unsigned long long*>(w + L.part_keys);
  da.part_att = reinterpret_cast<float*>(w + L.part_att);
  da.scan_ticket = reinterpret_cast<unsigned*>(w + L.scan_ticket);
  da.att_ticket = reinterpret_cast<unsigned*>(w + L.att_ticket);
  da.err = status_word ? status_word : reinterpret_cast<unsigned*>(w);
  da.b = s->batch; da.h = s->heads_q; da.g = s->heads_kv; da.d = s->head_dim; da.top_k = s->top_k;
  da.max_chunks = max_chunks; da.n_pages = n_pages; da.scale = eff_scale(s);
  da.bf16 = s->dtype == HILS_BF16;
  da.n_local = n_local(s);
  return cuda_status(hils::run_decode(da, (cudaStream_t)stream));
}

}  // extern "C"
