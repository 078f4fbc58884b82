// Row-wise HiLS attention on CUDA cores: intra-chunk softmax attention over
// each selected chunk and the own causal chunk, then the inter-chunk fusion
// (HiLS notes, section 5.3; Tide digest, Figure 3).  Used for fp32 prefill
// and for shapes outside the tensor-core kernel's shared-memory plan.
//
// One warp per (sequence, KV group, query): lane j owns keys j and j+32 of a
// chunk, and d/32 output columns.  The group's G query heads share every key
// and value load.  For each chunk the warp computes, per head, the running
// max m, the sum l of exp(s - m) and the unnormalised PV row; the fusion then
// weights chunk c by exp(shat_c - M) / Z' and the local branch by
// exp(LSE_local - M) / Z', with M the max of all log-masses and Z' their
// shifted sum.  The local branch is the own causal chunk or, with a sliding
// window of n_local chunks, the own chunk and the n_local - 1 chunks before
// it, merged chunk by chunk with the split-softmax rule.  The row's log Zhat
// = M + log Z' is written when an lse buffer is given.
#include "common.cuh"
#include "kernels.cuh"

namespace hils {

constexpr int kRowWarps = 4;

template <typename T, int D, int G>
struct ChunkAcc {
  float m[G], l[G], o[G][D / 32];
};

// Attention of the G query rows (in shared memory) over `nvalid` keys/values
// starting at kp/vp (row-major [B][D]).
template <typename T, int D, int G>
__device__ __forceinline__ void chunk_attend(const float* __restrict__ qS, const T* __restrict__ kp,
                                             const T* __restrict__ vp, int nvalid, float scale,
                                             ChunkAcc<T, D, G>& r) {
  const int lane = threadIdx.x & 31;
  const int j0 = lane, j1 = lane + 32;
  float s0[G], s1[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) { s0[hh] = 0.f; s1[hh] = 0.f; }
  const bool v0 = j0 < nvalid, v1 = j1 < nvalid;
#pragma unroll 4
  for (int e = 0; e < D; e += 4) {
    float4 k0 = v0 ? load4(kp + (size_t)j0 * D + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 k1 = v1 ? load4(kp + (size_t)j1 * D + e) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float4 qv = *reinterpret_cast<const float4*>(qS + hh * D + e);
      s0[hh] = fmaf(qv.x, k0.x, fmaf(qv.y, k0.y, fmaf(qv.z, k0.z, fmaf(qv.w, k0.w, s0[hh]))));
      s1[hh] = fmaf(qv.x, k1.x, fmaf(qv.y, k1.y, fmaf(qv.z, k1.z, fmaf(qv.w, k1.w, s1[hh]))));
    }
  }
  float p0[G], p1[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float a0 = v0 ? s0[hh] * scale : -INFINITY;
    const float a1 = v1 ? s1[hh] * scale : -INFINITY;
    const float m = warp_max(fmaxf(a0, a1));
    p0[hh] = v0 ? expf(a0 - m) : 0.f;
    p1[hh] = v1 ? expf(a1 - m) : 0.f;
    r.m[hh] = m;
    r.l[hh] = warp_sum(p0[hh] + p1[hh]);
#pragma unroll
    for (int x = 0; x < D / 32; ++x) r.o[hh][x] = 0.f;
  }
  for (int j = 0; j < nvalid; ++j) {
    const int src = j & 31;
    float vj[D / 32];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) vj[x] = to_f(vp[(size_t)j * D + lane + 32 * x]);
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0[hh] : p1[hh], src);
#pragma unroll
      for (int x = 0; x < D / 32; ++x) r.o[hh][x] = fmaf(pj, vj[x], r.o[hh][x]);
    }
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kRowWarps * 32) attend_rows_kernel(AttendRowsArgs a) {
  __shared__ __align__(16) float qS[kRowWarps][G * D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kRowWarps + warp;
  const int n_q = a.paged ? 1 : a.n;  // queries per (sequence, group)
  const long long total = (long long)a.b * a.g * n_q;
  if (row >= total) return;
  const int qi = (int)(row % n_q);
  const int gi = (int)((row / n_q) % a.g);
  const int bi = (int)(row / ((long long)n_q * a.g));
  const int K = a.top_k;
  const int B = kChunk;

  int pos;  // absolute position of the query
  if (a.paged) {
    pos = a.seq_lens[bi] - 1;
  } else {
    pos = qi;
  }
  T* out = static_cast<T*>(a.out);
  auto out_row = [&](int hh) -> T* {
    const size_t hq = (size_t)bi * a.h + gi * G + hh;
    return a.paged ? out + hq * D : out + (hq * a.n + qi) * D;
  };
  if (pos < 0) {  // empty sequence (decode): zero output
    for (int hh = 0; hh < G; ++hh)
      for (int x = 0; x < D / 32; ++x) out_row(hh)[lane + 32 * x] = from_f<T>(0.f);
    return;
  }
  // query rows
  const T* qbase = static_cast<const T*>(a.q);
  for (int x = lane; x < G * D; x += 32) {
    const int hh = x / D, e = x % D;
    const size_t hq = (size_t)bi * a.h + gi * G + hh;
    qS[warp][x] = to_f(a.paged ? qbase[hq * D + e] : qbase[(hq * a.n + qi) * D + e]);
  }
  __syncwarp();

  const T* kb = static_cast<const T*>(a.k);
  const T* vb = static_cast<const T*>(a.v);
  auto chunk_ptr = [&](const T* base, int c, bool& ok) -> const T* {
    ok = true;
    if (a.paged) {
      const int p = (c < a.max_chunks) ? a.block_table[(size_t)bi * a.max_chunks + c] : -1;
      if (p < 0 || p >= a.n_pages) { ok = false; return base; }
      return base + (((size_t)p * a.g + gi) * B) * D;
    }
    return base + (((size_t)bi * a.g + gi) * a.n + (size_t)c * B) * D;
  };

  const int own = pos / B;
  const int lo_c = max(0, own + 1 - a.n_local);  // first chunk of the local branch
  const int n_cand = lo_c;                        // remote candidates: c < lo_c
  ChunkAcc<T, D, G> r, loc;
  bool ok;
  float lse_own[G], acc[G][D / 32];
  // local branch, chunk by chunk (the last one causal up to the query)
  for (int c = lo_c; c <= own; ++c) {
    const T* kp = chunk_ptr(kb, c, ok);
    const T* vp = chunk_ptr(vb, c, ok);
    if (!ok) {
      set_error(a.err, kErrBadPage);
      for (int hh = 0; hh < G; ++hh)
        for (int x = 0; x < D / 32; ++x) out_row(hh)[lane + 32 * x] = from_f<T>(0.f);
      return;
    }
    chunk_attend<T, D, G>(qS[warp], kp, vp, c == own ? pos - own * B + 1 : B, a.scale, c == lo_c ? loc : r);
    if (c == lo_c) continue;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {  // merge r into loc
      const float m = fmaxf(loc.m[hh], r.m[hh]);
      const float fa = expf(loc.m[hh] - m), fb = expf(r.m[hh] - m);
      loc.l[hh] = loc.l[hh] * fa + r.l[hh] * fb;
#pragma unroll
      for (int x = 0; x < D / 32; ++x) loc.o[hh][x] = loc.o[hh][x] * fa + r.o[hh][x] * fb;
      loc.m[hh] = m;
    }
  }
  const int32_t* idx = a.idx + (((size_t)bi * a.g + gi) * n_q + qi) * K;
  float M[G], Zp[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    lse_own[hh] = loc.m[hh] + logf(loc.l[hh]);
    M[hh] = lse_own[hh];
  }
  // fusion max and normaliser over the selected surrogate masses
  for (int s = 0; s < K; ++s) {
    if (idx[s] < 0 || (!a.paged && idx[s] >= n_cand)) continue;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float sh = a.ssel[(((size_t)bi * a.h + gi * G + hh) * n_q + qi) * K + s];
      M[hh] = fmaxf(M[hh], sh);
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) Zp[hh] = expf(lse_own[hh] - M[hh]);
  for (int s = 0; s < K; ++s) {
    if (idx[s] < 0 || (!a.paged && idx[s] >= n_cand)) continue;
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      Zp[hh] += expf(a.ssel[(((size_t)bi * a.h + gi * G + hh) * n_q + qi) * K + s] - M[hh]);
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    // local branch: weight exp(LSE_local - M)/Z', intra part o/l  => o * exp(m - M) / Z'
    const float w = expf(loc.m[hh] - M[hh]) / Zp[hh];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) acc[hh][x] = loc.o[hh][x] * w;
    if (a.lse && lane == 0 && !a.paged)
      a.lse[((size_t)bi * a.h + gi * G + hh) * a.n + qi] = M[hh] + logf(Zp[hh]);
  }
  for (int s = 0; s < K; ++s) {
    const int c = idx[s];
    if (c < 0) continue;
    if (!a.paged && c >= n_cand) { set_error(a.err, kErrBadPage); continue; }
    const T* kc = chunk_ptr(kb, c, ok);
    const T* vc = chunk_ptr(vb, c, ok);
    if (!ok) { set_error(a.err, kErrBadPage); continue; }
    chunk_attend<T, D, G>(qS[warp], kc, vc, B, a.scale, r);
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float sh = a.ssel[(((size_t)bi * a.h + gi * G + hh) * n_q + qi) * K + s];
      const float w = expf(sh - M[hh]) / (Zp[hh] * r.l[hh]);
#pragma unroll
      for (int x = 0; x < D / 32; ++x) acc[hh][x] = fmaf(r.o[hh][x], w, acc[hh][x]);
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int x = 0; x < D / 32; ++x) out_row(hh)[lane + 32 * x] = from_f<T>(acc[hh][x]);
}

template <typename T, int D, int G>
static cudaError_t launch_rows(const AttendRowsArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.b * a.g * (a.paged ? 1 : a.n);
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + kRowWarps - 1) / kRowWarps;
  attend_rows_kernel<T, D, G><<<(unsigned)blocks, kRowWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t rows_by_group(const AttendRowsArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_rows<T, D, 1>(a, st);
    case 2: return launch_rows<T, D, 2>(a, st);
    case 4: return launch_rows<T, D, 4>(a, st);
    case 8: return launch_rows<T, D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_attend_rows(const AttendRowsArgs& a, cudaStream_t st) {
  if (a.n_local < 1) return cudaErrorInvalidValue;
  if (a.bf16) return a.d == 64 ? rows_by_group<__nv_bfloat16, 64>(a, st) : rows_by_group<__nv_bfloat16, 128>(a, st);
  return a.d == 64 ? rows_by_group<float, 64>(a, st) : rows_by_group<float, 128>(a, st);
}

}  // namespace hils
