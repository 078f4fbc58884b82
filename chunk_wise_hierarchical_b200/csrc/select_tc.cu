// Chunk scores on the tensor cores + per-query Top-K (HiLS notes, section
// 5.2: shat_{i,c} = q_i . kbar_c * scale + H_c, I_i = the K best candidates
// c < floor(i / B)), for one query head per KV head (G = 1) and K <= 32.
//
// One CTA scores 128 queries of one (sequence, head) against tiles of 128
// candidate chunks.  The fp32 summaries are split on the fly into bf16
// hi + lo parts (hi = bf16(kbar), lo = bf16(kbar - hi)) and both products
// accumulate into one fp32 TMEM tile, S = Q.hi^T + Q.lo^T, which keeps the
// score error near 2^-17 of |q||kbar| (well inside the 1e-3 tie band the
// selection is judged by).  Each thread then owns one query row: it reads its
// scores from TMEM 32 columns at a time, adds H_c and keeps its best KP
// (score, chunk) pairs as a list sorted by score in registers.  Candidates
// arrive in increasing chunk order, so a strict comparison on the fp32 score
// alone already puts an earlier (lower-index) chunk first among equal scores:
// a candidate enters only if its score is above the list's last, and is then
// inserted by one unrolled compare-and-shift pass.  Non-finite scores never
// enter (they are not candidates).
#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {
constexpr int kSelThreads = 128;
constexpr int kNc = 128;  // candidate chunks per tile

// S is sorted in descending order and x > S[KP-1]; entries of equal score stay
// ahead of x (they came from lower chunk indices).  Shifts the tail down by one
// and drops (x, c) into its place.
template <int KP>
__device__ __forceinline__ void sorted_insert_f(float (&S)[KP], int (&I)[KP], float x, int c) {
#pragma unroll
  for (int j = KP - 1; j > 0; --j) {
    const bool above_prev = x > S[j - 1];
    const bool above_here = x > S[j];
    S[j] = above_prev ? S[j - 1] : (above_here ? x : S[j]);
    I[j] = above_prev ? I[j - 1] : (above_here ? c : I[j]);
  }
  if (x > S[0]) {
    S[0] = x;
    I[0] = c;
  }
}
}  // namespace

template <int D, int KP>
__global__ void __launch_bounds__(kSelThreads) select_tc_kernel(SelectArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar_mma;
  __shared__ uint32_t tmem_base_s;
  __shared__ float s_h[kNc];

  const int t = threadIdx.x, warp = t >> 5;
  const int N = a.n, K = a.top_k, C = a.n_chunks;
  const int nqt = (N + 127) / 128;
  const int qt = blockIdx.x % nqt;
  const int hq = blockIdx.x / nqt;  // b * h + head (G = 1: KV head == query head)
  const int q0 = qt * 128;
  const int i = q0 + t;
  const bool active = i < N;
  const int n_cand = active ? n_candidates(i, a.n_local, C) : 0;
  const int tile_cand = n_candidates(min(N, q0 + 128) - 1, a.n_local, C);

  // shared memory: Q tile [128 x D] | kbar hi [kNc x D] | kbar lo [kNc x D], 128B-swizzled
  const uint32_t sQ = tc::smem_u32(sm);
  const uint32_t sHi = sQ + 128 * D * 2;
  const uint32_t sLo = sHi + kNc * D * 2;

  if (t == 0) {
    tc::mbar_init(tc::smem_u32(&bar_mma), 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), kNc);
  // Q tile: rows of the 128 queries (rows past N are zero)
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)hq * N + q0) * D;
  constexpr int CH = D / 8;
  for (int x = t; x < 128 * CH; x += kSelThreads) {
    const int r = x / CH, ch = x % CH;
    const bool ok = q0 + r < N;
    tc::cp_async16(sQ + (uint32_t)(ch >> 3) * 16384u + tc::sw128_chunk(r, ch & 7), qg + (ok ? (size_t)r * D + ch * 8 : 0),
                   ok ? 16 : 0);
  }
  tc::cp_async_wait_all();
  tc::fence_async_smem();  // the Q tile is read by the tensor core
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  float S[KP];
  int I[KP];
#pragma unroll
  for (int s = 0; s < KP; ++s) {
    S[s] = -INFINITY;  // below every candidate
    I[s] = -1;
  }
  uint32_t phase = 0;
  bool failed = false;
  for (int c0 = 0; c0 < tile_cand; c0 += kNc) {
    const int nc = min(kNc, tile_cand - c0);
    // summaries of this tile, split into bf16 hi + lo, written in the swizzled layout
    const float* kb = a.kbar + ((size_t)hq * C + c0) * D;
    for (int x = t; x < kNc * (D / 8); x += kSelThreads) {
      const int r = x / (D / 8), ch = x % (D / 8);
      uint4 hi4 = make_uint4(0, 0, 0, 0), lo4 = make_uint4(0, 0, 0, 0);
      if (r < nc) {
        const float4 f0 = *reinterpret_cast<const float4*>(kb + (size_t)r * D + ch * 8);
        const float4 f1 = *reinterpret_cast<const float4*>(kb + (size_t)r * D + ch * 8 + 4);
        const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
        uint32_t h[4], l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float h0 = __bfloat162float(__float2bfloat16_rn(f[2 * u]));
          const float h1 = __bfloat162float(__float2bfloat16_rn(f[2 * u + 1]));
          h[u] = tc::pack_bf16x2(h0, h1);
          l[u] = tc::pack_bf16x2(f[2 * u] - h0, f[2 * u + 1] - h1);
        }
        hi4 = make_uint4(h[0], h[1], h[2], h[3]);
        lo4 = make_uint4(l[0], l[1], l[2], l[3]);
      }
      const uint32_t o = (uint32_t)(ch >> 3) * (kNc * 128u) + tc::sw128_chunk(r, ch & 7);
      *reinterpret_cast<uint4*>(sm + (sHi - sQ) + o) = hi4;
      *reinterpret_cast<uint4*>(sm + (sLo - sQ) + o) = lo4;
    }
    for (int x = t; x < kNc; x += kSelThreads) s_h[x] = x < nc ? a.hbias[(size_t)hq * C + c0 + x] : 0.f;
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (t == 0) {
      constexpr uint32_t id = tc::make_idesc_bf16(128, kNc, false, false);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t sB = part == 0 ? sHi : sLo;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t da = tc::make_desc(sQ + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
          const uint64_t db = tc::make_desc(sB + (k >> 2) * (kNc * 128u) + (k & 3) * 32u, 16, 1024);
          tc::mma_bf16(tmem, da, db, id, (part | k) != 0);
        }
      }
      tc::mma_commit(tc::smem_u32(&bar_mma));
    }
    if (!tc::mbar_wait(tc::smem_u32(&bar_mma), phase, a.poll)) {
      set_error(a.err, kErrTimeout);
      failed = true;
    }
    if (__syncthreads_or(failed)) {
      // give up: the MMAs committed above may still be running; they finish (a wait with
      // the drain bound) before the tensor memory is released below
      tc::mbar_wait(tc::smem_u32(&bar_mma), phase, kDrainPolls);
      failed = true;
      break;
    }
    phase ^= 1u;
    tc::fence_after_sync();
    // this tile's candidates, 32 TMEM columns at a time.  The candidates above the list's
    // last score are first queued, in chunk order, in shared memory (the summary tiles are
    // free once the MMA has read them); the queue is then inserted in order, each entry
    // checked again against the rising threshold, so every decision is the one a candidate-
    // by-candidate insertion would take.  A warp then runs as many insertions as its longest
    // queue rather than one for every candidate some lane keeps.
    float* qx = reinterpret_cast<float*>(sm + (sHi - sQ));  // [32][128], thread-minor
    int* qc = reinterpret_cast<int*>(qx + 32 * kSelThreads);
#pragma unroll 1
    for (int cb = 0; cb < nc; cb += 32) {
      float sv[32];
      tc::tmem_ld32(tmem + cb + lane_off, sv);
      tc::tmem_wait_ld();
      const float thr = S[KP - 1];
      int cnt = 0;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int c = c0 + cb + u;
        const float x = fmaf(sv[u], a.scale, s_h[cb + u]);
        if (c < n_cand && x > thr) {
          qx[cnt * kSelThreads + t] = x;
          qc[cnt * kSelThreads + t] = c;
          ++cnt;
        }
      }
#pragma unroll 1
      for (int e = 0; e < cnt; ++e) {
        const float x = qx[e * kSelThreads + t];
        if (x > S[KP - 1]) sorted_insert_f(S, I, x, qc[e * kSelThreads + t]);
      }
    }
    tc::fence_before_sync();
    __syncthreads();  // TMEM and the summary tiles are reused by the next tile
    tc::fence_after_sync();
  }
  // the list is already in descending order; G = 1, so the key is the head's own score
  if (active && !failed) {
    int32_t* idx_out = a.idx + ((size_t)hq * N + i) * K;
    float* sc_out = a.score ? a.score + ((size_t)hq * N + i) * K : nullptr;
#pragma unroll
    for (int s = 0; s < KP; ++s) {
      if (s < K) {
        idx_out[s] = I[s];
        if (sc_out) sc_out[s] = I[s] >= 0 ? S[s] : -INFINITY;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kNc);
}

static size_t select_tc_smem(int D) { return 1024 + (size_t)128 * D * 2 + (size_t)2 * kNc * D * 2; }

bool select_tc_supported(int d, int G, int K, bool bf16) {
  return bf16 && G == 1 && (d == 64 || d == 128) && K >= 1 && K <= 32;
}

template <int D, int KP>
static cudaError_t launch_select_tc(const SelectArgs& a, cudaStream_t st) {
  const size_t smem = select_tc_smem(D);
  cudaError_t e = cudaFuncSetAttribute(select_tc_kernel<D, KP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((a.n + 127) / 128) * a.b * a.h;
  if (blocks == 0) return cudaSuccess;
  select_tc_kernel<D, KP><<<(unsigned)blocks, kSelThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t run_select_tc(const SelectArgs& a, cudaStream_t st) {
  if (a.top_k <= 16) return a.d == 64 ? launch_select_tc<64, 16>(a, st) : launch_select_tc<128, 16>(a, st);
  return a.d == 64 ? launch_select_tc<64, 32>(a, st) : launch_select_tc<128, 32>(a, st);
}

}  // namespace hils
