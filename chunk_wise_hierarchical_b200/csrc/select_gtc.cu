// Chunk scores on the tensor cores + per-query-group Top-K for grouped-query
// attention (G > 1 query heads per KV head).  (HiLS notes, section 5.2:
// shat_{h,i,c} = q_{h,i} . kbar_{h,c} * scale + H_{h,c}; the group's selection
// key is the max over its G heads, and the group keeps the K best candidates
// c < floor(i / B) + 1 - n_local, ties to the lower chunk index.)
//
// One CTA takes 128 queries of one (sequence, KV head).  The summaries are split
// once into bf16 hi + lo parts (gtc_split_kernel), so every head's score tile is
// S_h = Q_h hi_h^T + Q_h lo_h^T on the tensor cores, accumulated in fp32 in its
// own tensor-memory region (G regions of kNc = 64 chunk columns).  Q_h, hi_h and
// lo_h come by TMA into a two-deep ring of stages, one (tile, head) pair per stage.
// Each thread then owns one query: it reads its G heads' scores 8 columns at a
// time, forms the key (the max over heads of S * scale + H), and keeps its best KP
// candidates as a list sorted by key in registers (strict comparison: candidates
// arrive in increasing chunk order, so an earlier chunk stays first among equal
// keys).  Each list entry also names a record in shared memory that holds the G
// heads' own scores of that chunk; an entering candidate takes over the record of
// the entry it pushes out, so records never move.  The per-head scores of the
// final selection are read from the records.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {

constexpr int kGtcThreads = 128;
constexpr int kGtcNc = 64;  // candidate chunks per tile (per head region)

template <int D>
struct GtcCfg {
  static constexpr uint32_t kQ = 128 * D * 2;      // Q rows of one head: D/64 sub-tiles of 16 KB
  static constexpr uint32_t kB = kGtcNc * D * 2;   // hi (or lo) summaries: D/64 sub-tiles of 8 KB
  static constexpr uint32_t kStage = kQ + 2 * kB;
};

// S is sorted in descending order and x > S[KP-1]; entries of equal key stay ahead of
// x (they came from lower chunk indices).  Shifts the tail down by one and drops (x, r)
// into its place; returns the payload of the entry that fell off the end.
template <int KP>
__device__ __forceinline__ void gtc_insert(float (&S)[KP], int (&R)[KP], float x, int r) {
#pragma unroll
  for (int j = KP - 1; j > 0; --j) {
    const bool above_prev = x > S[j - 1];
    const bool above_here = x > S[j];
    S[j] = above_prev ? S[j - 1] : (above_here ? x : S[j]);
    R[j] = above_prev ? R[j - 1] : (above_here ? r : R[j]);
  }
  if (x > S[0]) {
    S[0] = x;
    R[0] = r;
  }
}

}  // namespace

// Summaries split into bf16 hi + lo parts: hi = bf16(kbar), lo = bf16(kbar - hi).
__global__ void gtc_split_kernel(const float* __restrict__ kbar, __nv_bfloat16* __restrict__ hi,
                                 __nv_bfloat16* __restrict__ lo, size_t n4) {
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= n4) return;
  const float4 f = reinterpret_cast<const float4*>(kbar)[x];
  const float h0 = __bfloat162float(__float2bfloat16_rn(f.x)), h1 = __bfloat162float(__float2bfloat16_rn(f.y));
  const float h2 = __bfloat162float(__float2bfloat16_rn(f.z)), h3 = __bfloat162float(__float2bfloat16_rn(f.w));
  reinterpret_cast<uint2*>(hi)[x] = make_uint2(tc::pack_bf16x2(h0, h1), tc::pack_bf16x2(h2, h3));
  reinterpret_cast<uint2*>(lo)[x] = make_uint2(tc::pack_bf16x2(f.x - h0, f.y - h1), tc::pack_bf16x2(f.z - h2, f.w - h3));
}

template <int D, int G, int KP>
__global__ void __launch_bounds__(kGtcThreads, 1) select_gtc_kernel(const __grid_constant__ GtcArgs a) {
  using C = GtcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar_full[2], bar_mma[2], bar_tile;
  __shared__ uint32_t tmem_base_s;
  __shared__ float s_h[G * kGtcNc];
  __shared__ volatile int s_abort;
  // records: per list entry r, head hh, thread t (thread-minor: conflict-free)
  float* s_rec = reinterpret_cast<float*>(sm + 2 * C::kStage);

  const int t = threadIdx.x, warp = t >> 5;
  const int N = a.n, K = a.top_k, Cn = a.n_chunks;
  const int nqt = (N + 127) / 128;
  const int qt = blockIdx.x % nqt;
  const int bg = blockIdx.x / nqt;  // b * g + KV head
  const int bi = bg / a.g, gi = bg % a.g;
  const int head0 = gi * G;
  const int q0 = qt * 128;
  const int i = q0 + t;
  const bool active = i < N;
  const int n_cand = active ? n_candidates(i, a.n_local, Cn) : 0;
  const int tile_cand = n_candidates(min(N, q0 + 128) - 1, a.n_local, Cn);
  const int n_tiles = (tile_cand + kGtcNc - 1) / kGtcNc;
  const int n_pairs = n_tiles * G;

  if (t == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_full[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_mma[s]), 1);
    }
    tc::mbar_init(tc::smem_u32(&bar_tile), 1);
    tc::mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), G * kGtcNc);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const uint32_t b = tc::smem_u32(bar);
    for (uint32_t it = 0; it < a.poll; ++it) {
      if (tc::mbar_test(b, parity)) return true;
      if ((it & 1023u) == 1023u && s_abort) return false;
    }
    set_error(a.err, kErrTimeout);
    s_abort = 1;
    return false;
  };
  auto stage_u32 = [&](int s) -> uint32_t { return tc::smem_u32(sm + s * C::kStage); };
  // (thread 0) the operands of pair p = (tile p / G, head p % G) into stage p % 2, once the
  // MMAs of pair p - 2 have read it
  int loads = 0, mmas = 0;
  auto issue_load = [&](int p) -> bool {
    const int s = p % 2;
    if (p >= 2 && !wait(&bar_mma[s], (uint32_t)(((p - 2) / 2) & 1))) return false;
    const int c0 = (p / G) * kGtcNc, hh = p % G;
    const int bh = bi * a.h + head0 + hh;
    const uint32_t sQ = stage_u32(s), sHi = sQ + C::kQ, sLo = sHi + C::kB;
    const uint32_t full = tc::smem_u32(&bar_full[s]);
    tc::mbar_arrive_expect_tx(full, C::kStage);
#pragma unroll
    for (int x = 0; x < D / 64; ++x) {
      tc::tma_load_3d(sQ + x * 16384u, &a.tmap_q, x * 64, q0, bh, full);
      tc::tma_load_3d(sHi + x * (kGtcNc * 128u), &a.tmap_hi, x * 64, c0, bh, full);
      tc::tma_load_3d(sLo + x * (kGtcNc * 128u), &a.tmap_lo, x * 64, c0, bh, full);
    }
    ++loads;
    return true;
  };

  float S[KP];
  int R[KP];  // chunk | record << 16
#pragma unroll
  for (int s = 0; s < KP; ++s) {
    S[s] = -INFINITY;  // below every candidate
    R[s] = -1 & 0xffff | (s << 16);
  }
  bool failed = false;
  if (t == 0) {
    for (int p = 0; p < 2 && p < n_pairs && !failed; ++p) failed = !issue_load(p);
  }
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int c0 = tile * kGtcNc;
    for (int x = t; x < G * kGtcNc; x += kGtcThreads) {
      const int hh = x / kGtcNc, c = c0 + x % kGtcNc;
      s_h[x] = c < Cn ? a.hbias[((size_t)bi * a.h + head0 + hh) * Cn + c] : 0.f;
    }
    if (t == 0 && !failed) {
      constexpr uint32_t id = tc::make_idesc_bf16(128, kGtcNc, false, false);
      for (int hh = 0; hh < G && !failed; ++hh) {
        const int p = tile * G + hh, s = p % 2;
        if (!wait(&bar_full[s], (uint32_t)((p / 2) & 1))) {
          failed = true;
          break;
        }
        tc::fence_after_sync();
        const uint32_t sQ = stage_u32(s), sHi = sQ + C::kQ, sLo = sHi + C::kB;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t sB = part == 0 ? sHi : sLo;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t da = tc::make_desc(sQ + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
            const uint64_t db = tc::make_desc(sB + (k >> 2) * (kGtcNc * 128u) + (k & 3) * 32u, 16, 1024);
            tc::mma_bf16(tmem + hh * kGtcNc, da, db, id, (part | k) != 0);
          }
        }
        tc::mma_commit(tc::smem_u32(&bar_mma[s]));
        ++mmas;
        if (p + 2 < n_pairs && !issue_load(p + 2)) failed = true;
      }
      // the tile's scores are complete once its last MMAs are
      if (!failed) tc::mma_commit(tc::smem_u32(&bar_tile));
    }
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    if (!wait(&bar_tile, (uint32_t)(tile & 1))) failed = true;
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    tc::fence_after_sync();
    // this tile's candidates, 8 columns of every head at a time
#pragma unroll 1
    for (int cb = 0; cb < kGtcNc; cb += 8) {
      float v[G][8];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) tc::tmem_ld8(tmem + hh * kGtcNc + cb + lane_off, v[hh]);
      tc::tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + cb + u;
        float sh[G], key = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          sh[hh] = fmaf(v[hh][u], a.scale, s_h[hh * kGtcNc + cb + u]);
          key = fmaxf(key, sh[hh]);
        }
        if (c < n_cand && key > S[KP - 1]) {
          const int rec = R[KP - 1] >> 16;  // the entry pushed out leaves its record
#pragma unroll
          for (int hh = 0; hh < G; ++hh) s_rec[(rec * G + hh) * kGtcThreads + t] = sh[hh];
          gtc_insert(S, R, key, c | (rec << 16));
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();  // the tensor memory is rewritten by the next tile's MMAs
    tc::fence_after_sync();
  }
  // on the way out every MMA and copy issued has completed: the MMAs of the last pairs
  // (their commits are the newest phases), and loads that no MMA consumed
  if (t == 0) {
    for (int p = max(0, mmas - 2); p < mmas; ++p)
      tc::mbar_wait(tc::smem_u32(&bar_mma[p % 2]), (uint32_t)((p / 2) & 1), kDrainPolls);
    for (int p = mmas; p < loads; ++p)
      tc::mbar_wait(tc::smem_u32(&bar_full[p % 2]), (uint32_t)((p / 2) & 1), kDrainPolls);
  }
  if (active && !failed) {
    int32_t* idx_out = a.idx + (((size_t)bi * a.g + gi) * N + i) * K;
#pragma unroll
    for (int s = 0; s < KP; ++s) {
      if (s < K) {
        const bool ok = S[s] > -INFINITY;
        idx_out[s] = ok ? (R[s] & 0xffff) : -1;
        if (a.score) {
          const int rec = R[s] >> 16;
#pragma unroll
          for (int hh = 0; hh < G; ++hh)
            a.score[(((size_t)bi * a.h + head0 + hh) * N + i) * K + s] =
                ok ? s_rec[(rec * G + hh) * kGtcThreads + t] : -INFINITY;
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, G * kGtcNc);
}

namespace {

template <int D, int G, int KP>
constexpr size_t gtc_smem() {
  return 1024 + 2 * (size_t)GtcCfg<D>::kStage + (size_t)KP * G * kGtcThreads * 4;
}

template <int D, int G, int KP>
cudaError_t launch_gtc(const GtcArgs& a, cudaStream_t st) {
  constexpr size_t smem = gtc_smem<D, G, KP>();
  static_assert(smem <= 227 * 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(select_gtc_kernel<D, G, KP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((a.n + 127) / 128) * a.b * a.g;
  if (blocks == 0) return cudaSuccess;
  select_gtc_kernel<D, G, KP><<<(unsigned)blocks, kGtcThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t gtc_by_k(const GtcArgs& a, cudaStream_t st) {
  if (a.top_k <= 16) return launch_gtc<D, G, 16>(a, st);
  if constexpr (32 * G * kGtcThreads * 4 + 2 * GtcCfg<D>::kStage + 1024 <= 227 * 1024)
    return launch_gtc<D, G, 32>(a, st);
  return cudaErrorNotSupported;
}

// A [rows][D] bf16 tensor, rows grouped by (b * h), as a rank-3 map with 64-column boxes of
// `box_rows` rows in the 128-byte swizzle; rows past `rows` read as zeros.
bool encode_rows_map(CUtensorMap* m, const void* base, int D, int rows, int bh, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool select_gtc_supported(int d, int G, int K, bool bf16) {
  if (!bf16 || (d != 64 && d != 128) || K < 1 || K > 32) return false;
  if (G != 2 && G != 4 && G != 8) return false;
  // the records of KP = 32 entries must fit beside the stages
  if (K > 16) {
    const size_t stage = d == 64 ? GtcCfg<64>::kStage : GtcCfg<128>::kStage;
    return 32 * (size_t)G * kGtcThreads * 4 + 2 * stage + 1024 <= 227 * 1024;
  }
  return true;
}

size_t gtc_split_bytes(int b, int h, int n_chunks, int d) { return (size_t)b * h * n_chunks * d * 2; }

cudaError_t run_select_gtc(GtcArgs a, cudaStream_t st) {
  const size_t n = (size_t)a.b * a.h * a.n_chunks * a.d;
  if (n > 0) {
    gtc_split_kernel<<<(unsigned)((n / 4 + 255) / 256), 256, 0, st>>>(a.kbar, a.kbar_hi, a.kbar_lo, n / 4);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (!encode_rows_map(&a.tmap_q, a.q, a.d, a.n, a.b * a.h, 128) ||
      !encode_rows_map(&a.tmap_hi, a.kbar_hi, a.d, a.n_chunks, a.b * a.h, kGtcNc) ||
      !encode_rows_map(&a.tmap_lo, a.kbar_lo, a.d, a.n_chunks, a.b * a.h, kGtcNc))
    return cudaErrorNotSupported;
  const int G = a.h / a.g;
  if (a.d == 64) {
    switch (G) {
      case 2: return gtc_by_k<64, 2>(a, st);
      case 4: return gtc_by_k<64, 4>(a, st);
      case 8: return gtc_by_k<64, 8>(a, st);
    }
  } else {
    switch (G) {
      case 2: return gtc_by_k<128, 2>(a, st);
      case 4: return gtc_by_k<128, 4>(a, st);
      case 8: return gtc_by_k<128, 8>(a, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace hils
