// Chunk-major prefill attention + fusion on the 5th-generation tensor cores
// (tcgen05 + TMEM), bf16 inputs, fp32 accumulation, head dim 64 or 128.
// (HiLS notes, section 5.3: w_ij = exp(s_ij)/Z_{i,c} * exp(shat_{i,c})/Zhat_i;
// local branch at its exact mass, section 5.2; Tide digest, Figure 3.)
//
// The output of query row r (query i, head h) is
//     o_r = sum_{x in terms(r)} exp(x - M_r) o_{r,x} / Z'_r,   Z'_r = sum_x exp(x - M_r),
// over its selected chunks (x = shat, o = the chunk's intra-chunk softmax output) and
// its local-branch chunks (x = the chunk's exact log-mass, o likewise), M_r the max of
// the x.  Each term o_{r,x} depends on the row and one chunk only, so the terms are
// computed chunk-major:
//   1. bucketing (cm_count, cm_plan, cm_scatter, cm_desc): every valid selection
//      (b, KV head, query, slot) of the whole sequence goes into its chunk's bucket;
//      buckets are cut into tiles of 128 rows (128 / G queries x the G heads of the
//      group), and the position of each selection's rows is recorded.  The local
//      branch needs no bucketing: the local bucket of chunk c holds the queries of
//      chunks c .. c + n_local - 1, in order.
//   2. attend_cm_kernel: per tile, S = Q_tile K_c^T, P = exp(S - m) (bf16), and
//      [O | l] = P [V_c | 1] on the tensor cores (the ones tile makes column d the row
//      sum l = sum_j P_j); the epilogue stores O / l as the row's bf16 partial and, for
//      local tiles, the log-mass m + log l.
//   3. cm_fuse_kernel: per row, the inter-chunk softmax over its terms, read back from
//      the partials in slot order (results do not depend on the tile a row landed in,
//      since every MMA row depends on its own A row only).
// Tiles are full wherever a bucket has 128 rows to give, whatever the block of
// queries they come from, and a tile's result leaves the SM without a read-modify-
// write of an accumulator, so tiles are independent of each other.
//
// attend_cm_kernel: one persistent CTA per SM.  The tile list is cut into blocks of U
// consecutive tiles, block k going to CTA k % gridDim.x, so a CTA's consecutive items
// mostly share their chunk.  Warp roles (512 threads), synchronised by mbarriers with
// bounded waits:
//   warp 0 lane 0   TMA producer: K_c and V_c into a K/V stage (which also holds a tile of
//                   ones), once per change of chunk; a stage is refilled after the last
//                   P.V that read it has completed
//   warp 1 lane 0   MMA issuer: S(0), S(1), then P.V(j), S(j + 2), ...
//   warps 2-3       gather of the tile's Q rows into a Q stage (whole-row cp.async, each
//                   copy arriving on the stage's barrier when it lands); a Q stage is
//                   released by the softmax once S has been read
//   warps 4-11      two softmax warpgroups on alternate items
//   warps 12-15     epilogue: tensor memory -> registers -> bf16 partial rows in global
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {

constexpr int kCmThreads = 512;
constexpr int kCmQpb = 1024;  // queries per CTA of the bucketing kernels
constexpr float kLog2eCm = 1.4426950408889634f;
constexpr float kLn2Cm = 0.6931471805599453f;

template <int D>
struct CmCfg {
  static constexpr int NQ = D == 64 ? 6 : 4;    // Q stages, released once S has read them
  static constexpr int NKV = D == 64 ? 3 : 2;   // K/V stages, one per change of chunk
  static constexpr int NP = 2;                  // S / P slots (one per softmax warpgroup)
  static constexpr int NO = D == 64 ? 3 : 2;    // P.V output slots
  static constexpr int NF = 8;                  // ring of row maxima handed to the epilogue
  static constexpr int U = 8;                   // consecutive tiles per block of the tile schedule
  static constexpr int NV = D + 16;             // P.V columns: D values, then 16 columns of sum_j P_j
  static constexpr uint32_t kOStride = D == 64 ? 96 : 160;
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = NP * 64;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kQ = 128 * D * 2;     // D/64 swizzled sub-tiles of 128 rows (16 KB each)
  static constexpr uint32_t kK = 64 * D * 2;      // D/64 sub-tiles of 64 keys (8 KB each)
  static constexpr uint32_t kV = 64 * D * 2;
  static constexpr uint32_t kOnes = 64 * 64 * 2;  // one more V-shaped sub-tile, of bf16 1.0
  static constexpr uint32_t kKV = kK + kV + kOnes;
  static constexpr uint32_t kOffKV = NQ * kQ;
  static constexpr uint32_t kOffM = kOffKV + NKV * kKV;
  static constexpr uint32_t kSmem = kOffM + NF * 128 * 4 + 1024;
};
static_assert(CmCfg<64>::kColO + CmCfg<64>::NO * CmCfg<64>::kOStride <= 512, "tensor memory plan, d = 64");
static_assert(CmCfg<128>::kColO + CmCfg<128>::NO * CmCfg<128>::kOStride <= 512, "tensor memory plan, d = 128");
// softmax(j) follows S(j), which follows P.V(j - NP), which follows the epilogue's release
// of item j - NP - NO: a ring of NF > NP + NO maxima is never overwritten before it is read.
static_assert(CmCfg<64>::NF > CmCfg<64>::NP + CmCfg<64>::NO, "max ring");
static_assert(CmCfg<64>::kSmem <= 227 * 1024 && CmCfg<128>::kSmem <= 227 * 1024, "shared memory");

__device__ __forceinline__ void cm_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
// 2^x in one MUFU instruction (arguments <= 0; results below the smallest normal flush to 0).
__device__ __forceinline__ float cm_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// What every role needs to know of a tile.
struct CmTile {
  int bg;      // b * g + KV head
  int c;       // chunk of K_c / V_c
  int base;    // selected: index of the tile's first entry in ent_q; local: first row in the bucket
  int n_rows;  // valid rows (rows past it are padding of the 128-row MMA)
  bool local;
};

template <int G>
__device__ __forceinline__ CmTile cm_tile(const CmArgs& a, int t) {
  CmTile x;
  if (t < a.n_lt) {
    const int lb = t / a.tl, tin = t - lb * a.tl;
    x.bg = lb / a.c_all;
    x.c = lb - x.bg * a.c_all;
    x.base = tin * 128;
    x.local = true;
    const int q_hi = min(a.n, (x.c + a.n_local) * kChunk);
    x.n_rows = max(0, min(128, (q_hi - x.c * kChunk) * G - x.base));
  } else {
    const int4 d = __ldg(a.desc + (t - a.n_lt));
    x.bg = d.x;
    x.c = d.y;
    x.base = d.z;
    x.n_rows = d.w;
    x.local = false;
  }
  return x;
}

}  // namespace

// ----------------------------------------------------------------------------
// Bucketing.  Grid: (b * g) x ceil(N / kCmQpb) CTAs of 512 threads; dynamic shared
// memory c_sel ints.  A selection (query i, slot s) is valid when 0 <= c < the query's
// candidate count (others are skipped; c past it is flagged as a bad index).
__global__ void __launch_bounds__(512) cm_count_kernel(const __grid_constant__ CmArgs a) {
  extern __shared__ int s_cnt[];
  const int nqb = (a.n + kCmQpb - 1) / kCmQpb;
  const int bg = blockIdx.x / nqb, qb = blockIdx.x % nqb;
  for (int c = threadIdx.x; c < a.c_sel; c += blockDim.x) s_cnt[c] = 0;
  __syncthreads();
  const int K = a.top_k;
  const int32_t* idx = a.idx + (size_t)bg * a.n * K;
  const int e0 = qb * kCmQpb * K, e1 = min(a.n, (qb + 1) * kCmQpb) * K;
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int c = __ldg(idx + e);
    if (c < 0) continue;
    if (c >= n_candidates(e / K, a.n_local, a.c_sel)) {
      set_error(a.err, kErrBadPage);
      continue;
    }
    atomicAdd(&s_cnt[c], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < a.c_sel; c += blockDim.x)
    if (s_cnt[c]) atomicAdd(a.cnt + (size_t)bg * a.c_sel + c, s_cnt[c]);
}

// One CTA of 1024 threads: tiles per bucket, their exclusive scan, the total; clears the
// scatter cursors and the abort flag.
template <int G>
__global__ void __launch_bounds__(1024) cm_plan_kernel(const __grid_constant__ CmArgs a) {
  __shared__ int s_wsum[32];
  const int nb = a.b * a.g * a.c_sel;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (nb + 1023) / 1024;
  const int lo = min(tid * seg, nb), hi = min(lo + seg, nb);
  int sum = 0;
  for (int j = lo; j < hi; ++j) sum += (a.cnt[j] * G + 127) / 128;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < 32; ++w) {
    if (w < warp) wbase += s_wsum[w];
    total += s_wsum[w];
  }
  int run = wbase + incl - sum;
  for (int j = lo; j < hi; ++j) {
    a.toff[j] = run;
    run += (a.cnt[j] * G + 127) / 128;
    a.cur[j] = 0;
  }
  if (tid == 0) {
    a.toff[nb] = total;
    *a.n_sel = total;
    *a.abort_flag = 0;
  }
}

// Same grid as cm_count_kernel: reserve each chunk's range in its bucket, then place every
// valid selection; record the partial row of each (query, slot), -1 for the others.
template <int G>
__global__ void __launch_bounds__(512) cm_scatter_kernel(const __grid_constant__ CmArgs a) {
  extern __shared__ int s_cnt[];
  const int nqb = (a.n + kCmQpb - 1) / kCmQpb;
  const int bg = blockIdx.x / nqb, qb = blockIdx.x % nqb;
  for (int c = threadIdx.x; c < a.c_sel; c += blockDim.x) s_cnt[c] = 0;
  __syncthreads();
  const int K = a.top_k;
  const int32_t* idx = a.idx + (size_t)bg * a.n * K;
  int* pos = a.pos + (size_t)bg * a.n * K;
  const int e0 = qb * kCmQpb * K, e1 = min(a.n, (qb + 1) * kCmQpb) * K;
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int c = __ldg(idx + e);
    if (c >= 0 && c < n_candidates(e / K, a.n_local, a.c_sel)) atomicAdd(&s_cnt[c], 1);
  }
  __syncthreads();
  int* cur = a.cur + (size_t)bg * a.c_sel;
  for (int c = threadIdx.x; c < a.c_sel; c += blockDim.x)
    if (s_cnt[c]) s_cnt[c] = atomicAdd(cur + c, s_cnt[c]);  // now this CTA's first rank in bucket c
  __syncthreads();
  const int* toff = a.toff + (size_t)bg * a.c_sel;
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int c = __ldg(idx + e);
    const int i = e / K;
    int p = -1;
    if (c >= 0 && c < n_candidates(i, a.n_local, a.c_sel)) {
      const int k = atomicAdd(&s_cnt[c], 1);
      const int t0 = toff[c];  // selected tile index of the bucket's first tile
      a.ent_q[(size_t)t0 * (128 / G) + k] = (bg * G) * a.n + i;  // Q row of the group's first head
      p = (a.n_lt + t0) * 128 + k * G;
    }
    pos[e] = p;
  }
}

// Thread per bucket: the descriptors of its tiles.
template <int G>
__global__ void cm_desc_kernel(const __grid_constant__ CmArgs a) {
  const int nb = a.b * a.g * a.c_sel;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= nb) return;
  const int t0 = a.toff[j], t1 = a.toff[j + 1], cnt = a.cnt[j];
  const int bg = j / a.c_sel, c = j - bg * a.c_sel;
  for (int t = t0; t < t1; ++t)
    a.desc[t] = make_int4(bg, c, t * (128 / G), min(128, cnt * G - (t - t0) * 128));
  // the entries past the bucket's count, in its last tile, are padding
  for (int e = t0 * (128 / G) + cnt; e < t1 * (128 / G); ++e) a.ent_q[e] = -1;
}

// ----------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kCmThreads, 1) attend_cm_kernel(const __grid_constant__ CmArgs a) {
  using C = CmCfg<D>;
  constexpr int NQ = C::NQ, NKV = C::NKV, NP = C::NP, NO = C::NO, NF = C::NF;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar_q[NQ], bar_qfree[NQ], bar_kv[NKV], bar_kvfree[NKV];
  __shared__ uint64_t bar_sfull[NP], bar_pfull[NP], bar_ofull[NO], bar_ofree[NO], bar_fready[NF];
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int s_abort;
  float* s_m = reinterpret_cast<float*>(sm + C::kOffM);  // [NF][128] row maxima (log2 domain)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.n;
  // Tile schedule: blocks of U consecutive tiles, block k to CTA k % gridDim.x.  Tiles of one
  // bucket are adjacent, so consecutive items mostly share their chunk and K/V stage, and the
  // whole grid sweeps the tile list in order, so the query rows it gathers stay in L2.
  constexpr int U = C::U;
  const int n_total = a.n_lt + *a.n_sel;
  const int n_blocks = (n_total + U - 1) / U;
  const int my_blocks = (int)blockIdx.x < n_blocks ? (n_blocks - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const bool owns_last = my_blocks > 0 && (n_blocks - 1) % (int)gridDim.x == (int)blockIdx.x;
  const int n_items = my_blocks * U - (owns_last ? n_blocks * U - n_total : 0);
  auto tile_at = [&](int i) { return ((int)blockIdx.x + (i / U) * (int)gridDim.x) * U + i % U; };

  if (tid == 0) {
    for (int s = 0; s < NQ; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_q[s]), 64);  // one completion arrival per gather thread
      tc::mbar_init(tc::smem_u32(&bar_qfree[s]), 1);
    }
    for (int s = 0; s < NKV; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_kv[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_kvfree[s]), 1);
    }
    for (int s = 0; s < NP; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_sfull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_pfull[s]), 128);
    }
    for (int s = 0; s < NO; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_ofull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_ofree[s]), 128);
    }
    for (int s = 0; s < NF; ++s) tc::mbar_init(tc::smem_u32(&bar_fready[s]), 128);
    tc::mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), C::kTmemCols);
  // the ones tile after V in every K/V stage (never overwritten: the copies fill K and V only)
  for (int s = 0; s < NKV; ++s)
    for (int x = tid; x < (int)(C::kOnes / 16); x += kCmThreads)
      reinterpret_cast<uint4*>(sm + C::kOffKV + s * C::kKV + C::kK + C::kV)[x] =
          make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  auto q_u32 = [&](int s) -> uint32_t { return tc::smem_u32(sm + s * C::kQ); };
  auto kv_u32 = [&](int s) -> uint32_t { return tc::smem_u32(sm + C::kOffKV + s * C::kKV); };
  auto tile = [&](int i) -> CmTile { return cm_tile<G>(a, tile_at(i)); };
  auto same_chunk = [](const CmTile& x, const CmTile& y) { return x.bg == y.bg && x.c == y.c; };
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
  const float sc2 = a.scale * kLog2eCm;

  // Register budgets per warpgroup (setmaxnreg): the block is launched with 128 registers
  // per thread (checked on the host), 128 x 512 = 65536; the producer warpgroup gives up 64
  // per thread and the softmax warpgroups take 32 more each (the epilogue keeps 128):
  // 64 + 160 + 160 + 128 = 512 = 4 x 128, so every increase can be met.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
    if (warp == 0) {
      // ============ TMA producer: K_c and V_c, once per change of chunk (a "generation") ============
      if (lane == 0) {
        int gen = 0;
        CmTile prev{}, nxt{};
        if (n_items > 0) nxt = tile(0);
        for (int i = 0; i < n_items; ++i) {
          const CmTile tl = nxt;
          if (i + 1 < n_items) nxt = tile(i + 1);
          if (i > 0 && same_chunk(tl, prev)) continue;
          prev = tl;
          const int s = gen % NKV;
          // the last P.V of generation gen - NKV, which used this stage, has completed
          if (gen >= NKV && !wait(&bar_kvfree[s], (uint32_t)(((gen - NKV) / NKV) & 1))) break;
          const uint32_t sK = kv_u32(s), sV = sK + C::kK;
          const uint32_t full = tc::smem_u32(&bar_kv[s]);
          tc::mbar_arrive_expect_tx(full, C::kK + C::kV);
#pragma unroll
          for (int x = 0; x < D / 64; ++x) {
            tc::tma_load_3d(sK + x * 8192u, &a.tmap_k, x * 64, tl.c * kChunk, tl.bg, full);
            tc::tma_load_3d(sV + x * 8192u, &a.tmap_v, x * 64, tl.c * kChunk, tl.bg, full);
          }
          ++gen;
          if (s_abort) break;
        }
        // every issued copy has landed before the CTA's shared memory is released
        for (int g = max(0, gen - NKV); g < gen; ++g)
          tc::mbar_wait(tc::smem_u32(&bar_kv[g % NKV]), (uint32_t)((g / NKV) & 1), kDrainPolls);
      }
    } else if (warp == 1) {
      // ======================= MMA issuer =======================
      if (lane == 0) {
        constexpr uint32_t idS = tc::make_idesc_bf16(128, 64, false, false);
        constexpr uint32_t idO = tc::make_idesc_bf16(128, C::NV, false, true);
        // K/V stage of items j .. j + 3, 8 bits each (P.V(j) follows S(j) by at most NP items)
        uint32_t kvs_of = 0;
        auto issue_s = [&](int i, int kvs) {
          const int b = i % NP;
          const uint32_t sQ = q_u32(i % NQ), sK = kv_u32(kvs);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t da = tc::make_desc(sQ + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
            const uint64_t db = tc::make_desc(sK + (k >> 2) * 8192u + (k & 3) * 32u, 16, 1024);
            tc::mma_bf16(tmem + C::kColS + b * 64, da, db, idS, k > 0);
          }
          tc::mma_commit(tc::smem_u32(&bar_sfull[b]));
        };
        auto issue_pv = [&](int i) {
          const int b = i % NP, o = i % NO;
          const uint32_t sV = kv_u32((int)((kvs_of >> (8 * (i & 3))) & 0xffu)) + C::kK;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // P (bf16) sits in the first 32 columns of S's slot: 16 keys = 8 columns per
            // step.  B is V's D/64 sub-tiles followed by the ones tile, 8 KB apart (LBO).
            const uint64_t db = tc::make_desc(sV + k * 2048u, 8192, 1024);
            tc::mma_bf16_tmem_a(tmem + C::kColO + o * C::kOStride, tmem + C::kColS + b * 64 + k * 8, db, idO,
                                k > 0);
          }
          tc::mma_commit(tc::smem_u32(&bar_ofull[o]));
        };
        int next_s = 0, next_pv = 0, gen = -1;
        CmTile prev{}, nxt{};
        if (n_items > 0) nxt = tile(0);
        auto do_s = [&](int i) -> bool {
          const CmTile tl = nxt;
          if (i + 1 < n_items) nxt = tile(i + 1);
          if (i == 0 || !same_chunk(tl, prev)) ++gen;
          prev = tl;
          kvs_of = (kvs_of & ~(0xffu << (8 * (i & 3)))) | ((uint32_t)(gen % NKV) << (8 * (i & 3)));
          if (!wait(&bar_q[i % NQ], (uint32_t)((i / NQ) & 1))) return false;
          if (!wait(&bar_kv[gen % NKV], (uint32_t)((gen / NKV) & 1))) return false;
          tc::fence_async_smem();  // the gathered rows (cp.async writes) -> the tensor core
          tc::fence_after_sync();
          issue_s(i, gen % NKV);
          ++next_s;
          return true;
        };
        // S(0) .. S(NP - 1), then P.V(j), S(j + NP), ...: S(j + NP) reuses the S/P slot of
        // item j, so it never goes before P.V(j) (tcgen05 MMAs run in issue order)
        bool go = true;
        for (int i = 0; i < NP && i < n_items && go; ++i) go = do_s(i);
        for (int j = 0; j < n_items && go; ++j) {
          if (!wait(&bar_pfull[j % NP], (uint32_t)((j / NP) & 1))) break;
          if (j >= NO && !wait(&bar_ofree[j % NO], (uint32_t)(((j - NO) / NO) & 1))) break;
          tc::fence_after_sync();
          issue_pv(j);
          ++next_pv;
          if (j + NP < n_items) go = do_s(j + NP);
        }
        // every MMA issued has completed before the tensor memory is released: MMAs complete
        // in issue order, and only this thread commits, so the last commit of each ring is
        // the newest phase of its barrier
        if (next_s > 0)
          tc::mbar_wait(tc::smem_u32(&bar_sfull[(next_s - 1) % NP]), (uint32_t)(((next_s - 1) / NP) & 1),
                        kDrainPolls);
        if (next_pv > 0)
          tc::mbar_wait(tc::smem_u32(&bar_ofull[(next_pv - 1) % NO]), (uint32_t)(((next_pv - 1) / NO) & 1),
                        kDrainPolls);
      }
    } else {
      // ======================= Q gather (warps 2-3, 64 rows each) =======================
      // Each thread's copies of an item arrive on the stage's barrier by themselves once they
      // have landed (cp.async.mbarrier.arrive.noinc), so the gather runs up to NQ items ahead
      // without waiting for any of them.  Each warp decides on its own to stop (warp-
      // uniformly); the stage's barrier then misses the other warp's arrivals and the MMA
      // issuer gives up.
      // A copy instruction moves whole rows: D/8 consecutive lanes take the 16-byte pieces of
      // one row, so an instruction touches 32 / (D/8) rows, each a single line.
      constexpr int CPR = D / 8, RPI = 32 / CPR;
      const int w0 = (warp - 2) * 64;  // this warp's first row of the tile
      int issued = 0;
      // Q row offsets (row of [b*h*N]) of tile rows w0 + 2 lane and w0 + 2 lane + 1 of item i,
      // -1 for padding: closed form for local tiles; for selected tiles the entry list holds
      // the row of the group's first head, loaded two items ahead and resolved at use (so the
      // load's latency never stalls the loop)
      struct Rows {
        int v[2];
        bool raw;  // v holds entries still to be resolved
      };
      auto rows_of = [&](int i) {
        Rows rr;
        const int t = tile_at(i);
        if (t < a.n_lt) {
          const int lb = t / a.tl, tin = t - lb * a.tl;
          const int bg = lb / a.c_all, c = lb - bg * a.c_all;
          const int q_hi = min(N, (c + a.n_local) * kChunk);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int xb = tin * 128 + w0 + 2 * lane + u;
            const int q = c * kChunk + xb / G;
            rr.v[u] = q < q_hi ? (bg * G + xb % G) * N + q : -1;
          }
          rr.raw = false;
        } else {
          const int base = (t - a.n_lt) * (128 / G);
#pragma unroll
          for (int u = 0; u < 2; ++u) rr.v[u] = __ldg(a.ent_q + base + (w0 + 2 * lane + u) / G);
          rr.raw = true;
        }
        return rr;
      };
      auto resolve = [&](const Rows& rr, int u) {
        const int e = rr.v[u];
        return !rr.raw ? e : e < 0 ? -1 : e + ((w0 + 2 * lane + u) % G) * N;
      };
      Rows r0{{-1, -1}, false}, r1{{-1, -1}, false};
      if (n_items > 0) r0 = rows_of(0);
      if (n_items > 1) r1 = rows_of(1);
      for (int i = 0; i < n_items; ++i) {
        const int s = i % NQ;
        if (i >= NQ && !__all_sync(0xffffffffu, wait(&bar_qfree[s], (uint32_t)(((i - NQ) / NQ) & 1)))) break;
        const int c0 = resolve(r0, 0), c1 = resolve(r0, 1);
        r0 = r1;
        if (i + 2 < n_items) r1 = rows_of(i + 2);
        const uint32_t sQ = q_u32(s);
        const int ch = lane % CPR;
#pragma unroll 4
        for (int k = 0; k < 64 / RPI; ++k) {
          const int x = k * RPI + lane / CPR;  // row within this warp's 64
          const int v0 = __shfl_sync(0xffffffffu, c0, x >> 1), v1 = __shfl_sync(0xffffffffu, c1, x >> 1);
          const int ro = (x & 1) ? v1 : v0;
          if (ro >= 0)
            tc::cp_async16(sQ + (uint32_t)(ch >> 3) * 16384u + tc::sw128_chunk(w0 + x, ch & 7),
                           a.q + (size_t)ro * D + ch * 8);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(&bar_q[s]))
                     : "memory");
        ++issued;
        if (__any_sync(0xffffffffu, s_abort != 0)) break;
      }
      // no copy, and no completion arrival, may still be in flight when the CTA ends
      asm volatile("cp.async.wait_all;" ::: "memory");
      for (int j = max(0, issued - NQ); j < issued; ++j)
        tc::mbar_wait(tc::smem_u32(&bar_q[j % NQ]), (uint32_t)((j / NQ) & 1), kDrainPolls);
    }
  } else if (warp < 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 160;");
    // ======================= softmax (two warpgroups, alternating items) =======================
    const int wg = (warp - 4) >> 2;  // items i with i % 2 == wg; S slot wg
    const int t = (tid - 128) & 127;  // tile row == TMEM lane
    const int wq = warp & 3;          // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    CmTile nxt{};
    if (wg < n_items) nxt = tile(wg);
    for (int i = wg; i < n_items; i += 2) {
      const int b = i % NP;
      const CmTile tl = nxt;
      if (i + 2 < n_items) nxt = tile(i + 2);
      // the warp leaves together (the tensor-memory loads below are warp-collective)
      if (!__all_sync(0xffffffffu, wait(&bar_sfull[b], (uint32_t)((i / NP) & 1)))) break;
      tc::fence_after_sync();
      if (t == 0) cm_arrive(tc::smem_u32(&bar_qfree[i % NQ]));  // S(i) has read its Q stage
      const bool row_ok = t < tl.n_rows;
      float m2 = 0.f;
      if (wq * 32 < tl.n_rows) {
        float s[64];
        tc::tmem_ld32(tmem + C::kColS + b * 64 + lane_off, s);
        tc::tmem_ld32(tmem + C::kColS + b * 64 + 32 + lane_off, s + 32);
        tc::tmem_wait_ld();
        // P = exp2(S * c - m), m = max_j S_j * c (log2 domain).  Local tiles mask the keys
        // after the query in its own chunk: key j is visible when j <= (row in bucket) / G.
        const int jmax = tl.local ? (tl.base + t) / G : 63;
        if (!tl.local && sc2 > 0.f) {
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
          for (int j = 8; j < 64; ++j) mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          const float mr = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                 fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
          m2 = mr * sc2;
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] = cm_ex2(fmaf(s[j], sc2, -m2));
        } else {
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = j <= jmax ? s[j] * sc2 : -INFINITY;
            mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          }
          m2 = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                     fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] = cm_ex2(s[j] - m2);
        }
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = row_ok ? tc::pack_bf16x2(s[2 * j], s[2 * j + 1]) : 0u;
        tc::tmem_st32(tmem + C::kColS + b * 64 + lane_off, pk);
      }
      if (tl.local) s_m[(i % NF) * 128 + t] = m2;
      tc::tmem_wait_st();
      tc::fence_before_sync();
      cm_arrive(tc::smem_u32(&bar_pfull[b]));
      cm_arrive(tc::smem_u32(&bar_fready[i % NF]));
    }
  } else {
    // ======================= epilogue (keeps the launch budget of 128) =======================
    const int t = tid - 384;
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    // stores 32 columns of the row, scaled by inv, as bf16
    auto store32 = [&](__nv_bfloat16* dst, const float* v, float inv) {
      uint4 w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        w[q] = make_uint4(tc::pack_bf16x2(v[8 * q] * inv, v[8 * q + 1] * inv),
                          tc::pack_bf16x2(v[8 * q + 2] * inv, v[8 * q + 3] * inv),
                          tc::pack_bf16x2(v[8 * q + 4] * inv, v[8 * q + 5] * inv),
                          tc::pack_bf16x2(v[8 * q + 6] * inv, v[8 * q + 7] * inv));
#pragma unroll
      for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(dst)[q] = w[q];
    };
    int gen = -1;
    CmTile prev{}, nxt{};
    if (n_items > 0) nxt = tile(0);
    for (int i = 0; i < n_items; ++i) {
      const int o = i % NO;
      const CmTile tl = nxt;
      if (i + 1 < n_items) nxt = tile(i + 1);
      if (i == 0 || !same_chunk(tl, prev)) ++gen;
      prev = tl;
      const bool ok = __all_sync(0xffffffffu, wait(&bar_ofull[o], (uint32_t)((i / NO) & 1)) &&
                                                  wait(&bar_fready[i % NF], (uint32_t)((i / NF) & 1)));
      if (!ok) break;
      tc::fence_after_sync();
      const int tg = tile_at(i);
      const bool row_ok = t < tl.n_rows;
      const uint32_t base = tmem + C::kColO + o * C::kOStride + lane_off;
      const bool quad = wq * 32 < tl.n_rows;
      float l[1], va[32], vb[32];
      if (quad) {
        tc::tmem_ld1(base + D, l);
        tc::tmem_ld32(base, va);
        tc::tmem_ld32(base + 32, vb);
        tc::tmem_wait_ld();
      }
      __nv_bfloat16* dst = a.part + ((size_t)tg * 128 + t) * D;
      const float inv = quad ? 1.0f / l[0] : 0.f;
      if constexpr (D == 128) {
        // the first half goes out first, then the second half is read
        if (quad && row_ok) {
          store32(dst, va, inv);
          store32(dst + 32, vb, inv);
        }
        if (quad) {
          tc::tmem_ld32(base + 64, va);
          tc::tmem_ld32(base + 96, vb);
          tc::tmem_wait_ld();
        }
      }
      tc::fence_before_sync();
      cm_arrive(tc::smem_u32(&bar_ofree[o]));  // item i has left tensor memory
      if (quad && row_ok) {
        store32(dst + D - 64, va, inv);
        store32(dst + D - 32, vb, inv);
        if (tl.local) a.plse[(size_t)tg * 128 + t] = (s_m[(i % NF) * 128 + t] + log2f(l[0])) * kLn2Cm;
      }
      // the last item of its chunk: P.V of every item that read this K/V stage has completed
      if (t == 0 && (i + 1 == n_items || !same_chunk(tl, nxt))) cm_arrive(tc::smem_u32(&bar_kvfree[gen % NKV]));
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0 && s_abort) atomicOr(a.abort_flag, 1);
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
}

// ----------------------------------------------------------------------------
// Fusion: D/8 lanes per row (8 elements each), rows in [b, h, N] order.
template <int D, int G>
__global__ void __launch_bounds__(256) cm_fuse_kernel(const __grid_constant__ CmArgs a) {
  constexpr int LPR = D / 8;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gid / LPR;
  const int ln = (int)(gid % LPR);
  const long long n_rows = (long long)a.b * a.h * a.n;
  if (row >= n_rows || *a.abort_flag) return;
  const int N = a.n, K = a.top_k;
  const int i = (int)(row % N);
  const int bh = (int)(row / N);
  const int bi = bh / a.h, head = bh % a.h, gi = head / G, hh = head % G;
  const int bg = bi * a.g + gi;
  const int own = i / kChunk;
  const int* pos = a.pos + ((size_t)bg * N + i) * K;
  const float* sc = a.ssel + ((size_t)bh * N + i) * K;
  // the row's terms: local-branch chunks (log-mass) and valid selections (shat)
  float M = -INFINITY;
  for (int l = 0; l < a.n_local && own - l >= 0; ++l) {
    const int c = own - l;
    const long long pr = ((long long)(bg * a.c_all + c) * a.tl) * 128 + (long long)(i - c * kChunk) * G + hh;
    M = fmaxf(M, __ldg(a.plse + pr));
  }
  for (int s = 0; s < K; ++s)
    if (__ldg(pos + s) >= 0) M = fmaxf(M, __ldg(sc + s));
  float Z = 0.f, acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u] = 0.f;
  auto accumulate = [&](float w, const uint4& pv) {
    const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[u]));
      acc[2 * u] = fmaf(w, f.x, acc[2 * u]);
      acc[2 * u + 1] = fmaf(w, f.y, acc[2 * u + 1]);
    }
  };
  for (int l = 0; l < a.n_local && own - l >= 0; ++l) {
    const int c = own - l;
    const long long pr = ((long long)(bg * a.c_all + c) * a.tl) * 128 + (long long)(i - c * kChunk) * G + hh;
    const float w = expf(__ldg(a.plse + pr) - M);
    Z += w;
    accumulate(w, __ldg(reinterpret_cast<const uint4*>(a.part + pr * D + ln * 8)));
  }
  // the selections in batches of 8: their positions and scores, then their 8 partial rows,
  // all in flight before any is used
  for (int s0 = 0; s0 < K; s0 += 8) {
    int p[8];
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      p[u] = s0 + u < K ? __ldg(pos + s0 + u) : -1;
      x[u] = p[u] >= 0 ? __ldg(sc + s0 + u) : 0.f;
    }
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = p[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.part + ((long long)p[u] + hh) * D + ln * 8))
                       : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (p[u] >= 0) {
        const float w = expf(x[u] - M);
        Z += w;
        accumulate(w, v[u]);
      }
    }
  }
  const float inv = 1.0f / Z;
  uint4 o;
  o.x = tc::pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = tc::pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = tc::pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = tc::pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(a.out + (size_t)row * D + ln * 8) = o;
  if (a.lse && ln == 0) a.lse[row] = M + logf(Z);
}

// ----------------------------------------------------------------------------
namespace {

template <int D, int G>
bool cm_regs_ok() {
  static int ok = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (ok < 0) {
    cudaFuncAttributes fa{};
    ok = cudaFuncGetAttributes(&fa, attend_cm_kernel<D, G>) == cudaSuccess && fa.numRegs == 128;
  }
  return ok == 1;
}

int sm_count() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 0;
  });
  return n;
}

template <int D, int G>
cudaError_t launch_cm(const CmArgs& a, cudaStream_t st) {
  if (!cm_regs_ok<D, G>()) return cudaErrorNotSupported;
  const int nb = a.b * a.g * a.c_sel;
  const int nqb = (a.n + kCmQpb - 1) / kCmQpb;
  const size_t cnt_smem = (size_t)a.c_sel * 4;
  cudaError_t e;
  if (nb > 0) {
    if ((e = cudaMemsetAsync(a.cnt, 0, (size_t)nb * 4, st)) != cudaSuccess) return e;
  }
  if (nb > 0 && a.top_k > 0) {
    if (cnt_smem > 48 * 1024) {
      if ((e = cudaFuncSetAttribute(cm_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cnt_smem)) !=
              cudaSuccess ||
          (e = cudaFuncSetAttribute(cm_scatter_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)cnt_smem)) != cudaSuccess)
        return e;
    }
    cm_count_kernel<<<a.b * a.g * nqb, 512, cnt_smem, st>>>(a);
  }
  cm_plan_kernel<G><<<1, 1024, 0, st>>>(a);
  // the scatter runs whenever there are slots: it also marks every invalid slot (-1), which
  // the fusion relies on (with no complete chunk, every slot is invalid)
  if (a.top_k > 0) cm_scatter_kernel<G><<<a.b * a.g * nqb, 512, cnt_smem, st>>>(a);
  if (nb > 0 && a.top_k > 0) cm_desc_kernel<G><<<(nb + 255) / 256, 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  constexpr size_t smem = CmCfg<D>::kSmem;
  if ((e = cudaFuncSetAttribute(attend_cm_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  const int grid = sm_count();
  if (grid <= 0) return cudaErrorNoDevice;
  attend_cm_kernel<D, G><<<grid, kCmThreads, smem, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long threads = (long long)a.b * a.h * a.n * (D / 8);
  cm_fuse_kernel<D, G><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t cm_by_group(const CmArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_cm<D, 1>(a, st);
    case 2: return launch_cm<D, 2>(a, st);
    case 4: return launch_cm<D, 4>(a, st);
    case 8: return launch_cm<D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool cm_shape_supported(int d, int G, int K, int N, int n_local) {
  if (d != 64 && d != 128) return false;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (K < 0 || K > 64 || n_local < 1 || n_local > 128) return false;
  if (N / kChunk > 32767) return false;
  return true;
}

bool cm_kernel_ready(int d, int G) {
  if (d == 64) {
    switch (G) {
      case 1: return cm_regs_ok<64, 1>();
      case 2: return cm_regs_ok<64, 2>();
      case 4: return cm_regs_ok<64, 4>();
      case 8: return cm_regs_ok<64, 8>();
    }
  } else if (d == 128) {
    switch (G) {
      case 1: return cm_regs_ok<128, 1>();
      case 2: return cm_regs_ok<128, 2>();
      case 4: return cm_regs_ok<128, 4>();
      case 8: return cm_regs_ok<128, 8>();
    }
  }
  return false;
}

CmScratch cm_scratch(int b, int h, int g, int n, int d, int K, int n_local) {
  CmScratch S{};
  const int G = h / g;
  S.c_sel = n / kChunk;
  S.c_all = (n + kChunk - 1) / kChunk;
  S.tl = (kChunk * n_local * G + 127) / 128;
  const size_t nb = (size_t)b * g * S.c_sel;
  const size_t n_lt = (size_t)b * g * S.c_all * S.tl;
  const size_t max_sel = ((size_t)b * g * n * K * G + 127) / 128 + nb;
  S.n_lt = (int)n_lt;
  S.max_sel = (int)max_sel;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t off = 0;
  S.cnt = off; off = up(off + (nb + 1) * 4);
  S.cur = off; off = up(off + (nb + 1) * 4);
  S.toff = off; off = up(off + (nb + 1) * 4);
  S.n_sel = off; off = up(off + 4);
  S.abort_flag = off; off = up(off + 4);
  S.desc = off; off = up(off + (max_sel + 1) * 16);
  S.ent_q = off; off = up(off + (max_sel + 1) * (128 / G) * 4);
  S.pos = off; off = up(off + (size_t)b * g * n * K * 4 + 4);
  S.part = off; off = up(off + (n_lt + max_sel) * 128 * d * 2);
  S.plse = off; off = up(off + n_lt * 128 * 4);
  S.total = off;
  return S;
}

cudaError_t run_attend_cm(CmArgs a, cudaStream_t st) {
  if (!encode_kv_tensor_map(&a.tmap_k, a.k, a.d, a.n, a.b * a.g) ||
      !encode_kv_tensor_map(&a.tmap_v, a.v, a.d, a.n, a.b * a.g))
    return cudaErrorNotSupported;
  return a.d == 64 ? cm_by_group<64>(a, st) : cm_by_group<128>(a, st);
}

}  // namespace hils
