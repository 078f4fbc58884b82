// Selected-chunk + own-chunk attention with the inter-chunk fusion on the
// 5th-generation tensor cores, bf16 inputs, fp32 accumulation, head dim 64.
// (HiLS notes, section 5.3: w_ij = exp(s_ij)/Z_{i,c} * exp(shat_{i,c})/Zhat_i;
// Tide digest, Figure 3.)
//
// Work decomposition: as in the row-owner kernel of attend_tc.cu, one CTA owns
// QB consecutive queries of one (sequence, KV head) and the G query heads of
// the group, R = QB * G = 512 rows whose fp32 output accumulators stay in
// shared memory.  The rows' selections are bucketed by chunk and cut into
// 128-row work items (own-chunk items first); per item
//     S = Q_tile K_c^T        tcgen05, A = Q rows from TENSOR MEMORY, B = K_c (smem)
//     P = f * exp(S - m)      registers -> bf16 -> tensor memory (S's slot)
//     O = P V_c               tcgen05, A = P from tensor memory, B = V_c (smem)
//     acc[row] (=|+=) O[row]  shared memory
// Differences from the first kernel, each aimed at its measured stalls:
//   * The gathered query rows never touch shared memory: the two softmax
//     warpgroups, which own alternate items, load the rows of their item after
//     next from global memory (L1/L2) into registers two items ahead and store
//     them into a tensor-memory Q slot with tcgen05.st, so the gather's latency
//     hides behind two items of work and the S MMA reads no shared memory for A.
//   * K_c and V_c come by TMA into a 3-deep ring (one mbarrier per stage).
//   * Bucket order keeps the epilogue's read-modify-write of the fp32
//     accumulators free of bank conflicts where it can: rows are interleaved by
//     the residue class (row mod 8) that the padded accumulator rows spread over
//     the banks, so each group of 8 tile rows (one shared-memory phase of 16-byte
//     accesses) hits 8 distinct bank groups wherever the classes allow it.
//   * An item's rows fill the 32-lane quadrants starting at quadrant 2 (i % 2),
//     so the items of the two softmax warpgroups, which run at the same time,
//     mostly use different sub-partitions of the SM.
//   * The tensor core computes each row's softmax denominator: P.V runs over 80
//     columns, V followed by a tile of ones, so column 64 holds sum_j P_j and the
//     softmax warps skip the row sum and the scaling; the epilogue applies the
//     row's scale (inter-chunk weight / sum) in the same FMA that accumulates.
// Warp roles (512 threads), synchronised by mbarriers with bounded waits:
//   warp 0 lane 0   TMA producer: K_c and V_c of item i into stage i % 3
//   warp 1 lane 0   MMA issuer: S(i) and P.V(j) as their inputs become ready
//   warps 4-11      two softmax warpgroups (items i % 2), also the Q loaders
//   warps 12-15     epilogue: tensor memory -> registers -> shared memory
// On a timed-out wait every role stops; the producer and the MMA issuer then
// wait (bounded) for what they issued before the tensor memory is released.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {

constexpr int kThreads3 = 512;
constexpr float kLog2e3 = 1.4426950408889634f;
constexpr uint32_t kOwnFlag3 = 0x80000000u;

struct Cfg3 {
  static constexpr int D = 64;
  static constexpr int NS = 3;  // K/V stages
  static constexpr int NP = 2;  // S/P slots
  static constexpr int NQ = 2;  // Q slots (a softmax warpgroup refills slot i % 2 once S(i) is done)
  static constexpr int NO = 3;  // P.V output slots, >= NS
  static constexpr int NF = 8;  // ring of per-row output scales handed from softmax to epilogue
  static constexpr int kRows = 512;
  static constexpr int NV = D + 16;  // P.V columns: D values, then 16 columns of sum_j P_j
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kOStride = 96;                 // output slots: NO x 96 (NV used)
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = NO * kOStride;         // S/P slots: NP x 64 columns
  static constexpr uint32_t kColQ = kColS + NP * 64;       // Q slots: NQ x D/2 columns (bf16 pairs)
  static constexpr uint32_t kStageK = 64 * D * 2, kStageV = 64 * D * 2;
  static constexpr uint32_t kStage = kStageK + kStageV;  // multiple of 1024
  static constexpr uint32_t kOnes = 64 * 64 * 2;         // 64 keys x 64 columns of bf16 1.0
};
static_assert(Cfg3::kColQ + Cfg3::NQ * Cfg3::D / 2 <= Cfg3::kTmemCols, "tensor memory plan");
static_assert(Cfg3::NO >= Cfg3::NS, "the producer waits for P.V(i - NS) on the output ring");
// softmax(j) follows S(j), which follows P.V(j - NP), which follows the epilogue's release of
// item j - NP - NO: a ring of NF > NP + NO scale slots is never overwritten before it is read
static_assert(Cfg3::NF > Cfg3::NP + Cfg3::NO, "scale ring");

constexpr uint32_t kAccStride = Cfg3::D * 4 + 16;  // fp32 accumulator row + 16 bytes of padding

struct Smem3 {
  uint32_t stage, ones, o, list, off, items, rowm, rowz, cnt, cur, fsc, total;
};

__host__ __device__ inline uint32_t align3(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline int max_items3(int G, int qb, int K, int n_cand) {
  const int own_tiles = (qb / 64 + 2) * ((64 * G + 127) / 128);
  return own_tiles + n_cand + (qb * K * G + 127) / 128 + 1;
}

// Classes of the conflict-free bucket order: the residue (row mod 8) of a
// selection entry's first row is (query offset * G) mod 8, so 8 / G classes.
__host__ __device__ constexpr int n_classes(int G) { return G >= 8 ? 1 : 8 / G; }

// Tile row t (the TMEM lane) of item i holds the item's list row x: rows go to the
// 32-lane quadrants in order starting at quadrant 2 * (i % 2), so an item of up to 64 rows
// fills two quadrants and consecutive items (one per softmax warpgroup, running at the
// same time) use the other two sub-partitions of the SM.  Within a quadrant, list rows
// stay consecutive, so each 8-row shared-memory phase sees 8 consecutive list rows.
__device__ __forceinline__ int list_row(int i, int t) { return ((((t >> 5) - 2 * (i & 1)) & 3) << 5) | (t & 31); }
// Whether quadrant q of item i holds any of its n_rows rows.
__device__ __forceinline__ bool quad_used(int i, int q, int n_rows) { return ((((q - 2 * (i & 1)) & 3)) << 5) < n_rows; }

__host__ __device__ inline Smem3 layout3(int G, int qb, int K, int n_cand) {
  Smem3 L;
  uint32_t off = 0;
  L.stage = off; off += Cfg3::NS * Cfg3::kStage;
  L.ones = off; off += Cfg3::kOnes;
  L.o = off; off += (uint32_t)qb * G * kAccStride;
  L.list = off; off = align3(off + (uint32_t)qb * K * 2, 16);
  L.off = off; off = align3(off + (uint32_t)(2 * n_cand + 2) * 4, 16);
  L.items = off; off = align3(off + (uint32_t)max_items3(G, qb, K, n_cand) * 4, 16);
  L.rowm = off; off += (uint32_t)qb * G * 4;
  L.rowz = off; off += (uint32_t)qb * G * 4;
  L.cnt = off; off += (uint32_t)(n_cand + 1) * 16;  // per chunk: 8 16-bit counters (one per class)
  L.cur = off; off += (uint32_t)(n_cand + 1) * 16;  // scatter cursors, same packing
  L.fsc = off; off += Cfg3::NF * 128 * 4;            // per tile row output scale, ring of NF items
  L.total = align3(off, 16);
  return L;
}

__device__ __forceinline__ float4* acc_f4(unsigned char* base, uint32_t o_off, int r, int j4) {
  // float4 j4 of row r; rows are padded by 16 bytes, so the bank group of the access is
  // (r + j4) mod 8 and rows of 8 distinct residues never collide
  return reinterpret_cast<float4*>(base + o_off + (size_t)r * kAccStride + (size_t)j4 * 16);
}

__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool bar_or(int id, int n, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}

// 2^x in one MUFU instruction; arguments are <= 0 here (logits minus their max), and a
// result below the smallest normal float flushes to zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Exclusive scan of v[0..n) in place over the whole block; returns the total.
__device__ int scan3(int* v, int n, int* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (n + kThreads3 - 1) / kThreads3;
  const int lo = min(tid * seg, n), hi = min(lo + seg, n);
  int sum = 0;
  for (int c = lo; c < hi; ++c) sum += v[c];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < kThreads3 / 32; ++w) {
    if (w < warp) wbase += wsum[w];
    total += wsum[w];
  }
  int run = wbase + incl - sum;
  for (int c = lo; c < hi; ++c) {
    const int x = v[c];
    v[c] = run;
    run += x;
  }
  __syncthreads();
  return total;
}

// 16-bit counter `cls` of the 8 packed into a chunk's four 32-bit words (a count never
// exceeds the block's nq * K <= 512 * 64 entries, so none can carry into its neighbour).
__device__ __forceinline__ int get_cnt(const uint32_t* w, int cls) {
  return (int)((w[cls >> 1] >> (16 * (cls & 1))) & 0xffffu);
}
__device__ __forceinline__ uint32_t add_cnt(uint32_t* w, int cls) {
  return (atomicAdd(&w[cls >> 1], 1u << (16 * (cls & 1))) >> (16 * (cls & 1))) & 0xffffu;
}

}  // namespace

template <int G>
__global__ void __launch_bounds__(kThreads3, 1) attend_tc3_kernel(const __grid_constant__ TcAttendArgs a) {
  using C = Cfg3;
  constexpr int D = C::D, NS = C::NS, NP = C::NP, NQ = C::NQ, NO = C::NO;
  constexpr int NCLS = n_classes(G);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  constexpr int NF = C::NF;
  __shared__ uint64_t bar_kv[NS], bar_sfull[NP], bar_pfull[NP], bar_qfull[NQ], bar_ofull[NO], bar_ofree[NO];
  __shared__ uint64_t bar_fready[NF];
  __shared__ uint32_t tmem_base_s;
  __shared__ int s_wsum[kThreads3 / 32];
  __shared__ int s_n_items;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.n, K = a.top_k, QB = a.qb;
  const int nqb = (N + QB - 1) / QB;
  const int blk = blockIdx.x % nqb;
  const int gi = (blockIdx.x / nqb) % a.g;
  const int bi = blockIdx.x / (nqb * a.g);
  const int q0 = blk * QB;
  const int nq = min(QB, N - q0);
  const int head0 = gi * G;
  const int n_cand = min((q0 + nq - 1) / kChunk, N / kChunk);
  const Smem3 L = layout3(G, QB, K, a.n_cand_max);

  uint16_t* s_list = reinterpret_cast<uint16_t*>(sm + L.list);
  int* s_off = reinterpret_cast<int*>(sm + L.off);   // [n_cand + 1] bucket offsets
  int* s_toff = s_off + (a.n_cand_max + 1);          // [n_cand] item offsets
  uint32_t* s_items = reinterpret_cast<uint32_t*>(sm + L.items);
  float* s_rowm = reinterpret_cast<float*>(sm + L.rowm);
  float* s_rowz = reinterpret_cast<float*>(sm + L.rowz);
  float* s_fsc = reinterpret_cast<float*>(sm + L.fsc);  // [NF][128]
  uint32_t* s_cnt = reinterpret_cast<uint32_t*>(sm + L.cnt);  // [n_cand][4] packed 16-bit counters
  uint32_t* s_cur = reinterpret_cast<uint32_t*>(sm + L.cur);

  const __nv_bfloat16* qg = a.q + ((size_t)bi * a.h + head0) * N * D;
  const int32_t* idxg = a.idx + ((size_t)bi * a.g + gi) * N * K;
  const float* sselg = a.ssel + ((size_t)bi * a.h + head0) * N * K;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) tc::mbar_init(tc::smem_u32(&bar_kv[s]), 1);
    for (int s = 0; s < NP; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_sfull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_pfull[s]), 128);
    }
    for (int s = 0; s < NQ; ++s) tc::mbar_init(tc::smem_u32(&bar_qfull[s]), 128);
    for (int s = 0; s < NO; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_ofull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_ofree[s]), 128);
    }
    for (int s = 0; s < NF; ++s) tc::mbar_init(tc::smem_u32(&bar_fready[s]), 128);
    tc::mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), C::kTmemCols);

  // ---------------- buckets (conflict-free order) and work items ----------------
  for (int x = tid; x < 4 * (n_cand + 1); x += kThreads3) s_cnt[x] = s_cur[x] = 0u;
  // the extra P.V columns: a 64-key tile of ones, so that columns D.. of the output hold
  // sum_j P_j, the row's softmax denominator, computed by the tensor core
  for (int x = tid; x < (int)(C::kOnes / 16); x += kThreads3)
    reinterpret_cast<uint4*>(sm + L.ones)[x] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  constexpr int kLB = 8;
  const int n_sel_all = nq * K;
  const int32_t* idx_blk = idxg + (size_t)q0 * K;
  for (int e0 = tid; e0 < n_sel_all; e0 += kThreads3 * kLB) {
    int cv[kLB];
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads3;
      cv[u] = e < n_sel_all ? __ldg(idx_blk + e) : -1;
    }
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads3;
      const int c = cv[u];
      if (c < 0) continue;
      const int qo = e / K;
      if (c >= (q0 + qo) / kChunk) { set_error(a.err, kErrBadPage); continue; }
      add_cnt(s_cnt + 4 * c, qo & (NCLS - 1));
    }
  }
  __syncthreads();
  for (int c = tid; c < n_cand; c += kThreads3) {
    int tot = 0;
#pragma unroll
    for (int cls = 0; cls < NCLS; ++cls) tot += get_cnt(s_cnt + 4 * c, cls);
    s_off[c] = tot;
    s_toff[c] = (tot * G + 127) / 128;  // tiles per chunk
  }
  __syncthreads();
  const int n_entries = scan3(s_off, n_cand, s_wsum);
  const int n_sel_items = scan3(s_toff, n_cand, s_wsum);
  if (tid == 0) {
    s_off[n_cand] = n_entries;
    s_toff[n_cand] = n_sel_items;
  }
  __syncthreads();
  for (int e0 = tid; e0 < n_sel_all; e0 += kThreads3 * kLB) {
    int cv[kLB];
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads3;
      cv[u] = e < n_sel_all ? __ldg(idx_blk + e) : -1;
    }
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads3;
      const int c = cv[u];
      const int qo = e / K;
      if (c < 0 || c >= (q0 + qo) / kChunk) continue;
      const int cls = qo & (NCLS - 1);
      const int k = (int)add_cnt(s_cur + 4 * c, cls);
      // round-robin position: every class contributes min(n, k) entries before rank k,
      // and the classes below this one that still have a rank-k entry come first
      int pos = 0;
#pragma unroll
      for (int c2 = 0; c2 < NCLS; ++c2) {
        const int n2 = get_cnt(s_cnt + 4 * c, c2);
        pos += min(n2, k) + ((c2 < cls && n2 > k) ? 1 : 0);
      }
      s_list[s_off[c] + pos] = (uint16_t)(qo | ((e % K) << 9));
    }
  }
  const int oc_first = q0 / kChunk, oc_last = (q0 + nq - 1) / kChunk;
  if (tid == 0) {
    int n = 0;
    for (int oc = oc_first; oc <= oc_last; ++oc) {
      const int qa = max(q0, oc * kChunk) - q0, qb = min(q0 + nq, oc * kChunk + kChunk) - q0;
      for (int t0 = 0; t0 < (qb - qa) * G; t0 += 128) s_items[n++] = kOwnFlag3 | ((uint32_t)oc << 16) | (uint32_t)t0;
    }
    s_n_items = n;
  }
  __syncthreads();
  const int n_own_items = s_n_items;
  for (int c = tid; c < n_cand; c += kThreads3) {
    const int rows = (s_off[c + 1] - s_off[c]) * G;
    int base = n_own_items + s_toff[c];
    for (int t0 = 0; t0 < rows; t0 += 128) s_items[base++] = ((uint32_t)c << 16) | (uint32_t)t0;
  }
  const int n_items = n_own_items + n_sel_items;
  __syncthreads();

  // An item is (own | chunk c, first list row t0); its lane t holds list row
  // x = list_row(i, t) of the 128 from t0 (own chunk: its rows in order; selected chunk:
  // the bucket's entries, G rows each), valid while x < the item's rows.
  struct Lane {
    bool own, quad_ok, ok;  // own item; quadrant has rows in this item; this lane has a row
    int c, r, slot;         // chunk, block row, score slot (selected chunks)
  };
  auto lane_of = [&](int i, int t) {
    Lane g;
    const uint32_t it = s_items[i];
    g.own = (it & kOwnFlag3) != 0;
    g.c = (int)((it >> 16) & 0x7fffu);
    const int t0 = (int)(it & 0xffffu);
    int n_rows;
    if (g.own) {
      const int qa = max(q0, g.c * kChunk) - q0, qb = min(q0 + nq, g.c * kChunk + kChunk) - q0;
      n_rows = min(128, (qb - qa) * G - t0);
    } else {
      n_rows = min(128, (s_off[g.c + 1] - s_off[g.c]) * G - t0);
    }
    const int x = list_row(i, t);
    g.quad_ok = quad_used(i, t >> 5, n_rows);
    g.ok = x < n_rows;
    g.r = 0;
    g.slot = -1;
    if (g.ok) {
      const int xx = t0 + x;
      if (g.own) {
        const int qa = max(q0, g.c * kChunk) - q0;
        g.r = qa * G + xx;
      } else {
        const uint32_t e = s_list[s_off[g.c] + xx / G];
        g.r = (int)(e & 511u) * G + xx % G;
        g.slot = (int)(e >> 9);
      }
    }
    return g;
  };
  auto stage_u32 = [&](int s) -> uint32_t { return tc::smem_u32(sm + L.stage + s * C::kStage); };
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
  const float sc2 = a.scale * kLog2e3;

  // Register budgets per warpgroup (setmaxnreg): the block is launched with 128 registers
  // per thread (checked on the host), 128 x 512 = 65536; the producer/MMA warpgroup gives
  // up 64 per thread and the softmax warpgroups take 32 more each (the epilogue keeps 128):
  // 64 + 160 + 160 + 128 = 512 = 4 x 128, so every increase can be met.
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
  if (warp == 0) {
    // ======================= TMA producer: K_c, V_c =======================
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_items; ++i) {
        const int s = i % NS;
        // P.V(i - NS), the last reader of this stage, has completed (it follows S(i - NS))
        if (i >= NS && !wait(&bar_ofull[(i - NS) % NO], (uint32_t)(((i - NS) / NO) & 1))) break;
        const int c = (int)((s_items[i] >> 16) & 0x7fffu);
        const uint32_t sK = stage_u32(s), sV = sK + C::kStageK;
        const uint32_t full = tc::smem_u32(&bar_kv[s]);
        tc::mbar_arrive_expect_tx(full, C::kStage);
        tc::tma_load_3d(sK, &a.tmap_k, 0, c * kChunk, bi * a.g + gi, full);
        tc::tma_load_3d(sV, &a.tmap_v, 0, c * kChunk, bi * a.g + gi, full);
        ++issued;
        if (s_abort) break;
      }
      // on the way out (normal or aborted), every issued copy has landed before the CTA's
      // shared memory is released: wait (bounded) for the last phase of each used stage
      for (int j = max(0, issued - NS); j < issued; ++j)
        tc::mbar_wait(tc::smem_u32(&bar_kv[j % NS]), (uint32_t)((j / NS) & 1), kDrainPolls);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idS = tc::make_idesc_bf16(128, 64, false, false);
      constexpr uint32_t idO = tc::make_idesc_bf16(128, C::NV, false, true);
      const uint32_t sOnes = tc::smem_u32(sm + L.ones);
      auto issue_s = [&](int i) {
        const int s = i % NS, b = i % NP, qs = i % NQ;
        const uint32_t sK = stage_u32(s);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          // A: the tile's query rows in tensor memory, 16 elements = 8 columns per step
          const uint64_t db = tc::make_desc(sK + (k & 3) * 32u, 16, 1024);
          tc::mma_bf16_tmem_a(tmem + C::kColS + b * 64, tmem + C::kColQ + qs * (D / 2) + k * 8, db, idS, k > 0);
        }
        tc::mma_commit(tc::smem_u32(&bar_sfull[b]));
      };
      auto issue_pv = [&](int i) {
        const int s = i % NS, b = i % NP, o = i % NO;
        const uint32_t sV = stage_u32(s) + C::kStageK;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // P (bf16) sits in the first 32 columns of S's slot: 16 keys = 8 columns per step.
          // B is V (N columns 0..63) followed by the ones tile (columns 64..79), one
          // 64-column atom apart: LBO is the distance from this V stage to the ones tile.
          const uint64_t db = tc::make_desc(sV + k * 2048u, sOnes - sV, 1024);
          tc::mma_bf16_tmem_a(tmem + C::kColO + o * C::kOStride, tmem + C::kColS + b * 64 + k * 8, db, idO, k > 0);
        }
        tc::mma_commit(tc::smem_u32(&bar_ofull[o]));
      };
      // Issue order S(0) .. S(NP - 1), then P.V(j), S(j + NP), ...: S(j + NP) reuses the S/P
      // slot of item j, so it can never go before P.V(j); every wait blocks (no spinning
      // that would take issue slots from the softmax and epilogue warps on this sub-partition)
      int next_s = 0, next_pv = 0;
      auto do_s = [&](int i) -> bool {
        if (!wait(&bar_qfull[i % NQ], (uint32_t)((i / NQ) & 1))) return false;
        if (!wait(&bar_kv[i % NS], (uint32_t)((i / NS) & 1))) return false;
        tc::fence_after_sync();
        issue_s(i);
        ++next_s;
        return true;
      };
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
      if (next_s > 0) tc::mbar_wait(tc::smem_u32(&bar_sfull[(next_s - 1) % NP]), (uint32_t)(((next_s - 1) / NP) & 1), kDrainPolls);
      if (next_pv > 0) tc::mbar_wait(tc::smem_u32(&bar_ofull[(next_pv - 1) % NO]), (uint32_t)(((next_pv - 1) / NO) & 1), kDrainPolls);
    }
  }
  } else if (warp >= 4 && warp < 12) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 160;");
    // ======================= softmax + Q loaders (two warpgroups, alternating items) =======================
    const int wg = (warp - 4) >> 2;    // items i with i % 2 == wg
    const int t = (tid - 128) & 127;   // tile row == TMEM lane
    const int wq = warp & 3;           // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    // per-row fusion terms of the selected chunks: Mx = max shat, Zx = sum exp(shat - Mx);
    // the own item turns them into (M, 1/Z') with LSE_own
    for (int r = tid - 128; r < nq * G; r += 256) {
      const int qo = r / G, hh = r % G, i = q0 + qo;
      const int32_t* ir = idxg + (size_t)i * K;
      const float* sr = sselg + ((size_t)hh * N + i) * K;
      float mx = -INFINITY, zx = 0.f;
      for (int s0 = 0; s0 < K; s0 += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int s = s0 + u;
          const int c = s < K ? __ldg(ir + s) : -1;
          const float x = s < K ? __ldg(sr + s) : -INFINITY;
          v[u] = (c >= 0 && c < i / kChunk) ? x : -INFINITY;
        }
        float bm = v[0];
#pragma unroll
        for (int u = 1; u < 8; ++u) bm = fmaxf(bm, v[u]);
        if (bm == -INFINITY) continue;
        const float nm = fmaxf(mx, bm);
        float add = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) add += expf(v[u] - nm);
        zx = zx * expf(mx - nm) + add;
        mx = nm;
      }
      s_rowm[r] = mx;
      s_rowz[r] = zx;
    }
    // query rows of item j for this thread's tile row (zeros past the item's rows)
    uint4 qr[D / 8];
    auto load_q = [&](int j) {
      const Lane g = lane_of(j, t);
      if (g.ok) {
        const int r = g.r;
        const uint4* src = reinterpret_cast<const uint4*>(qg + ((size_t)(r % G) * N + q0 + r / G) * D);
#pragma unroll
        for (int x = 0; x < D / 8; ++x) qr[x] = __ldg(src + x);
      } else {
#pragma unroll
        for (int x = 0; x < D / 8; ++x) qr[x] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto store_q = [&](int j) {  // Q slot j % NQ: the row as D/2 columns of bf16 pairs
      uint32_t w[32];
#pragma unroll
      for (int x = 0; x < D / 8; ++x) {
        w[4 * x] = qr[x].x; w[4 * x + 1] = qr[x].y; w[4 * x + 2] = qr[x].z; w[4 * x + 3] = qr[x].w;
      }
      tc::tmem_st32(tmem + C::kColQ + (j % NQ) * (D / 2) + lane_off, w);
    };
    // the first item of this warpgroup: its Q slot is fresh
    if (wg < n_items) {
      load_q(wg);
      store_q(wg);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      arrive(tc::smem_u32(&bar_qfull[wg % NQ]));
    }
    if (wg + 2 < n_items) load_q(wg + 2);
    bar_sync(1, 256);
    // score of this thread's row in item i (selected chunks only), loaded one item ahead
    auto row_score = [&](int i) -> float {
      if (i >= n_items) return 0.f;
      const Lane g = lane_of(i, t);
      if (g.own || !g.ok) return 0.f;
      return __ldg(sselg + ((size_t)(g.r % G) * N + q0 + g.r / G) * K + g.slot);
    };
    float sh_next = row_score(wg);
    bool synced_own = false;
    for (int i = wg; i < n_items; i += 2) {
      const int b = i % NP;
      const Lane g = lane_of(i, t);
      const bool own = g.own;
      const int c = g.c;
      const float sh = sh_next;
      sh_next = row_score(i + 2);
      if (!own && !synced_own) {
        bar_sync(1, 256);  // every row's (M, 1/Z') is final once the own items are done
        synced_own = true;
      }
      // the warp leaves together (the tensor-memory loads below are warp-collective)
      if (!__all_sync(0xffffffffu, wait(&bar_sfull[b], (uint32_t)((i / NP) & 1)))) break;
      tc::fence_after_sync();
      // S(i) is done, so Q slot i % NQ is free again: store the rows of item i + 2
      const bool refill = i + 2 < n_items;
      if (refill) store_q(i + 2);
      const bool row_ok = g.ok;
      if (g.quad_ok) {
        const int r = g.r;
        float s[64];
        tc::tmem_ld32(tmem + C::kColS + b * 64 + lane_off, s);
        tc::tmem_ld32(tmem + C::kColS + b * 64 + 32 + lane_off, s + 32);
        tc::tmem_wait_ld();
        // P = exp(S - m) unnormalised; the row's output scale goes to the epilogue:
        //   selected chunk: f = exp(shat - M) / Z', applied as f / sum_j P_j (the sum is the
        //                   tensor core's extra column), i.e. the intra-chunk softmax times
        //                   the inter-chunk weight;
        //   own chunk:      -exp(m - M) / Z' (negative: applied as is), the exact local mass.
        float fsc = 0.f;
        if (!own && sc2 > 0.f) {
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
          for (int j = 8; j < 64; ++j) mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          const float mr = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                 fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
          const float moff = mr * sc2;
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] = ex2(fmaf(s[j], sc2, -moff));
          if (row_ok) fsc = expf(sh - s_rowm[r]) * s_rowz[r];
        } else {
          const int jmax = (own && row_ok) ? (q0 + r / G) - c * kChunk : 63;
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = j <= jmax ? s[j] * sc2 : -INFINITY;
            mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          }
          const float m = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
          float lp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) lp[u] = 0.f;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = ex2(s[j] - m);
            lp[j & 7] += s[j];
          }
          if (row_ok && own) {
            const float l = ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
            const float lse = (m + log2f(l)) / kLog2e3;
            const float mx = s_rowm[r], zx = s_rowz[r];
            const float M = fmaxf(lse, mx);
            const float Z = expf(lse - M) + (zx > 0.f ? zx * expf(mx - M) : 0.f);
            s_rowm[r] = M;
            s_rowz[r] = 1.0f / Z;
            fsc = -(expf(m / kLog2e3 - M) / Z);
          } else if (row_ok) {
            fsc = expf(sh - s_rowm[r]) * s_rowz[r];
          }
        }
        s_fsc[(i % NF) * 128 + t] = fsc;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = tc::pack_bf16x2(s[2 * j], s[2 * j + 1]);
        tc::tmem_st32(tmem + C::kColS + b * 64 + lane_off, pk);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      arrive(tc::smem_u32(&bar_pfull[b]));
      arrive(tc::smem_u32(&bar_fready[i % NF]));
      if (refill) arrive(tc::smem_u32(&bar_qfull[(i + 2) % NQ]));
      if (i + 4 < n_items) load_q(i + 4);
    }
    if (!synced_own) bar_sync(1, 256);
  } else if (warp >= 12) {
    // ======================= epilogue (keeps the launch budget of 128) =======================
    const int t = tid - 384;
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const uint32_t tO0 = tmem + C::kColO;
    // acc[r] (own item: =, selected chunk: +=) scale * O[row], 32 columns at c0
    auto add32 = [&](const float* v, const Lane& g, int c0, float scale) {
      float4 u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        u[j] = g.own ? make_float4(0.f, 0.f, 0.f, 0.f) : *acc_f4(sm, L.o, g.r, (c0 >> 2) + j);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        u[j].x = fmaf(v[4 * j], scale, u[j].x);
        u[j].y = fmaf(v[4 * j + 1], scale, u[j].y);
        u[j].z = fmaf(v[4 * j + 2], scale, u[j].z);
        u[j].w = fmaf(v[4 * j + 3], scale, u[j].w);
        *acc_f4(sm, L.o, g.r, (c0 >> 2) + j) = u[j];
      }
    };
    for (int i = 0; i < n_items; ++i) {
      const int o = i % NO;
      const bool ok = __all_sync(0xffffffffu, wait(&bar_ofull[o], (uint32_t)((i / NO) & 1)) &&
                                                  wait(&bar_fready[i % NF], (uint32_t)((i / NF) & 1)));
      tc::fence_after_sync();
      const Lane g = lane_of(i, t);
      float va[32], vb[32], vs[1];
      if (ok && g.quad_ok) {
        const uint32_t base = tO0 + o * C::kOStride + lane_off;
        tc::tmem_ld32(base, va);
        tc::tmem_ld32(base + 32, vb);
        tc::tmem_ld1(base + D, vs);
      }
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      arrive(tc::smem_u32(&bar_ofree[o]));  // item i has left tensor memory
      if (ok && g.ok) {
        const float fv = s_fsc[(i % NF) * 128 + t];
        const float scale = fv < 0.f ? -fv : fv * __frcp_rn(vs[0]);
        add32(va, g, 0, scale);
        add32(vb, g, 32, scale);
      }
      // a row sits at different tile positions in different items: every item's
      // read-modify-writes finish before the next item's start (the barrier also votes
      // on leaving the loop, so all 128 threads leave together)
      if (bar_or(2, 128, !ok || s_abort)) break;
    }
  }

  // ---------------- write the block's rows ----------------
  tc::fence_before_sync();
  __syncthreads();
  if (!s_abort) {
    for (int x = tid; x < nq * G * (D / 4); x += kThreads3) {
      const int r = x / (D / 4), j4 = x % (D / 4);
      const int qo = r / G, hh = r % G;
      const float4 v = *acc_f4(sm, L.o, r, j4);
      uint2 pk;
      pk.x = tc::pack_bf16x2(v.x, v.y);
      pk.y = tc::pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(a.out + (((size_t)bi * a.h + head0 + hh) * N + q0 + qo) * D + j4 * 4) = pk;
    }
    // log Zhat = M + log Z', with (M, 1/Z') left in s_rowm / s_rowz by the own items
    if (a.lse)
      for (int r = tid; r < nq * G; r += kThreads3)
        a.lse[((size_t)bi * a.h + head0 + r % G) * N + q0 + r / G] = s_rowm[r] - logf(s_rowz[r]);
  }
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
}

// Queries per CTA for a shape, or 0 when the shared-memory plan does not fit.
static int pick_qb3(int G, int K, int N, size_t* smem_out) {
  int qb = Cfg3::kRows / G;
  const int n_cand_max = N / kChunk;
  for (; qb >= 16; qb >>= 1) {
    const Smem3 L = layout3(G, qb, K, n_cand_max);
    const size_t need = (size_t)L.total + 1024;
    if (need <= 227 * 1024 - 1024) {
      *smem_out = need;
      return qb;
    }
  }
  return 0;
}

// The register budgets of the warp roles add up to 128 registers per launched thread:
// the kernel is only used when it was compiled to exactly that many.
template <int G>
static bool regs_ok3() {
  static int ok = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (ok < 0) {
    cudaFuncAttributes fa{};
    ok = cudaFuncGetAttributes(&fa, attend_tc3_kernel<G>) == cudaSuccess && fa.numRegs == 128;
  }
  return ok == 1;
}

static bool regs_ok3_for(int G) {
  switch (G) {
    case 1: return regs_ok3<1>();
    case 2: return regs_ok3<2>();
    case 4: return regs_ok3<4>();
    case 8: return regs_ok3<8>();
  }
  return false;
}

bool attend_tc3_supported(int d, int G, int K, int N) {
  size_t smem;
  return d == 64 && K <= 64 && N / kChunk <= 32767 && pick_qb3(G, K, N, &smem) > 0 && regs_ok3_for(G);
}

template <int G>
static cudaError_t launch_tc3(TcAttendArgs a, cudaStream_t st) {
  size_t smem = 0;
  const int qb = pick_qb3(G, a.top_k, a.n, &smem);
  if (qb == 0) return cudaErrorInvalidConfiguration;
  a.qb = qb;
  a.n_cand_max = a.n / kChunk;
  cudaError_t e = cudaFuncSetAttribute(attend_tc3_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((a.n + qb - 1) / qb) * a.g * a.b;
  if (blocks == 0) return cudaSuccess;
  attend_tc3_kernel<G><<<(unsigned)blocks, kThreads3, smem, st>>>(a);
  return cudaGetLastError();
}

// The caller has encoded a.tmap_k / a.tmap_v (64 x 64 boxes, 128-byte swizzle).
cudaError_t run_attend_tc3(const TcAttendArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_tc3<1>(a, st);
    case 2: return launch_tc3<2>(a, st);
    case 4: return launch_tc3<4>(a, st);
    case 8: return launch_tc3<8>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hils
