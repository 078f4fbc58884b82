// Selected-chunk + own-chunk attention with the inter-chunk fusion on the
// 5th-generation tensor cores (tcgen05 + TMEM), bf16 inputs, fp32 accumulation.
// (HiLS notes, section 5.3: w_ij = exp(s_ij)/Z_{i,c} * exp(shat_{i,c})/Zhat_i;
// Tide digest, Figure 3.)
//
// Work decomposition ("row owner, chunk buckets").  One CTA owns a block of QB
// consecutive queries of one (sequence, KV head) and all G query heads of the
// group: R = QB*G rows (512 for d = 64, 128 for d = 128) whose fp32 output
// accumulators stay in shared memory for the whole CTA.  The CTA buckets its
// rows' selections by chunk (counting sort in shared memory) and turns them into
// a list of work items: 128-row tiles of (own chunk | selected chunk c, rows).
// Per item
//     S = Q_tile K_c^T              (tcgen05, M=128 N=64, S in TMEM)
//     P_j = f * exp(x_j - m)        (registers -> bf16, over S's TMEM columns)
//     O_tile = P V_c                (tcgen05, A = P from TMEM, M=128 N=d, TMEM)
//     O[row] (=|+=) O_tile[row]     (shared memory)
// so every (row, chunk) pair contributes its final weighted term and no
// partial result leaves the SM.  For a selected chunk f = exp(shat - M)/(Z' l);
// for the own chunk f = exp(m - M)/Z', where the own item completes the
// fusion max M and normaliser Z' from LSE_own = m + log l.  Own items run first.
//
// Warp roles (512 threads), synchronised by mbarriers with bounded waits:
//   warp 0      producer: cp.async gather of the tile's Q rows (completed, fenced
//               for the async proxy, then signalled) and a TMA load of K_c into a
//               ring of operand stages; a stage's Q/K half is reused once S has run
//   warp 1      producer (one thread): TMA load of V_c, released after P.V
//   warp 2      MMA issuer (one thread): an event loop issuing S(i) and P.V(j)
//               as their inputs become ready; one tcgen05.commit per MMA group
//   warps 4-11  two softmax warpgroups taking alternate items: TMEM ->
//               registers -> P (scaled by the row's fusion factor) -> TMEM
//   warps 12-15 epilogue warpgroup: TMEM -> registers -> shared-memory
//               accumulators (32-column halves, the next load overlapping)
// Rows outside a tile's count are computed and ignored (padding of the
// 128-row MMA).  Summation over chunks runs in chunk-index order, so results
// do not depend on the order of rows inside a bucket.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {

constexpr int kThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kOwnFlag = 0x80000000u;

template <int D>
struct TcCfg {
  static constexpr int NS = 2;                       // operand stages
  static constexpr int NP = 2;                       // S / P slots (TMEM)
  static constexpr int NO = 2;                       // P.V output slots (TMEM), >= NS
  static constexpr int kRows = D == 64 ? 512 : 128;  // target rows (QB * G) per CTA: more rows, fuller buckets
  static constexpr uint32_t kTmemCols = 512;  // NP S/P slots of 64 + NO output slots of D
  static constexpr uint32_t kStageA = 128 * D * 2, kStageK = 64 * D * 2, kStageV = 64 * D * 2;
  static constexpr uint32_t kStage = kStageA + kStageK + kStageV;
  static constexpr uint32_t kStageStride = (kStage + 1023) / 1024 * 1024;
};

struct TcSmem {
  uint32_t stage, o, list, off, items, rowm, rowz, cur, total;
};

__host__ __device__ inline uint32_t align_to(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline int max_items(int G, int qb, int K, int n_cand) {
  const int own_tiles = (qb / 64 + 2) * ((64 * G + 127) / 128);
  return own_tiles + n_cand + (qb * K * G + 127) / 128 + 1;
}

template <int D>
__host__ __device__ inline TcSmem tc_layout(int G, int qb, int K, int n_cand) {
  using C = TcCfg<D>;
  TcSmem L;
  uint32_t off = 0;
  L.stage = off; off += C::NS * C::kStageStride;
  L.o = off; off += (uint32_t)qb * G * D * 4;
  L.list = off; off = align_to(off + (uint32_t)qb * K * 2, 16);
  L.off = off; off = align_to(off + (uint32_t)(2 * n_cand + 2) * 4, 16);
  L.items = off; off = align_to(off + (uint32_t)max_items(G, qb, K, n_cand) * 4, 16);
  L.rowm = off; off += (uint32_t)qb * G * 4;
  L.rowz = off; off += (uint32_t)qb * G * 4;
  L.cur = off; off += (uint32_t)(n_cand + 1) * 4;  // scatter cursors of the bucket sort
  L.total = align_to(off, 16);
  return L;
}

__device__ __forceinline__ float4* o_row_f4(unsigned char* base, uint32_t o_off, int r, int j4, int D) {
  // float4 j4 of row r, XOR-swizzled by (r & 7) to spread rows over banks
  return reinterpret_cast<float4*>(base + o_off + (size_t)r * D * 4 + (size_t)((j4 ^ (r & 7)) * 16));
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also returns the OR of `pred` over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
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
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}

// Exclusive scan of v[0..n) in place over the whole block; returns the total.
__device__ int block_exclusive_scan(int* v, int n, int* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (n + kThreads - 1) / kThreads;
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
  for (int w = 0; w < kThreads / 32; ++w) {
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

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const __grid_constant__ TcAttendArgs a) {
  using C = TcCfg<D>;
  constexpr int NS = C::NS, NP = C::NP, NO = C::NO;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  // stage ring: Q tile + K chunk (full_qk) and V chunk (full_v).  A stage's Q/K half is
  // free once S of its item completed (sfull), its V half once P.V completed (ofull):
  // each MMA group is committed to exactly one barrier, which every consumer waits on
  static_assert(NS == NP, "stage and S-slot rings must have the same depth");
  // the V producer waits for P.V(i - NS) on the output ring: with NO >= NS the barrier
  // cannot run a full lap ahead of that wait (P.V(i - NS + NO) needs V(i))
  static_assert(NO >= NS && C::NP * 64 + NO * D <= (int)C::kTmemCols, "output ring");
  __shared__ uint64_t bar_full_qk[NS], bar_full_v[NS];
  __shared__ uint64_t bar_sfull[NP], bar_pfull[NP], bar_ofull[NO], bar_ofree[NO];
  __shared__ uint32_t tmem_base_s;
  __shared__ int s_wsum[kThreads / 32];
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
  const TcSmem L = tc_layout<D>(G, QB, K, a.n_cand_max);

  uint16_t* s_list = reinterpret_cast<uint16_t*>(sm + L.list);
  int* s_off = reinterpret_cast<int*>(sm + L.off);          // [n_cand + 1] bucket offsets
  int* s_toff = s_off + (a.n_cand_max + 1);                 // [n_cand] item offsets
  uint32_t* s_items = reinterpret_cast<uint32_t*>(sm + L.items);
  float* s_rowm = reinterpret_cast<float*>(sm + L.rowm);
  float* s_rowz = reinterpret_cast<float*>(sm + L.rowz);

  const __nv_bfloat16* qg = a.q + ((size_t)bi * a.h + head0) * N * D;
  const int32_t* idxg = a.idx + ((size_t)bi * a.g + gi) * N * K;
  const float* sselg = a.ssel + ((size_t)bi * a.h + head0) * N * K;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_full_qk[s]), 32 + 1);  // 32 producer lanes + K's expect_tx
      tc::mbar_init(tc::smem_u32(&bar_full_v[s]), 1);
    }
    for (int s = 0; s < NP; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_sfull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_pfull[s]), 128);
    }
    for (int s = 0; s < NO; ++s) {
      tc::mbar_init(tc::smem_u32(&bar_ofull[s]), 1);
      tc::mbar_init(tc::smem_u32(&bar_ofree[s]), 128);
    }
    tc::mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), C::kTmemCols);

  // ---------------- buckets and work items ----------------
  for (int c = tid; c <= n_cand; c += kThreads) s_off[c] = 0;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  // this CTA's selections are contiguous in idx: [q0*K, (q0+nq)*K); loads are issued in
  // batches before the shared-memory atomics so their latencies overlap
  constexpr int kLB = 8;
  const int n_sel_all = nq * K;
  const int32_t* idx_blk = idxg + (size_t)q0 * K;
  for (int e0 = tid; e0 < n_sel_all; e0 += kThreads * kLB) {
    int cv[kLB];
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads;
      cv[u] = e < n_sel_all ? __ldg(idx_blk + e) : -1;
    }
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads;
      const int c = cv[u];
      if (c < 0) continue;
      if (c >= (q0 + e / K) / kChunk) { set_error(a.err, kErrBadPage); continue; }
      atomicAdd(&s_off[c], 1);
    }
  }
  __syncthreads();
  for (int c = tid; c < n_cand; c += kThreads) s_toff[c] = (s_off[c] * G + 127) / 128;  // tiles per chunk
  __syncthreads();
  const int n_entries = block_exclusive_scan(s_off, n_cand, s_wsum);
  const int n_sel_items = block_exclusive_scan(s_toff, n_cand, s_wsum);
  // cursors for the scatter: a copy of the offsets
  int* cur = reinterpret_cast<int*>(sm + L.cur);
  for (int c = tid; c < n_cand; c += kThreads) cur[c] = s_off[c];
  if (tid == 0) s_off[n_cand] = n_entries;
  __syncthreads();
  for (int e0 = tid; e0 < n_sel_all; e0 += kThreads * kLB) {
    int cv[kLB];
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads;
      cv[u] = e < n_sel_all ? __ldg(idx_blk + e) : -1;
    }
#pragma unroll
    for (int u = 0; u < kLB; ++u) {
      const int e = e0 + u * kThreads;
      const int c = cv[u];
      const int qo = e / K;
      if (c < 0 || c >= (q0 + qo) / kChunk) continue;
      const int pos = atomicAdd(&cur[c], 1);
      s_list[pos] = (uint16_t)(qo | ((e % K) << 9));
    }
  }
  // items: the own chunks' tiles first, then every selected chunk's tiles
  const int oc_first = q0 / kChunk, oc_last = (q0 + nq - 1) / kChunk;
  if (tid == 0) {
    int n = 0;
    for (int oc = oc_first; oc <= oc_last; ++oc) {
      const int qa = max(q0, oc * kChunk) - q0, qb = min(q0 + nq, oc * kChunk + kChunk) - q0;
      for (int t0 = 0; t0 < (qb - qa) * G; t0 += 128) s_items[n++] = kOwnFlag | ((uint32_t)oc << 16) | (uint32_t)t0;
    }
    s_n_items = n;
  }
  __syncthreads();
  const int n_own_items = s_n_items;
  for (int c = tid; c < n_cand; c += kThreads) {
    const int rows = (s_off[c + 1] - s_off[c]) * G;
    int base = n_own_items + s_toff[c];
    for (int t0 = 0; t0 < rows; t0 += 128) s_items[base++] = ((uint32_t)c << 16) | (uint32_t)t0;
  }
  const int n_items = n_own_items + n_sel_items;
  __syncthreads();

  // item -> tile geometry
  auto item_rows = [&](uint32_t it, int& c, bool& own, int& t0, int& n_rows) {
    own = (it & kOwnFlag) != 0;
    c = (int)((it >> 16) & 0x7fffu);
    t0 = (int)(it & 0xffffu);
    if (own) {
      const int qa = max(q0, c * kChunk) - q0, qb = min(q0 + nq, c * kChunk + kChunk) - q0;
      n_rows = min(128, (qb - qa) * G - t0);
    } else {
      n_rows = min(128, (s_off[c + 1] - s_off[c]) * G - t0);
    }
  };
  // tile row t of an item -> row r of the block (and the score slot for selected chunks)
  auto row_of = [&](bool own, int c, int t0, int t, int& r, int& slot) {
    const int x = t0 + t;
    if (own) {
      const int qa = max(q0, c * kChunk) - q0;
      r = (qa + x / G) * G + x % G;
      slot = -1;
    } else {
      const uint32_t e = s_list[s_off[c] + x / G];
      r = (int)(e & 511u) * G + x % G;
      slot = (int)(e >> 9);
    }
  };
  auto stage_ptr = [&](int s) -> unsigned char* { return sm + L.stage + s * C::kStageStride; };
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
  const float sc2 = a.scale * kLog2e;

  if (warp == 0) {
    // ======================= producer: Q rows (cp.async gather) + K chunk (TMA) =======================
    // The Q rows are written through the generic proxy: each lane waits for its own
    // copies, fences them for the tensor core (async proxy), then arrives.  With two
    // stages one item's copies stay in flight while the next item is issued.  Every
    // decision to stop is taken by the whole warp (the counts below stay warp-uniform).
    int issued = 0, published = 0;
    auto publish = [&](int j) {  // item j's copies are complete and fenced
      tc::fence_async_smem();
      mbar_arrive(tc::smem_u32(&bar_full_qk[j % NS]));
      ++published;
    };
    for (int i = 0; i < n_items; ++i) {
      const int s = i % NS;
      if (i >= NS && !__all_sync(0xffffffffu, wait(&bar_sfull[(i - NS) % NP], (uint32_t)(((i - NS) / NP) & 1))))
        break;
      int c, t0, n_rows;
      bool own;
      item_rows(s_items[i], c, own, t0, n_rows);
      const uint32_t sA = tc::smem_u32(stage_ptr(s)), sK = sA + C::kStageA;
      const uint32_t full = tc::smem_u32(&bar_full_qk[s]);
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(full, C::kStageK);
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tc::tma_load_3d(sK + x * 8192u, &a.tmap_k, x * 64, c * kChunk, bi * a.g + gi, full);
      }
      constexpr int CH = D / 8;  // 16-byte pieces per row
      for (int t = lane; t < n_rows; t += 32) {
        int r, slot;
        row_of(own, c, t0, t, r, slot);
        const __nv_bfloat16* src = qg + ((size_t)(r % G) * N + q0 + r / G) * D;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
          tc::cp_async16(sA + (uint32_t)(ch >> 3) * 16384u + tc::sw128_chunk(t, ch & 7), src + ch * 8);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      ++issued;
      if constexpr (NS == 1) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        publish(i);
      } else {
        if (i >= 1) {
          asm volatile("cp.async.wait_group 1;" ::: "memory");
          publish(i - 1);
        }
        if (i == n_items - 1) {
          asm volatile("cp.async.wait_group 0;" ::: "memory");
          publish(i);
        }
      }
      if (__any_sync(0xffffffffu, s_abort != 0)) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // On the way out (normal or aborted) no copy may still be writing shared memory when the
    // CTA ends: items issued but not yet published are published now, so that their barrier
    // phases complete once the K tiles land, and lane 0 waits (drain bound) for the newest
    // phase of every stage used.
    while (published < issued) publish(published);
    if (lane == 0)
      for (int j = max(0, issued - NS); j < issued; ++j)
        tc::mbar_wait(tc::smem_u32(&bar_full_qk[j % NS]), (uint32_t)((j / NS) & 1), kDrainPolls);
  } else if (warp == 1) {
    // ======================= producer: V chunk (TMA) =======================
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_items; ++i) {
        const int s = i % NS;
        // P.V of item i - NS, the last reader of this stage's V, must have completed
        if (i >= NS && !wait(&bar_ofull[(i - NS) % NO], (uint32_t)(((i - NS) / NO) & 1))) break;
        const int c = (int)((s_items[i] >> 16) & 0x7fffu);
        const uint32_t sV = tc::smem_u32(stage_ptr(s)) + C::kStageA + C::kStageK;
        const uint32_t full = tc::smem_u32(&bar_full_v[s]);
        tc::mbar_arrive_expect_tx(full, C::kStageV);
#pragma unroll
        for (int x = 0; x < D / 64; ++x) tc::tma_load_3d(sV + x * 8192u, &a.tmap_v, x * 64, c * kChunk, bi * a.g + gi, full);
        ++issued;
        if (s_abort) break;
      }
      // every issued copy has landed before the CTA's shared memory is released
      for (int j = max(0, issued - NS); j < issued; ++j)
        tc::mbar_wait(tc::smem_u32(&bar_full_v[j % NS]), (uint32_t)((j / NS) & 1), kDrainPolls);
    }
  } else if (warp == 2) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t tS0 = tmem, tO0 = tmem + NP * 64;
      constexpr uint32_t idS = tc::make_idesc_bf16(128, 64, false, false);
      constexpr uint32_t idO = tc::make_idesc_bf16(128, D, false, true);
      auto issue_s = [&](int i) {
        const int s = i % NS, b = i % NP;
        const uint32_t sA = tc::smem_u32(stage_ptr(s)), sK = sA + C::kStageA;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t da = tc::make_desc(sA + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
          const uint64_t db = tc::make_desc(sK + (k >> 2) * 8192u + (k & 3) * 32u, 16, 1024);
          tc::mma_bf16(tS0 + b * 64, da, db, idS, k > 0);
        }
        tc::mma_commit(tc::smem_u32(&bar_sfull[b]));
      };
      auto issue_pv = [&](int i) {
        const int s = i % NS, b = i % NP, o = i % NO;
        const uint32_t sV = tc::smem_u32(stage_ptr(s)) + C::kStageA + C::kStageK;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // P (bf16) sits in the first 32 columns of S's slot: 16 keys = 8 columns per step
          const uint64_t db = tc::make_desc(sV + k * 2048u, 8192, 1024);
          tc::mma_bf16_tmem_a(tO0 + o * D, tS0 + b * 64 + k * 8, db, idO, k > 0);
        }
        // one commit per MMA group: a second commit would track no MMA and arrive at once
        tc::mma_commit(tc::smem_u32(&bar_ofull[o]));
      };
      // event loop: issue S(next_s) as soon as its operands have landed and its S slot
      // is free, and P.V(next_pv) as soon as its P is written and its TMEM slot is free
      int next_s = 0, next_pv = 0;
      uint32_t idle = 0;
      while (next_pv < n_items) {
        bool progressed = false;
        if (next_s < n_items && next_s < next_pv + NP &&
            tc::mbar_probe(tc::smem_u32(&bar_full_qk[next_s % NS]), (uint32_t)((next_s / NS) & 1))) {
          tc::fence_after_sync();
          issue_s(next_s);
          ++next_s;
          progressed = true;
        }
        if (next_pv < next_s &&
            tc::mbar_probe(tc::smem_u32(&bar_pfull[next_pv % NP]), (uint32_t)((next_pv / NP) & 1)) &&
            tc::mbar_probe(tc::smem_u32(&bar_full_v[next_pv % NS]), (uint32_t)((next_pv / NS) & 1)) &&
            (next_pv < NO ||
             tc::mbar_probe(tc::smem_u32(&bar_ofree[next_pv % NO]), (uint32_t)(((next_pv - NO) / NO) & 1)))) {
          tc::fence_after_sync();
          issue_pv(next_pv);
          ++next_pv;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (++idle >= a.poll || ((idle & 1023u) == 1023u && s_abort)) {
          if (!s_abort) {
            set_error(a.err, kErrTimeout);
            s_abort = 1;
          }
          break;
        }
      }
      // every MMA issued has completed before the tensor memory is released: MMAs complete
      // in issue order, and only this thread commits, so the last commit of each ring is
      // the newest phase of its barrier
      if (next_s > 0)
        tc::mbar_wait(tc::smem_u32(&bar_sfull[(next_s - 1) % NP]), (uint32_t)(((next_s - 1) / NP) & 1), kDrainPolls);
      if (next_pv > 0)
        tc::mbar_wait(tc::smem_u32(&bar_ofull[(next_pv - 1) % NO]), (uint32_t)(((next_pv - 1) / NO) & 1), kDrainPolls);
    }
  } else if (warp >= 4 && warp < 12) {
    // ======================= softmax (two warpgroups, alternating items) =======================
    // With one S slot a second warpgroup would wait on a barrier phase two ahead of the
    // last one it saw, which a parity wait cannot tell apart: one warpgroup then.
    constexpr int kWG = NP >= 2 ? 2 : 1;
    const int wg = (warp - 4) >> 2;      // warpgroup: handles items i with i % kWG == wg
    const int t = (tid - 128) & 127;     // tile row == TMEM lane
    const int wq = warp & 3;             // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    // per-row fusion terms of the selected chunks: Mx = max shat, Zx = sum exp(shat - Mx);
    // the own item turns them into (M, 1/Z') with LSE_own
    for (int r = tid - 128; r < nq * G; r += 256) {
      const int qo = r / G, hh = r % G, i = q0 + qo;
      const int32_t* ir = idxg + (size_t)i * K;
      const float* sr = sselg + ((size_t)hh * N + i) * K;
      float mx = -INFINITY, zx = 0.f;  // online max / shifted sum over the valid slots
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
    named_bar(1, 256);
    // score of this thread's row in item i (selected chunks only), loaded one item ahead
    auto row_score = [&](int i) -> float {
      if (i >= n_items) return 0.f;
      int c, t0, n_rows;
      bool own;
      item_rows(s_items[i], c, own, t0, n_rows);
      if (own || t >= n_rows) return 0.f;
      int r, slot;
      row_of(own, c, t0, t, r, slot);
      return __ldg(sselg + ((size_t)(r % G) * N + q0 + r / G) * K + slot);
    };
    float sh_next = row_score(wg);
    bool synced_own = false;
    for (int i = wg; i < n_items && wg < kWG; i += kWG) {
      const int b = i % NP;
      int c, t0, n_rows;
      bool own;
      item_rows(s_items[i], c, own, t0, n_rows);
      const float sh = sh_next;
      sh_next = row_score(i + kWG);
      if (!own && !synced_own) {
        named_bar(1, 256);  // every row's (M, 1/Z') is final once the own items are done
        synced_own = true;
      }
      // the warp leaves together (the tensor-memory loads below are warp-collective)
      if (!__all_sync(0xffffffffu, wait(&bar_sfull[b], (uint32_t)((i / NP) & 1)))) break;
      tc::fence_after_sync();
      const bool row_ok = t < n_rows;
      if (wq * 32 < n_rows) {
        int r = 0, slot = -1;
        if (row_ok) row_of(own, c, t0, t, r, slot);
        float s[64];
        tc::tmem_ld32(tmem + b * 64 + lane_off, s);
        tc::tmem_ld32(tmem + b * 64 + 32 + lane_off, s + 32);
        tc::tmem_wait_ld();
        float mult;  // the row's fusion factor, folded into P so that P.V is the final term
        if (!own && sc2 > 0.f) {
          // lean path (all 64 keys valid): raw max, p = exp2(S*c - m*c), one FFMA + ex2 each
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
          for (int j = 8; j < 64; ++j) mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          const float mr = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                 fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
          const float moff = mr * sc2;  // scale > 0: the max of the scaled logits
          float lp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) lp[u] = 0.f;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = exp2f(fmaf(s[j], sc2, -moff));
            lp[j & 7] += s[j];
          }
          const float l = ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
          mult = row_ok ? expf(sh - s_rowm[r]) * s_rowz[r] / l : 0.f;
        } else {
          // general path (own chunk: causal mask; LSE_own completes the fusion max and normaliser)
          const int jmax = (own && row_ok) ? (q0 + r / G) - c * kChunk : 63;
          float mp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = j <= jmax ? s[j] * sc2 : -INFINITY;  // log2 domain
            mp[j & 7] = fmaxf(mp[j & 7], s[j]);
          }
          const float m = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
          float lp[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) lp[u] = 0.f;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            s[j] = exp2f(s[j] - m);
            lp[j & 7] += s[j];
          }
          const float l = ((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7]));
          mult = 0.f;
          if (row_ok && own) {
            const float lse = (m + log2f(l)) / kLog2e;  // natural-log LSE_own
            const float mx = s_rowm[r], zx = s_rowz[r];
            const float M = fmaxf(lse, mx);
            const float Z = expf(lse - M) + (zx > 0.f ? zx * expf(mx - M) : 0.f);
            s_rowm[r] = M;
            s_rowz[r] = 1.0f / Z;
            mult = expf(m / kLog2e - M) / Z;
          } else if (row_ok) {
            mult = expf(sh - s_rowm[r]) * s_rowz[r] / l;
          }
        }
        // P = mult * p overwrites the first 32 columns of S's slot (this lane's row, already
        // in registers).  P.V(i - NP), the last reader of the slot, was issued before S(i)
        // and tcgen05 MMAs run in issue order, so the slot is free.
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = tc::pack_bf16x2(s[2 * j] * mult, s[2 * j + 1] * mult);
        tc::tmem_st32(tmem + b * 64 + lane_off, pk);
        tc::tmem_wait_st();
      }
      tc::fence_before_sync();
      mbar_arrive(tc::smem_u32(&bar_pfull[b]));
    }
    if (!synced_own) named_bar(1, 256);
  } else if (warp >= 12) {
    // ======================= epilogue =======================
    const int t = tid - 384;
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const uint32_t tO0 = tmem + NP * 64;
    struct Geo {
      bool own, warp_ok, row_ok;
      int r;
    };
    auto geo = [&](int i) {
      int c, t0, n_rows, slot;
      Geo g;
      item_rows(s_items[i], c, g.own, t0, n_rows);
      g.warp_ok = wq * 32 < n_rows;
      g.row_ok = t < n_rows;
      g.r = 0;
      if (g.row_ok) row_of(g.own, c, t0, t, g.r, slot);
      return g;
    };
    // acc[r] (own item: =, selected chunk: +=) the tile row's columns [c0, c0 + 32) in v;
    // P already carries the fusion factor, so the tile row is the final term
    auto add32 = [&](const float* v, const Geo& g, int c0) {
      float4 u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        u[j] = g.own ? make_float4(0.f, 0.f, 0.f, 0.f) : *o_row_f4(sm, L.o, g.r, (c0 >> 2) + j, D);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        u[j].x += v[4 * j];
        u[j].y += v[4 * j + 1];
        u[j].z += v[4 * j + 2];
        u[j].w += v[4 * j + 3];
        *o_row_f4(sm, L.o, g.r, (c0 >> 2) + j, D) = u[j];
      }
    };
    // A row sits at different tile positions in different items, so every item's
    // read-modify-writes finish (named barrier 2) before the next item's start.  The
    // barrier also votes on leaving the loop, so all 128 threads leave together.
    if constexpr (D == 64) {
      // 32-column halves in a software pipeline: the TMEM load of the next half runs
      // while the previous half is added into shared memory
      float va[32], vb[32];
      bool ok = true;
      Geo cur{};
      if (n_items > 0) {
        ok = __all_sync(0xffffffffu, wait(&bar_ofull[0], 0u));
        tc::fence_after_sync();
        cur = geo(0);
        if (ok && cur.warp_ok) tc::tmem_ld32(tO0 + lane_off, va);
        tc::tmem_wait_ld();
      }
      for (int i = 0; i < n_items; ++i) {
        const int o = i % NO;
        if (ok && cur.warp_ok) tc::tmem_ld32(tO0 + o * 64 + 32 + lane_off, vb);
        if (ok && cur.row_ok) add32(va, cur, 0);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        mbar_arrive(tc::smem_u32(&bar_ofree[o]));  // item i has left TMEM
        Geo nxt{};
        if (i + 1 < n_items) {
          ok = __all_sync(0xffffffffu, ok && wait(&bar_ofull[(i + 1) % NO], (uint32_t)(((i + 1) / NO) & 1)));
          tc::fence_after_sync();
          nxt = geo(i + 1);
          if (ok && nxt.warp_ok) tc::tmem_ld32(tO0 + ((i + 1) % NO) * 64 + lane_off, va);
        }
        if (ok && cur.row_ok) add32(vb, cur, 32);
        tc::tmem_wait_ld();
        if (named_bar_or(2, 128, !ok || s_abort)) break;
        cur = nxt;
      }
    } else {
      for (int i = 0; i < n_items; ++i) {
        const int o = i % NO;
        const bool ok = __all_sync(0xffffffffu, wait(&bar_ofull[o], (uint32_t)((i / NO) & 1)));
        tc::fence_after_sync();
        const Geo g = geo(i);
        if (ok && g.warp_ok) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float v[32];
            tc::tmem_ld32(tO0 + o * D + c0 + lane_off, v);
            tc::tmem_wait_ld();
            if (g.row_ok) add32(v, g, c0);
          }
        }
        tc::fence_before_sync();
        mbar_arrive(tc::smem_u32(&bar_ofree[o]));
        if (named_bar_or(2, 128, !ok || s_abort)) break;
      }
    }
  }

  // ---------------- write the block's rows ----------------
  tc::fence_before_sync();
  __syncthreads();
  if (!s_abort) {
    for (int x = tid; x < nq * G * (D / 4); x += kThreads) {
      const int r = x / (D / 4), j4 = x % (D / 4);
      const int qo = r / G, hh = r % G;
      const float4 v = *o_row_f4(sm, L.o, r, j4, D);
      uint2 pk;
      pk.x = tc::pack_bf16x2(v.x, v.y);
      pk.y = tc::pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(a.out + (((size_t)bi * a.h + head0 + hh) * N + q0 + qo) * D + j4 * 4) = pk;
    }
    // log Zhat = M + log Z', with (M, 1/Z') left in s_rowm / s_rowz by the own items
    if (a.lse)
      for (int r = tid; r < nq * G; r += kThreads)
        a.lse[((size_t)bi * a.h + head0 + r % G) * N + q0 + r / G] = s_rowm[r] - logf(s_rowz[r]);
  }
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, C::kTmemCols);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [b*g][N][D] bf16 tensor as a rank-3 map with 64 x 64 boxes in the 128-byte
// swizzle of the MMA operand tiles; rows past N read as zeros.
static bool encode_kv_map(CUtensorMap* m, const void* base, int D, int N, int bg) {
  return encode_kv_tensor_map(m, base, D, N, bg);
}
bool encode_kv_tensor_map(CUtensorMap* m, const void* base, int D, int N, int bg) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)bg};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Queries per CTA for a shape, or 0 when the shared-memory plan does not fit.
template <int D>
static int pick_qb(int G, int K, int N, size_t* smem_out) {
  int qb = TcCfg<D>::kRows / G;
  const int n_cand_max = N / kChunk;
  for (; qb >= 16; qb >>= 1) {
    const TcSmem L = tc_layout<D>(G, qb, K, n_cand_max);
    const size_t need = (size_t)L.total + 1024;
    if (need <= 227 * 1024 - 1024) {  // leave room for the static shared variables
      *smem_out = need;
      return qb;
    }
  }
  return 0;
}

bool attend_tc_supported(int d, int G, int K, int N) {
  size_t smem;
  if (K > 64 || N / kChunk > 32767 || tensor_map_encoder() == nullptr) return false;
  if (d == 64 && attend_tc3_supported(d, G, K, N)) return true;
  return d == 64 ? pick_qb<64>(G, K, N, &smem) > 0 : d == 128 ? pick_qb<128>(G, K, N, &smem) > 0 : false;
}

template <int D, int G>
static cudaError_t launch_tc(TcAttendArgs a, cudaStream_t st) {
  size_t smem = 0;
  const int qb = pick_qb<D>(G, a.top_k, a.n, &smem);
  if (qb == 0) return cudaErrorInvalidConfiguration;
  a.qb = qb;
  a.n_cand_max = a.n / kChunk;
  if (!encode_kv_map(&a.tmap_k, a.k, D, a.n, a.b * a.g) || !encode_kv_map(&a.tmap_v, a.v, D, a.n, a.b * a.g))
    return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((a.n + qb - 1) / qb) * a.g * a.b;
  if (blocks == 0) return cudaSuccess;
  attend_tc_kernel<D, G><<<(unsigned)blocks, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t tc_by_group(const TcAttendArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_tc<D, 1>(a, st);
    case 2: return launch_tc<D, 2>(a, st);
    case 4: return launch_tc<D, 4>(a, st);
    case 8: return launch_tc<D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_attend_tc(const TcAttendArgs& a, int d, cudaStream_t st) {
  if (d == 64 && attend_tc3_supported(d, a.h / a.g, a.top_k, a.n)) {
    TcAttendArgs b = a;
    if (!encode_kv_map(&b.tmap_k, b.k, 64, b.n, b.b * b.g) || !encode_kv_map(&b.tmap_v, b.v, 64, b.n, b.b * b.g))
      return cudaErrorNotSupported;
    return run_attend_tc3(b, st);
  }
  return d == 64 ? tc_by_group<64>(a, st) : tc_by_group<128>(a, st);
}

}  // namespace hils
