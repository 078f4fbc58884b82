// Single-token decode over a paged chunk cache (HiLS notes, sections 5.2-5.4,
// applied to the newest query of each sequence).  Two HBM-bound kernels,
// chained with programmatic dependent launch:
//
// 1. decode_scan_kernel -- grid (sequence, range of candidate chunks).  Each CTA
//    reads the cached summaries of its range page by page, all heads at once (a
//    page's [h][d] fp32 block is contiguous), scores them (q . kbar * scale + H, GQA
//    max over the group's heads) and, one warp per KV head, writes the range's best
//    K keys as a sorted list.
// 2. decode_attend_kernel -- one warp per half chunk (32 keys) of the local
//    branch or of one Top-K slot, all G heads sharing each K/V load.  The local
//    branch does not depend on the selection and is computed before the kernel
//    waits for the scan grid.  Then warp 0 of every CTA merges its KV head's range
//    lists into the Top-K (a warp tournament over the sorted lists, staged in
//    shared memory), and each slot's warps look up the chunk's page and attend to
//    it.  Each warp writes its half's (max, sum, unnormalised output); the last CTA
//    of the (sequence, KV head) -- an atomic ticket; no CTA waits on another --
//    fuses them with the inter-chunk softmax of notes section 5.3 (local branch at
//    its exact log-mass).
// The ticket is reset by the CTA that consumes it, so both kernels can be replayed
// (CUDA graphs) without clearing the workspace.
#pragma once
#include "common.cuh"
#include "kernels.cuh"

namespace hils {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kMaxRange = 256;          // candidate chunks per scan CTA, at most ...
constexpr int kMinRange = 16;           // ... and at least
constexpr int kScanCtasTarget = 4 * 148;  // about four scan CTAs per SM of a B200


constexpr int kMaxListsPerLane = 4;
constexpr int kStageKeys = 512;         // keys of range lists staged in shared memory per merging warp
constexpr int kMaxDecodeLocal = 16;     // local-branch chunks a decode step supports


__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((unsigned long long)hi << 32) | lo;
}

// Descending bitonic sort of the warp's 32*E keys; element i lives in lane i / E,
// register i % E.  All 32 lanes call it.
template <int E>
__device__ __forceinline__ void warp_sort_desc(unsigned long long (&v)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= E) {  // partner in lane ^ (j / E), same register
        const int lj = j / E;
        const bool lower = (lane & lj) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const bool desc = ((lane * E + e) & k) == 0;
          const unsigned long long o = shfl_xor_u64(v[e], lj);
          const bool keep_max = lower == desc;
          v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
        }
      } else {  // partner in this lane, register e ^ j
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if ((e ^ j) > e) {
            const bool desc = ((lane * E + e) & k) == 0;
            const unsigned long long x = v[e], y = v[e ^ j];
            const bool sw = desc ? x < y : x > y;
            v[e] = sw ? y : x;
            v[e ^ j] = sw ? x : y;
          }
        }
      }
    }
  }
}
// The largest of the warp's 64-bit keys: two 32-bit warp reductions (redux.sync), the
// high words first, then the low words among the lanes that hold the largest high word.
__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long v) {
  const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32));
  const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32) == hi ? (uint32_t)v : 0u);
  return ((unsigned long long)hi << 32) | lo;
}

// Top-K of one KV head over this CTA's range: the key of chunk j is the max over the
// group's heads of s_score[j][head] (a NaN, from a bad page, makes the key 0).  Writes
// the K best keys (0 where the range has fewer) in descending order.
// E <= 2: a bitonic sort of the warp's 32 E keys.  E >= 4: each lane sorts its own E keys,
// then each of the K steps takes the warp's largest head (keys are unique: they carry the
// chunk index) and the lane that held it moves to its next key -- K steps of two warp
// reductions instead of the sort's 15 exchange stages of 2 E shuffles each, which, with
// every scan warp of the SM sorting at once, queue on the SM's shuffle unit.
template <int E, int G>
__device__ __forceinline__ void range_topk(const float* s_score, int H, int gi, int nc, int c_lo, int K,
                                           unsigned long long* out) {
  const int lane = threadIdx.x & 31;
  unsigned long long v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int j = e * 32 + lane;  // any placement works: the keys are sorted next
    unsigned long long key = 0;
    if (j < nc) {
      float best = -INFINITY;
      bool bad = false;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float x = s_score[(size_t)j * H + gi * G + hh];
        bad |= x != x;
        best = fmaxf(best, x);
      }
      key = bad ? 0ull : pack_key(best, c_lo + j);
    }
    v[e] = key;
  }
  if constexpr (E <= 2) {
    warp_sort_desc<E>(v);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int i = lane * E + e;
      if (i < K) out[i] = v[e];
    }
    for (int i = 32 * E + lane; i < K; i += 32) out[i] = 0ull;
  } else {
    // odd-even transposition sort of the lane's keys, descending
#pragma unroll
    for (int r = 0; r < E; ++r)
#pragma unroll
      for (int e = r & 1; e + 1 < E; e += 2) {
        const unsigned long long x = v[e], y = v[e + 1];
        v[e] = x > y ? x : y;
        v[e + 1] = x > y ? y : x;
      }
    int s = 0;
    for (; s < K; ++s) {
      const unsigned long long wb = warp_max_key(v[0]);
      if (wb == 0ull) break;  // every key taken (warp-uniform)
      if (lane == 0) out[s] = wb;
      if (v[0] == wb) {
#pragma unroll
        for (int e = 0; e + 1 < E; ++e) v[e] = v[e + 1];
        v[E - 1] = 0ull;
      }
    }
    for (int i = s + lane; i < K; i += 32) out[i] = 0ull;
  }
}

constexpr int kTour = 32 * kMaxListsPerLane;  // lists one tournament takes
constexpr int kGroupKeys = 512;               // group results a grouped merge keeps (n_groups K)

// Copies the first KW keys of each of n_lists lists of K keys (list l at parts + l K) into
// the warp's window: list l, key p at win[l KW + p].  All loads are in flight at once.
// Called by all 32 lanes.
__device__ __forceinline__ void stage_lists(unsigned long long* win, const unsigned long long* parts, int n_lists,
                                            int KW, int K) {
  const int lane = threadIdx.x & 31;
  const int n_win = n_lists * KW;
  __syncwarp();  // the window's previous contents have been read
  for (int x0 = 0; x0 < n_win; x0 += 32 * 16) {
    unsigned long long tmp[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int x = x0 + 32 * u + lane;
      tmp[u] = x < n_win ? __ldcg(parts + (size_t)(x / KW) * K + x % KW) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int x = x0 + 32 * u + lane;
      if (x < n_win) win[x] = tmp[u];
    }
  }
  __syncwarp();
}

// Tournament over n_lists <= kTour sorted lists of K keys (list l at parts + l K), whose
// first KW keys are staged at w + l KW: each step is a warp max over the lists' heads (keys
// are unique: they carry the chunk index), so a step waits on shared memory only; a list
// that wins more than KW - 1 times reads on from global memory.  Lane l follows lists l,
// l + 32, ..., holding each list's head and the key after it.  Returns the best K in
// descending order: slot lane in r0, slot lane + 32 in r1 (0: empty).  LPL: lists per lane
// (n_lists <= 32 LPL).
template <int LPL>
__device__ __forceinline__ void list_tournament_n(const unsigned long long* parts, const unsigned long long* w,
                                                  int n_lists, int KW, int K, unsigned long long& r0,
                                                  unsigned long long& r1) {
  const int lane = threadIdx.x & 31;
  auto key_at = [&](int l, int p) -> unsigned long long {
    return p < KW ? w[l * KW + p] : p < K ? __ldcg(parts + (size_t)l * K + p) : 0ull;
  };
  int pos[LPL];
  unsigned long long head[LPL], next[LPL];
#pragma unroll
  for (int m = 0; m < LPL; ++m) {
    const int l = lane + 32 * m;
    const bool live = l < n_lists;
    pos[m] = 0;
    head[m] = live ? key_at(l, 0) : 0ull;
    next[m] = live ? key_at(l, 1) : 0ull;
  }
  r0 = 0ull;
  r1 = 0ull;
  for (int s = 0; s < K; ++s) {
    unsigned long long lb = head[0];
#pragma unroll
    for (int m = 1; m < LPL; ++m) lb = head[m] > lb ? head[m] : lb;
    const unsigned long long wb = warp_max_key(lb);
    if (wb == 0ull) break;  // every list is exhausted (warp-uniform)
#pragma unroll
    for (int m = 0; m < LPL; ++m) {
      if (head[m] == wb) {  // this lane's list m holds the winner: advance it
        ++pos[m];
        head[m] = next[m];
        next[m] = key_at(lane + 32 * m, pos[m] + 1);
      }
    }
    if ((s & 31) == lane) {
      if (s < 32) r0 = wb;
      else r1 = wb;
    }
  }
}

__device__ __forceinline__ void list_tournament(const unsigned long long* parts, const unsigned long long* w,
                                                int n_lists, int KW, int K, unsigned long long& r0,
                                                unsigned long long& r1) {
  if (n_lists <= 32) list_tournament_n<1>(parts, w, n_lists, KW, K, r0, r1);
  else if (n_lists <= 64) list_tournament_n<2>(parts, w, n_lists, KW, K, r0, r1);
  else list_tournament_n<kMaxListsPerLane>(parts, w, n_lists, KW, K, r0, r1);
}

// Whether the merge of nsplit range lists of K keys fits: one tournament, or groups of
// kTour lists whose results (n_groups K keys) stay in shared memory and are merged by one
// more tournament (n_groups <= kTour).
__host__ __device__ inline bool decode_merge_fits(int nsplit, int K) {
  const int n_groups = (nsplit + kTour - 1) / kTour;
  return nsplit <= kTour || (n_groups <= kTour && n_groups * K <= kGroupKeys);
}

// The Top-K of one KV head from its nsplit range lists (list l at parts + l K), by one warp:
// one tournament, or with more than kTour lists a tournament per group of kTour lists
// (results kept in grp_keys) and a final one over the groups' results.  win: the warp's
// window of kStageKeys keys.  Returns slot lane in r0, slot lane + 32 in r1 (0: empty).
__device__ __forceinline__ void merge_lists(const unsigned long long* parts, int nsplit, int K,
                                            unsigned long long* win, unsigned long long* grp_keys,
                                            unsigned long long& r0, unsigned long long& r1) {
  const int lane = threadIdx.x & 31;
  if (nsplit <= kTour) {
    const int KW = max(1, min(K, kStageKeys / max(1, nsplit)));
    stage_lists(win, parts, nsplit, KW, K);
    list_tournament(parts, win, nsplit, KW, K, r0, r1);
    return;
  }
  const int n_groups = (nsplit + kTour - 1) / kTour;
  for (int grp = 0; grp < n_groups; ++grp) {
    const int nl = min(kTour, nsplit - grp * kTour);
    const int KW = max(1, min(K, kStageKeys / nl));
    const unsigned long long* gp = parts + (size_t)grp * kTour * K;
    stage_lists(win, gp, nl, KW, K);
    list_tournament(gp, win, nl, KW, K, r0, r1);
    if (lane < K) grp_keys[grp * K + lane] = r0;
    if (lane + 32 < K) grp_keys[grp * K + lane + 32] = r1;
  }
  __syncwarp();
  list_tournament(parts, grp_keys, n_groups, K, K, r0, r1);  // every key in shared memory
}

// Scan: CTA per (sequence, range of chunks), all heads.  A page's summaries of all
// heads, [h][d] fp32, are one contiguous block; thread t holds float4 t + 256 k of it
// (FPT per thread), so each page is read with fully coalesced 16-byte loads, PB pages
// in flight per thread.  Per (chunk, head) the dot with q is reduced over the d/4
// lanes of the head row, scaled and biased by H into shared memory; then one warp per
// KV head takes the range's best K and writes them as a sorted list, which the attention
// kernel merges with the other ranges' lists.
// Four CTAs per SM (64 registers a thread): a page gather's bandwidth grows with the
// warps resident on the SM far more than with the loads each warp has in flight.
// S: element type of the cached summaries (fp32, or bf16 for the compact cache).
// MULTI: a page's block is narrower than the CTA, so one load step covers several pages.
template <typename T, int D, int G, typename S, int FPT, bool MULTI>
__global__ void __launch_bounds__(kScanThreads, 4) decode_scan_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) float s_score[];  // [range][h]; reused by the merge
  __shared__ int s_page[kMaxRange];
  constexpr int EPP = 16 / (int)sizeof(S);       // summary elements per 16-byte piece
  constexpr int QPR = D / EPP;                   // pieces per head row
  // load steps per batch: 8 pages' worth of fp32 pieces per thread (bf16 pieces hold twice
  // the elements, so half the steps keep the registers the same)
  constexpr int PB = FPT >= 8 ? 1 : (8 / FPT) * 4 / EPP > 0 ? (8 / FPT) * 4 / EPP : 1;

  pdl_launch_dependents();  // the attend grid may start its selection-independent prologue
  const int t = threadIdx.x, warp = t >> 5;
  const int split = blockIdx.x % a.nsplit;
  const int bi = blockIdx.x / a.nsplit;
  const int H = a.h, K = a.top_k, R = a.range;
  const int c_lo = split * R;
  const int32_t* bt = a.block_table + (size_t)bi * a.max_chunks;
  const int L = a.seq_lens[bi];
  const int own = L > 0 ? (L - 1) / kChunk : 0;
  const int n_cand = min(max(0, own + 1 - a.n_local), a.max_chunks);  // chunks before the local branch
  const int nc = max(0, min(n_cand, c_lo + R) - c_lo);
  for (int x = t; x < nc; x += kScanThreads) s_page[x] = bt[c_lo + x];
  // A page's summaries [h][d] are F 16-byte pieces.  When a page block is smaller than
  // the CTA, one load step covers PPI pages (thread t: page t / F, piece t % F);
  // otherwise thread t takes pieces t + 256 k of one page.
  const int F = H * QPR;
  const int PPI = MULTI ? kScanThreads / F : 1;
  const int w = MULTI ? t / F : 0;
  const int fl = MULTI ? t % F : t;
  const bool tw = !MULTI || w < PPI;
  float qf[FPT][EPP];
#pragma unroll
  for (int k = 0; k < FPT; ++k) {
    const int f = fl + k * kScanThreads;
    const T* qp = static_cast<const T*>(a.q) + ((size_t)bi * H + f / QPR) * D + (f % QPR) * EPP;
#pragma unroll
    for (int e = 0; e < EPP; ++e) qf[k][e] = tw && f < F ? to_f(qp[e]) : 0.f;
  }
  __syncthreads();

  // Pages are processed in batches of PB load steps: the batch's loads are all in flight
  // before the first is reduced.
  const uint4* kb16 = reinterpret_cast<const uint4*>(a.kbar_pages);
  struct Batch {
    uint4 kv[PB][FPT];
    float hv[PB][FPT];  // H of the lane's head (read by the lane that writes the score)
    int pg[PB];
  };
  auto load = [&](Batch& B, int j0) {
#pragma unroll
    for (int u = 0; u < PB; ++u) {
      const int j = j0 + u * PPI + w;
      B.pg[u] = tw && j < nc ? s_page[j] : -1;
      const bool ok = B.pg[u] >= 0 && B.pg[u] < a.n_pages;
#pragma unroll
      for (int k = 0; k < FPT; ++k) {
        const int f = fl + k * kScanThreads;
        B.kv[u][k] = ok && f < F ? __ldg(kb16 + (size_t)B.pg[u] * F + f) : make_uint4(0, 0, 0, 0);
        B.hv[u][k] = ok && f < F && f % QPR == 0 ? __ldg(a.hbias_pages + (size_t)B.pg[u] * H + f / QPR) : 0.f;
      }
    }
  };
  auto reduce = [&](const Batch& B, int j0) {
#pragma unroll
    for (int u = 0; u < PB; ++u) {
      const int j = j0 + u * PPI + w;
#pragma unroll
      for (int k = 0; k < FPT; ++k) {
        const int f = fl + k * kScanThreads;
        float x[EPP];
        if constexpr (sizeof(S) == 2) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&B.kv[u][k]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 y = __bfloat1622float2(h2[i]);
            x[2 * i] = y.x;
            x[2 * i + 1] = y.y;
          }
        } else {
          x[0] = __uint_as_float(B.kv[u][k].x); x[1] = __uint_as_float(B.kv[u][k].y);
          x[2] = __uint_as_float(B.kv[u][k].z); x[3] = __uint_as_float(B.kv[u][k].w);
        }
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < EPP; ++e) dot = fmaf(qf[k][e], x[e], dot);
#pragma unroll
        for (int o = QPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (tw && j < nc && f < F && f % QPR == 0) {
          const int head = f / QPR, p = B.pg[u];
          float sc = NAN;
          if (p >= 0 && p < a.n_pages) sc = fmaf(dot, a.scale, B.hv[u][k]);
          else set_error(a.err, kErrBadPage);
          s_score[(size_t)j * H + head] = sc;
        }
      }
    }
  };
  for (int j0 = 0; j0 < nc; j0 += PB * PPI) {
    Batch bt_;
    load(bt_, j0);
    reduce(bt_, j0);
  }
  __syncthreads();

  // per KV head: this range's best K (merged into the head's Top-K by the attention kernel)
  const int E = nc <= 32 ? 1 : nc <= 64 ? 2 : nc <= 128 ? 4 : 8;
  for (int gi = warp; gi < a.g; gi += kScanWarps) {
    unsigned long long* part = a.part_keys + (((size_t)bi * a.g + gi) * a.nsplit + split) * K;
    switch (E) {
      case 1: range_topk<1, G>(s_score, H, gi, nc, c_lo, K, part); break;
      case 2: range_topk<2, G>(s_score, H, gi, nc, c_lo, K, part); break;
      case 4: range_topk<4, G>(s_score, H, gi, nc, c_lo, K, part); break;
      default: range_topk<8, G>(s_score, H, gi, nc, c_lo, K, part); break;
    }
  }
}

// ---------------------------------------------------------------------------
// Attention: one warp per half chunk (32 keys) of a local-branch chunk or of a Top-K
// slot, all G heads sharing each K/V load.  Lanes own keys for Q.K (each reads its key
// row) and output columns for P.V (V rows are read across the lanes); nothing is
// staged, so many warps fit per SM.  Each warp writes its half's (max, sum,
// unnormalised output) per head; the last CTA of the (sequence, KV head) combines the
// halves of each chunk and fuses the chunks with the inter-chunk softmax of notes
// section 5.3.  The local branch -- the own chunk, or with a sliding window the last
// n_local chunks up to the new token -- enters as one term at its exact log-mass.
constexpr int kAttWarps = 4;

// Raw register types for one lane's share of a V row (CPL elements of T).
template <int BYTES> struct RawT;
template <> struct RawT<4> { using type = uint32_t; };
template <> struct RawT<8> { using type = uint2; };
template <> struct RawT<16> { using type = uint4; };

template <typename T, int CPL>
__device__ __forceinline__ void raw_to_f(const typename RawT<CPL * sizeof(T)>::type& r, float (&f)[CPL]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&r);
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < CPL; ++i) f[i] = __uint_as_float(w[i]);
  }
}

template <typename T>
__device__ __forceinline__ void load_row16(const T* src, float (&f)[16 / sizeof(T)]) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(h[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  } else {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kAttWarps * 32, G == 1 ? 8 : 3) decode_attend_kernel(DecodeArgs a) {
  constexpr int CPL = D / 32;                  // output columns per lane (adjacent)
  constexpr int EPP = 16 / (int)sizeof(T);     // elements per 16-byte piece
  constexpr int PPR = D / EPP;                 // pieces per key row
  __shared__ __align__(16) float qS[G][D];
  __shared__ float s_w[G][2 * (kMaxTopK + kMaxDecodeLocal)];  // fusion weight of each half chunk, per head
  __shared__ __align__(16) unsigned long long s_win[kStageKeys];  // the merging warp's window of list keys
  __shared__ unsigned long long s_grp[kGroupKeys];                // group results of a grouped merge
  __shared__ unsigned long long s_key[kMaxTopK];                  // the selection: key of each slot (0: empty)
  __shared__ int s_last;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int ngrp = a.att_ctas;
  const int grp_i = blockIdx.x % ngrp;
  const int gi = (blockIdx.x / ngrp) % a.g;
  const int bi = blockIdx.x / (ngrp * a.g);
  const int K = a.top_k;
  const int NL = a.n_local;
  // item 2s + hf: slot s < NL the local chunk own - s, slot s >= NL Top-K slot s - NL; half hf
  const int n_items = 2 * (K + NL);
  const size_t part_stride = (size_t)G * (D + 2);
  float* part = a.part_att + ((size_t)bi * a.g + gi) * (size_t)n_items * part_stride;
  const int L = a.seq_lens[bi];
  for (int x = t; x < G * D; x += blockDim.x)
    qS[x / D][x % D] = to_f(static_cast<const T*>(a.q)[((size_t)bi * a.h + gi * G) * D + x]);
  __syncthreads();

  const int item = grp_i * kAttWarps + warp;
  const int hf = item & 1;
  auto run_item = [&](int c, int p, int nvalid) {
    float* dst = part + (size_t)item * part_stride;
    if (c >= 0 && (p < 0 || p >= a.n_pages)) set_error(a.err, kErrBadPage);
    const int n_half = min(32, nvalid - 32 * hf);  // valid keys in this half
    if (c < 0 || p < 0 || p >= a.n_pages || n_half <= 0) {
      if (lane < G) dst[lane * (D + 2)] = -INFINITY;  // absent
      return;
    }
    const size_t row0 = (((size_t)p * a.g + gi) * kChunk + 32 * hf) * D;
    const T* kp = static_cast<const T*>(a.k_pages) + row0;
    const T* vp = static_cast<const T*>(a.v_pages) + row0;
    // Every load of the item is issued up front (its K row for Q.K, lane = key; the
    // first VB rows of V for P.V, lane = output columns), so the item costs one memory
    // round trip when VB covers the half.
    using VRaw = typename RawT<CPL * sizeof(T)>::type;
    constexpr int VB = CPL * sizeof(T) <= 4 ? 32 : 16;  // V rows per batch (registers)
    const bool valid = lane < n_half;
    uint4 kraw[PPR];
#pragma unroll
    for (int pc = 0; pc < PPR; ++pc)
      kraw[pc] = valid ? *reinterpret_cast<const uint4*>(kp + (size_t)lane * D + pc * EPP) : make_uint4(0, 0, 0, 0);
    VRaw vraw[VB];
#pragma unroll
    for (int u = 0; u < VB; ++u)
      if (u < n_half) vraw[u] = *reinterpret_cast<const VRaw*>(vp + (size_t)u * D + lane * CPL);
    float s[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) s[hh] = 0.f;
#pragma unroll
    for (int pc = 0; pc < PPR; ++pc) {
      float f[EPP];
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&kraw[pc]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 x = __bfloat1622float2(h2[i]);
          f[2 * i] = x.x;
          f[2 * i + 1] = x.y;
        }
      } else {
        f[0] = __uint_as_float(kraw[pc].x); f[1] = __uint_as_float(kraw[pc].y);
        f[2] = __uint_as_float(kraw[pc].z); f[3] = __uint_as_float(kraw[pc].w);
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < EPP; ++e) s[hh] = fmaf(qS[hh][pc * EPP + e], f[e], s[hh]);
    }
    float pr[G], o[G][CPL];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float x = valid ? s[hh] * a.scale : -INFINITY;
      const float m = warp_max(x);
      pr[hh] = valid ? expf(x - m) : 0.f;
      const float l = warp_sum(pr[hh]);
      if (lane == 0) {
        dst[hh * (D + 2)] = m;
        dst[hh * (D + 2) + 1] = l;
      }
#pragma unroll
      for (int x2 = 0; x2 < CPL; ++x2) o[hh][x2] = 0.f;
    }
    // P.V over the rows in registers, then any further batches
    for (int j0 = 0; j0 < n_half; j0 += VB) {
      if (j0 > 0) {
#pragma unroll
        for (int u = 0; u < VB; ++u)
          if (j0 + u < n_half) vraw[u] = *reinterpret_cast<const VRaw*>(vp + (size_t)(j0 + u) * D + lane * CPL);
      }
#pragma unroll
      for (int u = 0; u < VB; ++u) {
        if (j0 + u >= n_half) break;
        float vj[CPL];
        raw_to_f<T, CPL>(vraw[u], vj);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float pj = __shfl_sync(0xffffffffu, pr[hh], (j0 + u) & 31);
#pragma unroll
          for (int x2 = 0; x2 < CPL; ++x2) o[hh][x2] = fmaf(pj, vj[x2], o[hh][x2]);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int x2 = 0; x2 < CPL; ++x2) dst[hh * (D + 2) + 2 + lane * CPL + x2] = o[hh][x2];
  };

  // the local branch does not depend on the selection: compute it before waiting
  const int own = L > 0 ? (L - 1) / kChunk : 0;
  if (item < 2 * NL && L > 0) {
    const int c = own - (item >> 1);  // absent (c < 0) before the sequence's first chunk
    run_item(c, c >= 0 && c < a.max_chunks ? a.block_table[(size_t)bi * a.max_chunks + c] : -1,
             c == own ? L - own * kChunk : kChunk);
  }
  pdl_wait_primary();
  // The Top-K of this KV head, merged from the scan's range lists by warp 0 of every CTA of
  // the (sequence, KV head): the scan grid has completed, so no CTA waits on another.
  if (K > 0) {
    if (warp == 0) {
      unsigned long long r0, r1;
      merge_lists(a.part_keys + ((size_t)bi * a.g + gi) * a.nsplit * K, a.nsplit, K, s_win, s_grp, r0, r1);
      if (lane < K) s_key[lane] = r0;
      if (lane + 32 < K) s_key[lane + 32] = r1;
    }
    __syncthreads();
  }
  if (item >= 2 * NL && item < n_items) {
    const int sl = (item >> 1) - NL;
    const unsigned long long key = s_key[sl];
    const int c = key ? (int)key_chunk(key) : -1;  // a candidate: c < max_chunks
    const int p = c >= 0 ? a.block_table[(size_t)bi * a.max_chunks + c] : -1;
    if (L > 0) run_item(c, p, kChunk);
    if (hf == 0) {
      // the slot's outputs, written once: its chunk, and each query head's own score of it
      // (G = 1: the selection key is the head's own score)
      if (lane == 0) a.idx[((size_t)bi * a.g + gi) * K + sl] = c;
      if constexpr (G == 1) {
        if (lane == 0) a.ssel[((size_t)bi * a.h + gi) * K + sl] = key ? unorderable((uint32_t)(key >> 32)) : -INFINITY;
      } else {
        float acc[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) acc[hh] = 0.f;
        if (c >= 0 && p >= 0 && p < a.n_pages) {  // a selected chunk's page was valid when it was scored
          const size_t row0 = ((size_t)p * a.h + gi * G) * D;
          if (a.kbar_bf16) {
            const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(a.kbar_pages) + row0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
#pragma unroll
              for (int e = lane; e < D; e += 32) acc[hh] = fmaf(qS[hh][e], __bfloat162float(kb[hh * D + e]), acc[hh]);
          } else {
            const float* kb = static_cast<const float*>(a.kbar_pages) + row0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
#pragma unroll
              for (int e = lane; e < D; e += 32) acc[hh] = fmaf(qS[hh][e], __ldg(kb + hh * D + e), acc[hh]);
          }
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float dot = warp_sum(acc[hh]);
          const float sc = c >= 0 && p >= 0 && p < a.n_pages
                               ? fmaf(dot, a.scale, __ldg(a.hbias_pages + (size_t)p * a.h + gi * G + hh))
                               : -INFINITY;
          if (lane == 0) a.ssel[((size_t)bi * a.h + gi * G + hh) * K + sl] = sc;
        }
      }
    }
  }

  __threadfence();
  __syncthreads();
  if (t == 0) s_last = atomicAdd(a.att_ticket + (size_t)bi * a.g + gi, 1u) == (unsigned)(ngrp - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  T* out = static_cast<T*>(a.out);
  if (L <= 0) {
    for (int x = t; x < G * D; x += blockDim.x) out[((size_t)bi * a.h + gi * G) * D + x] = from_f<T>(0.f);
    if (t == 0) a.att_ticket[(size_t)bi * a.g + gi] = 0;
    return;
  }
  // fusion weights, one warp per head.  Every (m, l) pair and score the weights need is
  // loaded at once, one L2 round trip: lane it < 2 NL holds local half it (NL <= 16), and
  // lane s Top-K slots s and s + 32 (K <= 64) with both their halves.  The local halves
  // give (mL, lL), LSE_local = mL + log lL; a slot's chunk takes its (m, l) from its halves.
  for (int hh = warp; hh < G; hh += kAttWarps) {
    const float* sc_row = a.ssel + ((size_t)bi * a.h + gi * G + hh) * K;
    auto ml_of = [&](int it) {  // (m, l) of half item it; l is meaningful only where m is finite
      return __ldcg(reinterpret_cast<const float2*>(part + (size_t)it * part_stride + hh * (D + 2)));
    };
    const float2 loc = lane < 2 * NL ? ml_of(lane) : make_float2(-INFINITY, 0.f);
    float2 mlh[2][2];
    float lg[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int sl = lane + 32 * rr;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) mlh[rr][h2] = sl < K ? ml_of(2 * (NL + sl) + h2) : make_float2(-INFINITY, 0.f);
      lg[rr] = sl < K ? __ldcg(sc_row + sl) : -INFINITY;
    }
    const float mL = warp_max(loc.x);
    const float lL = warp_sum(loc.x == -INFINITY ? 0.f : loc.y * expf(loc.x - mL));
    const float lseL = mL + logf(lL);  // the own chunk always holds the new token: finite
    float ms[2], ls[2];
    bool ok[2];
    float M = lseL;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      ms[rr] = fmaxf(mlh[rr][0].x, mlh[rr][1].x);
      ok[rr] = ms[rr] != -INFINITY;
      ls[rr] = 0.f;
      if (ok[rr]) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
          if (mlh[rr][h2].x != -INFINITY) ls[rr] += mlh[rr][h2].y * expf(mlh[rr][h2].x - ms[rr]);
      } else {
        lg[rr] = -INFINITY;
      }
      M = fmaxf(M, lg[rr]);
    }
    M = warp_max(M);
    float z = 0.f;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) z += ok[rr] ? expf(lg[rr] - M) : 0.f;
    const float Z = warp_sum(z) + expf(lseL - M);
    // local halves: exp(LSE_local - M)/Z * o/lL, i.e. exp(m_h - M)/Z * o_h per half
    if (lane < 2 * NL) s_w[hh][lane] = loc.x == -INFINITY ? 0.f : expf(loc.x - M) / Z;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int sl = lane + 32 * rr;
      if (sl < K) {
        // selected: exp(shat - M)/(Z l) * o, with the chunk's (m, l, o) combined from its
        // halves (o_h rescaled by exp(m_h - m))
        const float wsl = !ok[rr] ? 0.f : expf(lg[rr] - M) / (Z * ls[rr]);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
          s_w[hh][2 * (NL + sl) + h2] = mlh[rr][h2].x == -INFINITY ? 0.f : wsl * expf(mlh[rr][h2].x - ms[rr]);
      }
    }
  }
  __syncthreads();
  // weighted sum of the half-chunk outputs over items [i0, i1) for (head hh, column col);
  // the partials of kFB items are all loaded before they are summed.  Absent halves were
  // never written: their values are loaded but not used.
  constexpr bool kSplit = 2 * G * D == kAttWarps * 32;  // see below
  constexpr int kFB = kSplit ? 20 : 16;
  auto wsum = [&](int hh, int col, int i0, int i1) {
    const float* pc = part + (size_t)hh * (D + 2) + 2 + col;
    float acc = 0.f;
    for (int it0 = i0; it0 < i1; it0 += kFB) {
      float v[kFB];
#pragma unroll
      for (int u = 0; u < kFB; ++u) v[u] = it0 + u < i1 ? __ldcg(pc + (size_t)(it0 + u) * part_stride) : 0.f;
#pragma unroll
      for (int u = 0; u < kFB; ++u) {
        const float w = it0 + u < i1 ? s_w[hh][it0 + u] : 0.f;
        if (w != 0.f) acc = fmaf(v[u], w, acc);
      }
    }
    return acc;
  };
  // With G D = 64 the CTA's 128 threads take (head, column) x (first or second half of
  // the items), so that K + NL <= 20 costs one round trip; the halves meet in shared memory.
  if constexpr (kSplit) {
    __shared__ float s_acc[G * D];
    const int x = t % (G * D), sp = t / (G * D);
    const int n_half = (n_items + 1) / 2;
    const float acc = wsum(x / D, x % D, sp * n_half, min(n_items, (sp + 1) * n_half));
    if (sp == 1) s_acc[x] = acc;
    __syncthreads();
    if (sp == 0) out[((size_t)bi * a.h + gi * G) * D + x] = from_f<T>(acc + s_acc[x]);
  } else {
    for (int x = t; x < G * D; x += blockDim.x)
      out[((size_t)bi * a.h + gi * G) * D + x] = from_f<T>(wsum(x / D, x % D, 0, n_items));
  }
  if (t == 0) a.att_ticket[(size_t)bi * a.g + gi] = 0;
}

template <typename T, int D, int G, typename S, int FPT, bool MULTI = false>
static cudaError_t launch_scan(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.range * a.h * sizeof(float);  // the range's scores
  cudaError_t e = cudaFuncSetAttribute(decode_scan_kernel<T, D, G, S, FPT, MULTI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_scan_kernel<T, D, G, S, FPT, MULTI><<<(unsigned)a.b * a.nsplit, kScanThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, int G, typename S>
static cudaError_t launch_scan_by_width(const DecodeArgs& a, cudaStream_t st) {
  const int f16 = a.h * D * (int)sizeof(S) / 16;  // 16-byte pieces per page of summaries
  const int fpt = (f16 + kScanThreads - 1) / kScanThreads;
  if (f16 < kScanThreads) return launch_scan<T, D, G, S, 1, true>(a, st);
  return fpt <= 1 ? launch_scan<T, D, G, S, 1>(a, st)
       : fpt <= 2 ? launch_scan<T, D, G, S, 2>(a, st)
       : fpt <= 4 ? launch_scan<T, D, G, S, 4>(a, st)
                  : launch_scan<T, D, G, S, 8>(a, st);
}

template <typename T, int D, int G>
static cudaError_t launch_decode(DecodeArgs a, cudaStream_t st) {
  const unsigned bg = (unsigned)a.b * a.g;
  if (bg == 0) return cudaSuccess;
  if (!decode_supported(a.h, D)) return cudaErrorInvalidValue;
  if (a.top_k > 0) {
    cudaError_t e;
    if (a.kbar_bf16) {
      if constexpr (sizeof(T) == 2) e = launch_scan_by_width<T, D, G, __nv_bfloat16>(a, st);
      else return cudaErrorInvalidValue;  // the compact summary cache is for bf16 models
    } else {
      e = launch_scan_by_width<T, D, G, float>(a, st);
    }
    if (e != cudaSuccess) return e;
  }
  a.att_ctas = (2 * (a.top_k + a.n_local) + kAttWarps - 1) / kAttWarps;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bg * a.att_ctas);
  cfg.blockDim = dim3(kAttWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = a.top_k > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_attend_kernel<T, D, G>, a);
}

}  // namespace hils
