// Single-token decode over a paged chunk cache (HiLS notes, sections 5.2-5.4,
// applied to the newest query of each sequence).  Two HBM-bound kernels,
// chained with programmatic dependent launch:
//
// 1. decode_scan_kernel -- grid (sequence, KV head, range of kScanChunks
//    candidate chunks).  Each CTA scores its range against the cached
//    summaries (q . kbar * scale + H, GQA max over the group's heads), sorts
//    the range's packed keys (bitonic, shared memory) and writes its best K.
//    The last CTA of the (sequence, KV head) -- an atomic ticket; no CTA waits
//    on another -- merges the lists into the final Top-K and writes each
//    head's own score of the selected chunks.
// 2. decode_attend_kernel -- one warp per chunk (own chunk or one Top-K slot),
//    all G heads sharing each K/V load, K and V staged in shared memory with
//    cp.async.  The own chunk does not depend on the selection and is
//    computed before the kernel waits for the scan grid.  Each warp writes
//    its chunk's (max, sum, unnormalised output); the last CTA of the
//    (sequence, KV head) fuses them with the inter-chunk softmax of notes
//    section 5.3 (own chunk at its exact log-mass).
// Tickets are reset by the CTA that consumes them, so both kernels can be
// replayed (CUDA graphs) without clearing the workspace.
#include "common.cuh"
#include "kernels.cuh"

namespace hils {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanChunks = 128;   // candidate chunks per scan CTA (power of two)
constexpr int kMergeCap = 2048;    // keys the merging CTA sorts at once (power of two)

// chunks (warps) per attend CTA: K and V of a chunk are staged per warp, so wide rows get fewer warps
template <typename T, int D>
__host__ __device__ constexpr int att_warps() { return sizeof(T) * D <= 256 ? 4 : 2; }

int decode_splits(int max_chunks) { return max(1, (max_chunks + kScanChunks - 1) / kScanChunks); }

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Descending bitonic sort of keys[0..n), n a power of two; the whole block calls it.
template <int THREADS>
__device__ void block_sort_desc(unsigned long long* keys, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (x < y) : (x > y)) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kScanThreads) decode_scan_kernel(DecodeArgs a) {
  constexpr int LPR = D / 4;              // lanes per summary row (one float4 each)
  constexpr int RPW = 32 / LPR;           // rows per warp step
  __shared__ unsigned long long s_keys[kMergeCap];
  __shared__ float s_score[kScanChunks * G];
  __shared__ int s_page[kScanChunks];
  __shared__ int s_sel[kMaxTopK];
  __shared__ int s_last;

  pdl_launch_dependents();  // the attend grid may start its selection-independent prologue
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // CTA order (sequence, range, KV head): the CTAs of all heads of one range run
  // together, so each page's summary block is read from DRAM in one burst
  const int gi = blockIdx.x % a.g;
  const int split = (blockIdx.x / a.g) % a.nsplit;
  const int bi = blockIdx.x / (a.nsplit * a.g);
  const int K = a.top_k;
  const int c_lo = split * kScanChunks;
  const int32_t* bt = a.block_table + (size_t)bi * a.max_chunks;
  // block-table slice and the query are loaded alongside the sequence length
  for (int x = t; x < kScanChunks; x += kScanThreads)
    s_page[x] = c_lo + x < a.max_chunks ? bt[c_lo + x] : -1;
  const int sub = lane % LPR;
  float4 qv[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
    qv[hh] = load4(static_cast<const T*>(a.q) + ((size_t)bi * a.h + gi * G + hh) * D + sub * 4);
  const int L = a.seq_lens[bi];
  const int own = L > 0 ? (L - 1) / kChunk : 0;
  const int n_cand = min(own, a.max_chunks);
  const int nc = max(0, min(n_cand, c_lo + kScanChunks) - c_lo);
  __syncthreads();

  // score rows (chunk, head): every warp issues kBatch loads before reducing them
  constexpr int kBatch = 8;
  const int n_rows = nc * G;
  const int step = kScanWarps * RPW;
  for (int r0 = warp * RPW; r0 < n_rows; r0 += step * kBatch) {
    float4 kv[kBatch];
    int pg[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = r0 + u * step + lane / LPR;
      pg[u] = -1;
      kv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < n_rows) {
        const int p = s_page[r / G];
        if (p >= 0 && p < a.n_pages) {
          pg[u] = p;
          kv[u] = __ldg(reinterpret_cast<const float4*>(a.kbar_pages + ((size_t)p * a.h + gi * G + r % G) * D + sub * 4));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = r0 + u * step + lane / LPR;
      const int hh = r % G;
      float4 q = qv[0];
#pragma unroll
      for (int x = 1; x < G; ++x)
        if (hh == x) q = qv[x];
      float dot = fmaf(q.x, kv[u].x, fmaf(q.y, kv[u].y, fmaf(q.z, kv[u].z, q.w * kv[u].w)));
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (r < n_rows && sub == 0) {
        const int p = pg[u];
        if (p < 0) set_error(a.err, kErrBadPage);
        s_score[r] = p >= 0 ? fmaf(dot, a.scale, __ldg(a.hbias_pages + (size_t)p * a.h + gi * G + hh)) : NAN;
      }
    }
  }
  __syncthreads();
  for (int cl = t; cl < kScanChunks; cl += kScanThreads) {
    unsigned long long key = 0;
    if (cl < nc) {
      float best = -INFINITY;
      bool bad = false;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float v = s_score[cl * G + hh];
        bad |= (v != v);
        best = fmaxf(best, v);
      }
      key = bad ? 0ull : pack_key(best, c_lo + cl);
    }
    s_keys[cl] = key;
  }
  __syncthreads();
  block_sort_desc<kScanThreads>(s_keys, kScanChunks);
  unsigned long long* part = a.part_keys + (((size_t)bi * a.g + gi) * a.nsplit + split) * K;
  for (int s = t; s < K; s += kScanThreads) part[s] = s_keys[s];
  __threadfence();
  __syncthreads();
  if (t == 0) s_last = atomicAdd(a.scan_ticket + (size_t)bi * a.g + gi, 1u) == (unsigned)(a.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA: merge the per-range lists (running best K + next slice) ----
  const unsigned long long* parts = a.part_keys + ((size_t)bi * a.g + gi) * a.nsplit * K;
  const int n_all = a.nsplit * K;
  for (int x = t; x < K; x += kScanThreads) s_keys[x] = 0;
  for (int start = 0; start < n_all; start += kMergeCap - K) {
    const int take = min(kMergeCap - K, n_all - start);
    const int n2 = pow2_ceil(K + take);
    __syncthreads();
    for (int x = t; x < n2 - K; x += kScanThreads) s_keys[K + x] = x < take ? __ldcg(parts + start + x) : 0ull;
    __syncthreads();
    block_sort_desc<kScanThreads>(s_keys, n2);
  }
  for (int s = t; s < K; s += kScanThreads) {
    const unsigned long long key = s_keys[s];
    s_sel[s] = key ? key_chunk(key) : -1;
  }
  __syncthreads();
  for (int s = t; s < K; s += kScanThreads) {
    const int c = s_sel[s];
    a.idx[((size_t)bi * a.g + gi) * K + s] = c;
    a.sel_page[((size_t)bi * a.g + gi) * K + s] = c >= 0 ? bt[c] : -1;
  }
  if constexpr (G == 1) {
    // the selection key is the head's own score
    for (int s = t; s < K; s += kScanThreads) {
      const unsigned long long key = s_keys[s];
      a.ssel[((size_t)bi * a.h + gi) * K + s] = key ? unorderable((uint32_t)(key >> 32)) : -INFINITY;
    }
  } else {
    // each head's own score of the selected chunks: one warp per (slot, head)
    for (int x = warp; x < K * G; x += kScanWarps) {
      const int s = x / G, hh = x % G;
      const int c = s_sel[s];
      float sc = -INFINITY;
      if (c >= 0) {
        const int p = bt[c];
        const float* kb = a.kbar_pages + ((size_t)p * a.h + gi * G + hh) * D;
        const T* qr = static_cast<const T*>(a.q) + ((size_t)bi * a.h + gi * G + hh) * D;
        float acc = 0.f;
#pragma unroll
        for (int e = lane; e < D; e += 32) acc = fmaf(to_f(qr[e]), __ldg(kb + e), acc);
        acc = warp_sum(acc);
        sc = fmaf(acc, a.scale, __ldg(a.hbias_pages + (size_t)p * a.h + gi * G + hh));
      }
      if (lane == 0) a.ssel[((size_t)bi * a.h + gi * G + hh) * K + s] = sc;
    }
  }
  if (t == 0) a.scan_ticket[(size_t)bi * a.g + gi] = 0;
}

// ---------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(att_warps<T, D>() * 32) decode_attend_kernel(DecodeArgs a) {
  constexpr int kAttWarps = att_warps<T, D>();
  constexpr int CPL = D / 32;                 // output columns per lane (adjacent)
  constexpr int RS = D + 16 / (int)sizeof(T); // padded shared row (elements): rows hit different banks
  extern __shared__ __align__(16) unsigned char dyn[];
  T* s_kv = reinterpret_cast<T*>(dyn);        // [warps][2][64][RS]
  __shared__ __align__(16) float qS[G][D];
  __shared__ float s_w[kAttWarps][kMaxTopK + 1];
  __shared__ int s_last;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int ngrp = a.att_ctas;
  const int grp_i = blockIdx.x % ngrp;
  const int gi = (blockIdx.x / ngrp) % a.g;
  const int bi = blockIdx.x / (ngrp * a.g);
  const int K = a.top_k;
  const int n_items = K + 1;                  // item 0: own chunk; item s >= 1: Top-K slot s-1
  const size_t part_stride = (size_t)G * (D + 2);
  float* part = a.part_att + ((size_t)bi * a.g + gi) * (size_t)n_items * part_stride;
  const int L = a.seq_lens[bi];
  for (int x = t; x < G * D; x += blockDim.x)
    qS[x / D][x % D] = to_f(static_cast<const T*>(a.q)[((size_t)bi * a.h + gi * G) * D + x]);
  __syncthreads();

  T* sk = s_kv + (size_t)warp * 2 * kChunk * RS;
  T* sv = sk + (size_t)kChunk * RS;
  const int item = grp_i * kAttWarps + warp;
  // one chunk: returns false if absent
  auto run_item = [&](int c, int p, int nvalid) {
    float* dst = part + (size_t)item * part_stride;
    if (c >= 0 && (p < 0 || p >= a.n_pages)) set_error(a.err, kErrBadPage);
    if (c < 0 || p < 0 || p >= a.n_pages) {
      if (lane < G) dst[lane * (D + 2)] = -INFINITY;  // absent
      return;
    }
    const T* kp = static_cast<const T*>(a.k_pages) + (((size_t)p * a.g + gi) * kChunk) * D;
    const T* vp = static_cast<const T*>(a.v_pages) + (((size_t)p * a.g + gi) * kChunk) * D;
    constexpr int CH = D * (int)sizeof(T) / 16;  // 16-byte pieces per row
    for (int x = lane; x < kChunk * CH; x += 32) {
      const int r = x / CH, ch = x % CH;
      const uint32_t bytes = r < nvalid ? 16u : 0u;
      const size_t src = r < nvalid ? (size_t)r * D + ch * (16 / sizeof(T)) : 0;
      const uint32_t dk = (uint32_t)__cvta_generic_to_shared(sk + (size_t)r * RS + ch * (16 / sizeof(T)));
      const uint32_t dv = (uint32_t)__cvta_generic_to_shared(sv + (size_t)r * RS + ch * (16 / sizeof(T)));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dk), "l"(kp + src), "r"(bytes) : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dv), "l"(vp + src), "r"(bytes) : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    const int j0 = lane, j1 = lane + 32;
    const bool v0 = j0 < nvalid, v1 = j1 < nvalid;
    float s0[G], s1[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) { s0[hh] = 0.f; s1[hh] = 0.f; }
#pragma unroll 8
    for (int e = 0; e < D; e += 4) {
      const float4 k0 = load4(sk + (size_t)j0 * RS + e);
      const float4 k1 = load4(sk + (size_t)j1 * RS + e);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float4 qv = *reinterpret_cast<const float4*>(&qS[hh][e]);
        s0[hh] = fmaf(qv.x, k0.x, fmaf(qv.y, k0.y, fmaf(qv.z, k0.z, fmaf(qv.w, k0.w, s0[hh]))));
        s1[hh] = fmaf(qv.x, k1.x, fmaf(qv.y, k1.y, fmaf(qv.z, k1.z, fmaf(qv.w, k1.w, s1[hh]))));
      }
    }
    float p0[G], p1[G], o[G][CPL];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float a0 = v0 ? s0[hh] * a.scale : -INFINITY;
      const float a1 = v1 ? s1[hh] * a.scale : -INFINITY;
      const float m = warp_max(fmaxf(a0, a1));
      p0[hh] = v0 ? expf(a0 - m) : 0.f;
      p1[hh] = v1 ? expf(a1 - m) : 0.f;
      const float l = warp_sum(p0[hh] + p1[hh]);
      if (lane == 0) {
        dst[hh * (D + 2)] = m;
        dst[hh * (D + 2) + 1] = l;
      }
#pragma unroll
      for (int x = 0; x < CPL; ++x) o[hh][x] = 0.f;
    }
    for (int j = 0; j < nvalid; ++j) {
      float vj[CPL];
      if constexpr (CPL == 2) {
        const float2 f = sizeof(T) == 2
                             ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sv + (size_t)j * RS + lane * 2))
                             : *reinterpret_cast<const float2*>(sv + (size_t)j * RS + lane * 2);
        vj[0] = f.x;
        vj[1] = f.y;
      } else {
        const float4 f = load4(sv + (size_t)j * RS + lane * 4);
        vj[0] = f.x; vj[1] = f.y; vj[2] = f.z; vj[3] = f.w;
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0[hh] : p1[hh], j & 31);
#pragma unroll
        for (int x = 0; x < CPL; ++x) o[hh][x] = fmaf(pj, vj[x], o[hh][x]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int x = 0; x < CPL; ++x) dst[hh * (D + 2) + 2 + lane * CPL + x] = o[hh][x];
  };

  // the own chunk does not depend on the selection: compute it before waiting
  const int own = L > 0 ? (L - 1) / kChunk : 0;
  if (item == 0 && L > 0)
    run_item(own, own < a.max_chunks ? a.block_table[(size_t)bi * a.max_chunks + own] : -1, L - own * kChunk);
  pdl_wait_primary();
  if (item >= 1 && item < n_items && L > 0) {
    const size_t slot = ((size_t)bi * a.g + gi) * K + item - 1;
    run_item(a.idx[slot], a.sel_page[slot], kChunk);
  }

  __threadfence();
  __syncthreads();
  if (t == 0) s_last = atomicAdd(a.att_ticket + (size_t)bi * a.g + gi, 1u) == (unsigned)(ngrp - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  T* out = static_cast<T*>(a.out);
  // fusion, one warp per head: lane s holds item s (3 rounds cover K + 1 <= 65 items)
  for (int hh = warp; hh < G; hh += kAttWarps) {
    T* orow = out + ((size_t)bi * a.h + gi * G + hh) * D;
    if (L <= 0) {
      for (int x = lane; x < D; x += 32) orow[x] = from_f<T>(0.f);
      continue;
    }
    const float* sc_row = a.ssel + ((size_t)bi * a.h + gi * G + hh) * K;
    float lg[3], mm[3], ll[3];
    bool ok[3];
    float M = -INFINITY;
#pragma unroll
    for (int rr = 0; rr < 3; ++rr) {
      const int it = lane + 32 * rr;
      ok[rr] = false;
      lg[rr] = -INFINITY;
      mm[rr] = 0.f;
      ll[rr] = 1.f;
      if (it < n_items) {
        const float* pp = part + (size_t)it * part_stride + hh * (D + 2);
        mm[rr] = __ldcg(pp);
        ll[rr] = __ldcg(pp + 1);
        ok[rr] = mm[rr] != -INFINITY;
        if (ok[rr]) lg[rr] = it == 0 ? mm[rr] + logf(ll[rr]) : __ldcg(sc_row + it - 1);
      }
      M = fmaxf(M, lg[rr]);
    }
    M = warp_max(M);
    float z = 0.f;
#pragma unroll
    for (int rr = 0; rr < 3; ++rr) z += ok[rr] ? expf(lg[rr] - M) : 0.f;
    const float Z = warp_sum(z);
#pragma unroll
    for (int rr = 0; rr < 3; ++rr) {
      const int it = lane + 32 * rr;
      // own: exp(LSE_own - M)/Z * o/l = exp(m - M)/Z * o ; selected: exp(shat - M)/(Z l) * o
      if (it < n_items)
        s_w[warp][it] = !ok[rr] ? 0.f : (it == 0 ? expf(mm[rr] - M) / Z : expf(lg[rr] - M) / (Z * ll[rr]));
    }
    __syncwarp();
    float acc[CPL];
#pragma unroll
    for (int x = 0; x < CPL; ++x) acc[x] = 0.f;
#pragma unroll 4
    for (int it = 0; it < n_items; ++it) {
      const float w = s_w[warp][it];
      if (w == 0.f) continue;
      const float* pp = part + (size_t)it * part_stride + hh * (D + 2) + 2 + lane * CPL;
#pragma unroll
      for (int x = 0; x < CPL; ++x) acc[x] = fmaf(__ldcg(pp + x), w, acc[x]);
    }
#pragma unroll
    for (int x = 0; x < CPL; ++x) orow[lane * CPL + x] = from_f<T>(acc[x]);
    __syncwarp();
  }
  if (t == 0) a.att_ticket[(size_t)bi * a.g + gi] = 0;
}

template <typename T, int D, int G>
static cudaError_t launch_decode(DecodeArgs a, cudaStream_t st) {
  const unsigned bg = (unsigned)a.b * a.g;
  if (bg == 0) return cudaSuccess;
  if (a.top_k > 0) {
    decode_scan_kernel<T, D, G><<<bg * a.nsplit, kScanThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  constexpr int AW = att_warps<T, D>();
  constexpr int RS = D + 16 / (int)sizeof(T);
  constexpr size_t smem = (size_t)AW * 2 * kChunk * RS * sizeof(T);
  static_assert(smem <= 200 * 1024, "decode attention staging exceeds shared memory");
  a.att_ctas = (a.top_k + 1 + AW - 1) / AW;
  cudaError_t e = cudaFuncSetAttribute(decode_attend_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bg * a.att_ctas);
  cfg.blockDim = dim3(AW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = a.top_k > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_attend_kernel<T, D, G>, a);
}

template <typename T, int D>
static cudaError_t decode_by_group(const DecodeArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_decode<T, D, 1>(a, st);
    case 2: return launch_decode<T, D, 2>(a, st);
    case 4: return launch_decode<T, D, 4>(a, st);
    case 8: return launch_decode<T, D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_decode(DecodeArgs a, cudaStream_t st) {
  a.nsplit = decode_splits(a.max_chunks);
  if (a.bf16) return a.d == 64 ? decode_by_group<__nv_bfloat16, 64>(a, st) : decode_by_group<__nv_bfloat16, 128>(a, st);
  return a.d == 64 ? decode_by_group<float, 64>(a, st) : decode_by_group<float, 128>(a, st);
}

}  // namespace hils
