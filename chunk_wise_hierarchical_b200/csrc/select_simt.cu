// Chunk scores + streaming Top-K on CUDA cores (HiLS notes, section 5.2:
// shat_{i,c} = q_i . kbar_c * scale + H_c, I_i = the K best candidates;
// section 5.4: under GQA the key is the max over the group's heads).
//
// fp32 arithmetic throughout (exact for fp32 inputs up to rounding order).
// One thread per query row of one KV group; the group's G query rows live in
// shared memory, the summaries of a tile of chunks are staged in shared memory
// and read as broadcasts.  Each thread keeps its Top-K list in shared memory:
// a candidate replaces the current worst entry when its packed key (score,
// then lower chunk index) is larger; chunks arrive in increasing index order
// so equal scores keep the earlier chunk.
#include "common.cuh"
#include "kernels.cuh"

namespace hils {

constexpr int kSelCT = 4;  // chunks per staged tile

template <typename T, int D, int G>
__global__ void select_simt_kernel(SelectArgs a, int qt) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int t = threadIdx.x;
  const int K = a.top_k;
  // carve: qS [qt][G*D+1] f32 | kbS [CT][G][D] f32 | hbS [CT][G] | keyL [K][qt] u64 | scL [K][G][qt] f32
  float* qS = reinterpret_cast<float*>(smem_raw);
  const int qstride = G * D + 1;
  float* kbS = qS + qt * qstride;
  float* hbS = kbS + kSelCT * G * D;
  unsigned long long* keyL =
      reinterpret_cast<unsigned long long*>(hbS + ((kSelCT * G + 1) & ~1));  // 8-byte aligned
  float* scL = reinterpret_cast<float*>(keyL + (size_t)K * qt);

  const int n_qtiles = (a.n + qt - 1) / qt;
  const int qtile = blockIdx.x % n_qtiles;
  const int gi = (blockIdx.x / n_qtiles) % a.g;
  const int bi = blockIdx.x / (n_qtiles * a.g);
  const int i = qtile * qt + t;
  const bool active = i < a.n;
  const int n_cand = active ? n_candidates(i, a.n_local, a.n_chunks) : 0;

  // stage q rows of the G heads (fp32)
  for (int hh = 0; hh < G; ++hh) {
    const T* qrow = static_cast<const T*>(a.q) + (((size_t)bi * a.h + gi * G + hh) * a.n + i) * D;
    for (int e = 0; e < D; e += 4) {
      float4 v = active ? load4(qrow + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      float* dst = qS + t * qstride + hh * D + e;
      dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
  }
  int last_i = min(a.n - 1, qtile * qt + qt - 1);
  const int tile_cand = n_candidates(last_i, a.n_local, a.n_chunks);

  int cnt = 0, minpos = 0;
  unsigned long long minkey = ~0ull;
  for (int c0 = 0; c0 < tile_cand; c0 += kSelCT) {
    __syncthreads();
    for (int x = t; x < kSelCT * G * D; x += blockDim.x) {
      const int c = c0 + x / (G * D);
      const int hh = (x / D) % G;
      const int e = x % D;
      kbS[x] = c < a.n_chunks
                   ? a.kbar[(((size_t)bi * a.h + gi * G + hh) * a.n_chunks + c) * D + e]
                   : 0.f;
    }
    for (int x = t; x < kSelCT * G; x += blockDim.x) {
      const int c = c0 + x / G, hh = x % G;
      hbS[x] = c < a.n_chunks ? a.hbias[((size_t)bi * a.h + gi * G + hh) * a.n_chunks + c] : 0.f;
    }
    __syncthreads();
    float sc[kSelCT][G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float acc[kSelCT];
#pragma unroll
      for (int cc = 0; cc < kSelCT; ++cc) acc[cc] = 0.f;
      const float* qr = qS + t * qstride + hh * D;
#pragma unroll 4
      for (int e = 0; e < D; ++e) {
        const float qe = qr[e];
#pragma unroll
        for (int cc = 0; cc < kSelCT; ++cc) acc[cc] = fmaf(qe, kbS[(cc * G + hh) * D + e], acc[cc]);
      }
#pragma unroll
      for (int cc = 0; cc < kSelCT; ++cc) sc[cc][hh] = fmaf(acc[cc], a.scale, hbS[cc * G + hh]);
    }
#pragma unroll
    for (int cc = 0; cc < kSelCT; ++cc) {
      const int c = c0 + cc;
      if (c >= n_cand || K == 0) continue;
      float best = sc[cc][0];
#pragma unroll
      for (int hh = 1; hh < G; ++hh) best = fmaxf(best, sc[cc][hh]);
      const unsigned long long key = pack_key(best, c);
      int pos = -1;
      if (cnt < K) {
        pos = cnt++;
        if (key < minkey) { minkey = key; minpos = pos; }
      } else if (key > minkey) {
        pos = minpos;
      }
      if (pos >= 0) {
        keyL[(size_t)pos * qt + t] = key;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) scL[((size_t)pos * G + hh) * qt + t] = sc[cc][hh];
        if (pos == minpos && cnt == K) {
          // rescan for the new worst entry
          minkey = ~0ull;
          for (int s = 0; s < K; ++s) {
            unsigned long long kk = keyL[(size_t)s * qt + t];
            if (kk < minkey) { minkey = kk; minpos = s; }
          }
        }
      }
    }
  }
  if (!active) return;
  // emit in descending key order (selection sort over the list)
  int32_t* idx_out = a.idx + (((size_t)bi * a.g + gi) * a.n + i) * K;
  for (int s = 0; s < K; ++s) {
    int bpos = -1;
    unsigned long long bkey = 0;
    for (int x = 0; x < cnt; ++x) {
      unsigned long long kk = keyL[(size_t)x * qt + t];
      if (kk > bkey) { bkey = kk; bpos = x; }
    }
    if (bpos < 0) {
      idx_out[s] = -1;
      if (a.score)
        for (int hh = 0; hh < G; ++hh)
          a.score[(((size_t)bi * a.h + gi * G + hh) * a.n + i) * K + s] = -INFINITY;
      continue;
    }
    idx_out[s] = key_chunk(bkey);
    if (a.score)
      for (int hh = 0; hh < G; ++hh)
        a.score[(((size_t)bi * a.h + gi * G + hh) * a.n + i) * K + s] = scL[((size_t)bpos * G + hh) * qt + t];
    keyL[(size_t)bpos * qt + t] = 0;
  }
}

// Register variant for K <= 32: one thread per (query, head) -- thread t takes query
// t / G and head t % G of its KV group, so a thread holds one d-row of q (shared
// memory, padded rows) and computes its head's scores; the group's max comes from
// shuffles over its G consecutive lanes.  Every lane of a group keeps the same list of
// the best KP (key, chunk) pairs sorted by key in registers, plus its own head's score
// of each listed chunk (shifted together with the keys).  Chunks arrive in increasing
// index order, so a strict fp32 comparison of keys keeps the lower index first among
// equal keys; non-finite keys never enter.
template <int KP>
__device__ __forceinline__ void sorted_insert2(float (&L)[KP], int (&I)[KP], float (&S)[KP], float x, int c,
                                               float sx) {
#pragma unroll
  for (int j = KP - 1; j > 0; --j) {
    const bool above_prev = x > L[j - 1];
    const bool above_here = x > L[j];
    L[j] = above_prev ? L[j - 1] : (above_here ? x : L[j]);
    I[j] = above_prev ? I[j - 1] : (above_here ? c : I[j]);
    S[j] = above_prev ? S[j - 1] : (above_here ? sx : S[j]);
  }
  if (x > L[0]) {
    L[0] = x;
    I[0] = c;
    S[0] = sx;
  }
}

template <typename T, int D, int G, int KP>
__global__ void __launch_bounds__(128) select_group_kernel(SelectArgs a) {
  constexpr int QT = 128 / G;  // queries per CTA
  constexpr int QS = D + 1;    // padded q row (floats)
  constexpr int KS = D + 1;    // padded summary row
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qS = reinterpret_cast<float*>(smem_raw);  // [128][QS]
  float* kbS = qS + 128 * QS;                      // [kSelCT][G][KS]
  float* hbS = kbS + kSelCT * G * KS;              // [kSelCT][G]
  const int t = threadIdx.x, lane = t & 31;
  const int hh = t % G, qo = t / G;
  const int K = a.top_k;
  const int n_qtiles = (a.n + QT - 1) / QT;
  const int qtile = blockIdx.x % n_qtiles;
  const int gi = (blockIdx.x / n_qtiles) % a.g;
  const int bi = blockIdx.x / (n_qtiles * a.g);
  const int i = qtile * QT + qo;
  const bool active = i < a.n;
  const int n_cand = active ? n_candidates(i, a.n_local, a.n_chunks) : 0;
  const size_t head = (size_t)bi * a.h + gi * G + hh;
  {
    const T* qrow = static_cast<const T*>(a.q) + (head * a.n + (active ? i : 0)) * D;
    for (int e = 0; e < D; e += 4) {
      const float4 v = active ? load4(qrow + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      float* dst = qS + t * QS + e;
      dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    }
  }
  const int last_i = min(a.n - 1, qtile * QT + QT - 1);
  const int tile_cand = n_candidates(last_i, a.n_local, a.n_chunks);
  float L[KP], Sc[KP];
  int I[KP];
#pragma unroll
  for (int s = 0; s < KP; ++s) {
    L[s] = -INFINITY;  // below every candidate
    I[s] = -1;
    Sc[s] = -INFINITY;
  }
  for (int c0 = 0; c0 < tile_cand; c0 += kSelCT) {
    __syncthreads();
    for (int x = t; x < kSelCT * G * D; x += blockDim.x) {
      const int cc = x / (G * D), h2 = (x / D) % G, e = x % D;
      const int c = c0 + cc;
      kbS[(cc * G + h2) * KS + e] =
          c < a.n_chunks ? a.kbar[(((size_t)bi * a.h + gi * G + h2) * a.n_chunks + c) * D + e] : 0.f;
    }
    for (int x = t; x < kSelCT * G; x += blockDim.x) {
      const int c = c0 + x / G, h2 = x % G;
      hbS[x] = c < a.n_chunks ? a.hbias[((size_t)bi * a.h + gi * G + h2) * a.n_chunks + c] : 0.f;
    }
    __syncthreads();
    float acc[kSelCT];
#pragma unroll
    for (int cc = 0; cc < kSelCT; ++cc) acc[cc] = 0.f;
    const float* qr = qS + t * QS;
#pragma unroll 8
    for (int e = 0; e < D; ++e) {
      const float qe = qr[e];
#pragma unroll
      for (int cc = 0; cc < kSelCT; ++cc) acc[cc] = fmaf(qe, kbS[(cc * G + hh) * KS + e], acc[cc]);
    }
#pragma unroll
    for (int cc = 0; cc < kSelCT; ++cc) {
      const int c = c0 + cc;
      const float own = fmaf(acc[cc], a.scale, hbS[cc * G + hh]);
      float best = own;
#pragma unroll
      for (int o = 1; o < G; o <<= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
      if (c < n_cand && best > L[KP - 1]) sorted_insert2(L, I, Sc, best, c, own);
    }
  }
  (void)lane;
  if (!active) return;
  int32_t* idx_out = a.idx + (((size_t)bi * a.g + gi) * a.n + i) * K;
  float* sc_out = a.score ? a.score + (head * a.n + i) * K : nullptr;
#pragma unroll
  for (int s = 0; s < KP; ++s) {
    if (s < K) {
      if (hh == 0) idx_out[s] = I[s];
      if (sc_out) sc_out[s] = I[s] >= 0 ? Sc[s] : -INFINITY;
    }
  }
}

static size_t group_smem(int G, int D) {
  return ((size_t)128 * (D + 1) + (size_t)kSelCT * G * (D + 1) + kSelCT * G) * 4;
}

template <typename T, int D, int G, int KP>
static cudaError_t launch_group(const SelectArgs& a, cudaStream_t st) {
  const size_t smem = group_smem(G, D);
  cudaError_t e = cudaFuncSetAttribute(select_group_kernel<T, D, G, KP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  constexpr int QT = 128 / G;
  const long long blocks = (long long)((a.n + QT - 1) / QT) * a.g * a.b;
  if (blocks == 0) return cudaSuccess;
  select_group_kernel<T, D, G, KP><<<(unsigned)blocks, 128, smem, st>>>(a);
  return cudaGetLastError();
}

static size_t select_smem(int qt, int G, int D, int K) {
  size_t f = (size_t)qt * (G * D + 1) + kSelCT * G * D + ((kSelCT * G + 1) & ~1);
  return f * 4 + (size_t)K * qt * 8 + (size_t)K * G * qt * 4;
}

template <typename T, int D, int G>
static cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  int qt = 128;
  while (qt > 16 && select_smem(qt, G, D, a.top_k) > 200 * 1024) qt >>= 1;
  size_t smem = select_smem(qt, G, D, a.top_k);
  if (smem > 220 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(select_simt_kernel<T, D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)((a.n + qt - 1) / qt) * a.g * a.b;
  if (blocks == 0) return cudaSuccess;
  select_simt_kernel<T, D, G><<<(unsigned)blocks, qt, smem, st>>>(a, qt);
  return cudaGetLastError();
}

template <typename T, int D, int G>
static cudaError_t launch_by_k(const SelectArgs& a, cudaStream_t st) {
  if (a.top_k <= 16) return launch_group<T, D, G, 16>(a, st);
  if (a.top_k <= 32) return launch_group<T, D, G, 32>(a, st);
  return launch_select<T, D, G>(a, st);  // K up to 64: lists in shared memory
}

template <typename T, int D>
static cudaError_t select_by_group(const SelectArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_by_k<T, D, 1>(a, st);
    case 2: return launch_by_k<T, D, 2>(a, st);
    case 4: return launch_by_k<T, D, 4>(a, st);
    case 8: return launch_by_k<T, D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_select_simt(const SelectArgs& a, cudaStream_t st) {
  if (a.bf16) return a.d == 64 ? select_by_group<__nv_bfloat16, 64>(a, st) : select_by_group<__nv_bfloat16, 128>(a, st);
  return a.d == 64 ? select_by_group<float, 64>(a, st) : select_by_group<float, 128>(a, st);
}

}  // namespace hils
