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
  const int n_cand = active ? min(i / kChunk, a.n_chunks) : 0;

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
  const int tile_cand = min(last_i / kChunk, a.n_chunks);

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

template <typename T, int D>
static cudaError_t select_by_group(const SelectArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_select<T, D, 1>(a, st);
    case 2: return launch_select<T, D, 2>(a, st);
    case 4: return launch_select<T, D, 4>(a, st);
    case 8: return launch_select<T, D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_select_simt(const SelectArgs& a, cudaStream_t st) {
  if (a.bf16) return a.d == 64 ? select_by_group<__nv_bfloat16, 64>(a, st) : select_by_group<__nv_bfloat16, 128>(a, st);
  return a.d == 64 ? select_by_group<float, 64>(a, st) : select_by_group<float, 128>(a, st);
}

}  // namespace hils
