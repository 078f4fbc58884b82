// Landmark summaries (HiLS notes, section 5.1): for every complete chunk and
// query head, p = softmax(l_c . k_j * scale) over the chunk's B keys,
// kbar = sum_j p_j k_j and H = -sum_j p_j log p_j, computed stably as
// H = log Z - sum_j e_j (s_j - m) / Z with e_j = exp(s_j - m), Z = sum_j e_j.
//
// One CTA per (sequence, KV head, chunk) reads the chunk's B x d keys once
// (coalesced) and serves all G query heads of the group from shared memory,
// so K crosses HBM exactly once.  The kernel is HBM-bound.
#include "common.cuh"
#include "kernels.cuh"

namespace hils {

// KB: element type of the written kbar (fp32, or bf16 for a compact paged summary cache).
template <typename T, int D, typename KB>
__global__ void __launch_bounds__(128) summarize_kernel(
    const T* __restrict__ k, const T* __restrict__ lm, KB* __restrict__ kbar,
    float* __restrict__ hbias, int h, int g, int n_seq, int n_chunks, float scale,
    const int32_t* __restrict__ page_ids, int n_pages) {
  __shared__ float kS[kChunk][D + 1];
  __shared__ float lS[D];
  __shared__ float pS[kChunk];
  __shared__ float redm[4], redz[4], redzs[4];

  const int tid = threadIdx.x;
  const int grp = h / g;
  const T* kbase;
  const T* lbase;      // landmark of query head (gi * grp) for this chunk
  size_t lm_head_stride, out_head_stride, hb_head_stride;
  KB* kb_out;
  float* hb_out;
  if (page_ids == nullptr) {
    // blockIdx.x = ((bi * g) + gi) * n_chunks + c
    const int c = blockIdx.x % n_chunks;
    const int bg = blockIdx.x / n_chunks;
    const int gi = bg % g;
    const int bi = bg / g;
    kbase = k + (((size_t)bi * g + gi) * n_seq + (size_t)c * kChunk) * D;
    lm_head_stride = (size_t)n_chunks * D;
    lbase = lm + (((size_t)bi * h + (size_t)gi * grp) * n_chunks + c) * D;
    out_head_stride = (size_t)n_chunks * D;
    kb_out = kbar + (((size_t)bi * h + (size_t)gi * grp) * n_chunks + c) * D;
    hb_head_stride = n_chunks;
    hb_out = hbias + ((size_t)bi * h + (size_t)gi * grp) * n_chunks + c;
  } else {
    // blockIdx.x = listed_index * g + gi
    const int gi = blockIdx.x % g;
    const int p = page_ids[blockIdx.x / g];
    if (p < 0 || p >= n_pages) return;  // documented: out-of-range ids are skipped
    kbase = k + (((size_t)p * g + gi) * kChunk) * D;
    lm_head_stride = D;
    lbase = lm + ((size_t)p * h + (size_t)gi * grp) * D;
    out_head_stride = D;
    kb_out = kbar + ((size_t)p * h + (size_t)gi * grp) * D;
    hb_head_stride = 1;
    hb_out = hbias + (size_t)p * h + (size_t)gi * grp;
  }

  // Stage the chunk's keys as fp32 (4 elements per thread per step).
  for (int e4 = tid; e4 < kChunk * D / 4; e4 += blockDim.x) {
    float4 v = load4(kbase + (size_t)e4 * 4);
    const int j = (e4 * 4) / D, e = (e4 * 4) % D;
    kS[j][e] = v.x; kS[j][e + 1] = v.y; kS[j][e + 2] = v.z; kS[j][e + 3] = v.w;
  }

  for (int hh = 0; hh < grp; ++hh) {
    __syncthreads();  // kS ready / previous head done with lS, pS
    for (int e = tid; e < D; e += blockDim.x) lS[e] = to_f(lbase[hh * lm_head_stride + e]);
    __syncthreads();
    float s = -INFINITY;
    if (tid < kChunk) {
      float acc = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) acc = fmaf(lS[e], kS[tid][e], acc);
      s = acc * scale;
    }
    // block max over the 64 logits (warps 0 and 1)
    float m = warp_max(s);
    if ((tid & 31) == 0) redm[tid >> 5] = m;
    __syncthreads();
    m = fmaxf(redm[0], redm[1]);
    float ex = 0.f, exs = 0.f;
    if (tid < kChunk) {
      ex = expf(s - m);
      exs = ex * (s - m);
    }
    float z = warp_sum(ex);
    float zs = warp_sum(exs);
    if ((tid & 31) == 0) { redz[tid >> 5] = z; redzs[tid >> 5] = zs; }
    __syncthreads();
    z = redz[0] + redz[1];
    zs = redzs[0] + redzs[1];
    if (tid < kChunk) pS[tid] = ex / z;
    __syncthreads();
    for (int e = tid; e < D; e += blockDim.x) {
      float acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < kChunk; ++j) acc = fmaf(pS[j], kS[j][e], acc);
      kb_out[hh * out_head_stride + e] = from_f<KB>(acc);
    }
    if (tid == 0) hb_out[hh * hb_head_stride] = logf(z) - zs / z;
  }
}

template <typename T, int D>
static cudaError_t launch_summarize(const T* k, const T* lm, void* kbar, bool kbar_bf16, float* hbias, int b,
                                    int h, int g, int n_seq, int n_chunks, float scale,
                                    const int32_t* page_ids, int n_listed, int n_pages,
                                    cudaStream_t st) {
  unsigned blocks = page_ids ? (unsigned)n_listed * g : (unsigned)b * g * n_chunks;
  if (blocks == 0) return cudaSuccess;
  if (kbar_bf16)
    summarize_kernel<T, D, __nv_bfloat16><<<blocks, 128, 0, st>>>(
        k, lm, static_cast<__nv_bfloat16*>(kbar), hbias, h, g, n_seq, n_chunks, scale, page_ids, n_pages);
  else
    summarize_kernel<T, D, float><<<blocks, 128, 0, st>>>(k, lm, static_cast<float*>(kbar), hbias, h, g, n_seq,
                                                          n_chunks, scale, page_ids, n_pages);
  return cudaGetLastError();
}

cudaError_t run_summarize(const SummarizeArgs& a, cudaStream_t st) {
  if (a.bf16) {
    auto k = static_cast<const __nv_bfloat16*>(a.k);
    auto l = static_cast<const __nv_bfloat16*>(a.lm);
    if (a.d == 64)
      return launch_summarize<__nv_bfloat16, 64>(k, l, a.kbar, a.kbar_bf16, a.hbias, a.b, a.h, a.g, a.n, a.n_chunks,
                                                 a.scale, a.page_ids, a.n_listed, a.n_pages, st);
    return launch_summarize<__nv_bfloat16, 128>(k, l, a.kbar, a.kbar_bf16, a.hbias, a.b, a.h, a.g, a.n, a.n_chunks,
                                                a.scale, a.page_ids, a.n_listed, a.n_pages, st);
  }
  auto k = static_cast<const float*>(a.k);
  auto l = static_cast<const float*>(a.lm);
  if (a.d == 64)
    return launch_summarize<float, 64>(k, l, a.kbar, a.kbar_bf16, a.hbias, a.b, a.h, a.g, a.n, a.n_chunks, a.scale,
                                       a.page_ids, a.n_listed, a.n_pages, st);
  return launch_summarize<float, 128>(k, l, a.kbar, a.kbar_bf16, a.hbias, a.b, a.h, a.g, a.n, a.n_chunks, a.scale,
                                      a.page_ids, a.n_listed, a.n_pages, st);
}

}  // namespace hils
