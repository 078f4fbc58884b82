// Selected-chunk + own-chunk attention with the inter-chunk fusion on the
// 5th-generation tensor cores (tcgen05 + TMEM), bf16 inputs, fp32 accumulation.
// (HiLS notes, section 5.3: w_ij = exp(s_ij)/Z_{i,c} * exp(shat_{i,c})/Zhat_i;
// Tide digest, Figure 3.)
//
// Work decomposition ("row owner, chunk buckets").  One CTA owns a block of QB
// consecutive queries of one (sequence, KV head) and all G query heads of the
// group: R = QB*G rows whose fp32 output accumulators stay in shared memory for
// the whole CTA.  The CTA buckets its rows' selections by chunk (counting sort
// in shared memory), then walks the chunks in index order.  For chunk c the
// rows that selected it are gathered into 128-row tiles:
//     S = Q_tile K_c^T          (tcgen05, M=128 N=64, S in TMEM)
//     P'_j = exp(x_j - m) * alpha / l,  alpha = exp(shat - M) / Z'   (registers)
//     O_tile = P' V_c           (tcgen05, M=128 N=d, TMEM)
//     O[row] += O_tile[row]     (shared memory)
// so every (row, chunk) pair contributes its already-weighted term and no
// partial result leaves the SM.  The own causal chunk is processed first; it
// fixes LSE_own and with it the fusion max M and normaliser Z' of each row.
// Rows outside a tile's count are computed and ignored (padding of the
// 128-row MMA).  Summation over chunks runs in chunk-index order, so results
// do not depend on the order of rows inside a bucket.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_util.cuh"

namespace hils {

namespace {

constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct TcSmem {
  uint32_t a, k, v, p;       // byte offsets of the swizzled operand tiles
  uint32_t o;                // fp32 accumulators [R][D] (float4 XOR-swizzled by row)
  uint32_t list;             // u16 bucket entries
  uint32_t off;              // int offsets [n_cand + 1]
  uint32_t cur;              // int cursors [n_cand]
  uint32_t rowm, rowz;       // per row: fusion max M and 1/Z'
  uint32_t tile;             // per tile row: r | slot << 16
  uint32_t total;
};

__host__ __device__ inline uint32_t align_to(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline TcSmem tc_layout(int D, int G, int qb, int K, int n_cand) {
  TcSmem L;
  uint32_t off = 0;
  L.a = off; off += 128 * D * 2;
  L.k = off; off += 64 * D * 2;
  L.v = off; off += 64 * D * 2;
  L.p = off; off += 128 * 64 * 2;
  L.o = off; off += (uint32_t)qb * G * D * 4;
  L.list = off; off = align_to(off + (uint32_t)qb * K * 2, 16);
  L.off = off; off += (uint32_t)(n_cand + 1) * 4;
  L.cur = off; off = align_to(off + (uint32_t)n_cand * 4, 16);
  L.rowm = off; off += (uint32_t)qb * G * 4;
  L.rowz = off; off += (uint32_t)qb * G * 4;
  L.tile = off; off += 128 * 4;
  L.total = align_to(off, 16);
  return L;
}

__device__ __forceinline__ float4* o_row_f4(unsigned char* base, uint32_t o_off, int r, int j4, int D) {
  // float4 j4 of row r, XOR-swizzled by (r & 7) to spread rows over banks
  return reinterpret_cast<float4*>(base + o_off + (size_t)r * D * 4 + (size_t)((j4 ^ (r & 7)) * 16));
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(TcAttendArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_base_s;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int N = a.n, K = a.top_k, QB = a.qb;
  const int nqb = (N + QB - 1) / QB;
  const int blk = blockIdx.x % nqb;
  const int gi = (blockIdx.x / nqb) % a.g;
  const int bi = blockIdx.x / (nqb * a.g);
  const int q0 = blk * QB;
  const int nq = min(QB, N - q0);
  const int head0 = gi * G;
  const int n_cand = min((q0 + nq - 1) / kChunk, N / kChunk);  // chunks any row of the block may select
  const TcSmem L = tc_layout(D, G, QB, K, a.n_cand_max);
  constexpr uint32_t kTmemCols = D == 64 ? 128 : 256;

  uint16_t* s_list = reinterpret_cast<uint16_t*>(sm + L.list);
  int* s_off = reinterpret_cast<int*>(sm + L.off);
  int* s_cur = reinterpret_cast<int*>(sm + L.cur);
  float* s_rowm = reinterpret_cast<float*>(sm + L.rowm);
  float* s_rowz = reinterpret_cast<float*>(sm + L.rowz);
  uint32_t* s_tile = reinterpret_cast<uint32_t*>(sm + L.tile);
  const uint32_t sA = tc::smem_u32(sm + L.a), sK = tc::smem_u32(sm + L.k), sV = tc::smem_u32(sm + L.v),
                 sP = tc::smem_u32(sm + L.p);
  const uint32_t barS = tc::smem_u32(&bars[0]), barO = tc::smem_u32(&bars[1]);

  const __nv_bfloat16* qg = a.q + ((size_t)bi * a.h + head0) * N * D;       // head0 rows
  const __nv_bfloat16* kg = a.k + ((size_t)bi * a.g + gi) * N * D;
  const __nv_bfloat16* vg = a.v + ((size_t)bi * a.g + gi) * N * D;
  const int32_t* idxg = a.idx + ((size_t)bi * a.g + gi) * N * K;
  const float* sselg = a.ssel + ((size_t)bi * a.h + head0) * N * K;

  if (tid == 0) {
    tc::mbar_init(barS, 1);
    tc::mbar_init(barO, 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(&tmem_base_s), kTmemCols);

  // ---- bucket the block's selections by chunk (counting sort) ----
  for (int c = tid; c <= n_cand; c += kThreads) s_off[c] = 0;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t tS = tmem, tO = tmem + 64;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

  for (int e = tid; e < nq * K; e += kThreads) {
    const int qo = e / K, i = q0 + qo;
    const int c = idxg[(size_t)i * K + (e % K)];
    if (c < 0) continue;
    if (c >= i / kChunk) { set_error(a.err, kErrBadPage); continue; }
    atomicAdd(&s_off[c], 1);
  }
  __syncthreads();
  {  // exclusive scan of s_off[0..n_cand) in place, s_off[n_cand] = total
    const int seg = (n_cand + kThreads - 1) / kThreads;
    const int lo = min(tid * seg, n_cand), hi = min(lo + seg, n_cand);
    int sum = 0;
    for (int c = lo; c < hi; ++c) sum += s_off[c];
    // block-wide exclusive scan of the per-thread sums
    int incl = sum;
    const int lane = tid & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __shared__ int wsum[kThreads / 32];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += wsum[w];
    int run = wbase + incl - sum;
    __syncthreads();
    for (int c = lo; c < hi; ++c) {
      const int x = s_off[c];
      s_off[c] = run;
      s_cur[c] = run;
      run += x;
    }
    if (tid == kThreads - 1) s_off[n_cand] = wbase + incl;
  }
  __syncthreads();
  for (int e = tid; e < nq * K; e += kThreads) {
    const int qo = e / K, s = e % K, i = q0 + qo;
    const int c = idxg[(size_t)i * K + s];
    if (c < 0 || c >= i / kChunk) continue;
    const int pos = atomicAdd(&s_cur[c], 1);
    s_list[pos] = (uint16_t)(qo | (s << 9));
  }
  __syncthreads();

  uint32_t phase = 0;
  bool failed = false;
  const float sc2 = a.scale * kLog2e;

  // loads one chunk's K and V (rows >= nvalid zero-filled) into the swizzled tiles
  auto load_kv = [&](int c, int nvalid) {
    const __nv_bfloat16* kc = kg + (size_t)c * kChunk * D;
    const __nv_bfloat16* vc = vg + (size_t)c * kChunk * D;
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int x = tid; x < kChunk * CH; x += kThreads) {
      const int r = x / CH, ch = x % CH;
      const uint32_t o = (uint32_t)(ch >> 3) * 8192u + tc::sw128_chunk(r, ch & 7);
      const bool ok = r < nvalid;
      const size_t src = ok ? (size_t)r * D + ch * 8 : 0;
      tc::cp_async16(sK + o, kc + src, ok ? 16 : 0);
      tc::cp_async16(sV + o, vc + src, ok ? 16 : 0);
    }
  };
  // gathers the Q rows of a tile: row t -> (query offset, head)
  auto gather_q = [&](int n_rows) {
    constexpr int CH = D / 8;
    for (int x = tid; x < n_rows * CH; x += kThreads) {
      const int t = x / CH, ch = x % CH;
      const int r = (int)(s_tile[t] & 0xffffu);
      const int qo = r / G, hh = r % G;
      const __nv_bfloat16* src = qg + ((size_t)hh * N + q0 + qo) * D + ch * 8;
      tc::cp_async16(sA + (uint32_t)(ch >> 3) * 16384u + tc::sw128_chunk(t, ch & 7), src);
    }
  };
  // S = Q K^T into TMEM (one thread)
  auto issue_s = [&]() {
    constexpr uint32_t id = tc::make_idesc_bf16(128, 64, false, false);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint64_t da = tc::make_desc(sA + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
      const uint64_t db = tc::make_desc(sK + (k >> 2) * 8192u + (k & 3) * 32u, 16, 1024);
      tc::mma_bf16(tS, da, db, id, k > 0);
    }
    tc::mma_commit(barS);
  };
  // O_tile = P V into TMEM (one thread)
  auto issue_pv = [&]() {
    constexpr uint32_t id = tc::make_idesc_bf16(128, D, false, true);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t da = tc::make_desc(sP + k * 32u, 16, 1024);
      const uint64_t db = tc::make_desc(sV + k * 2048u, 8192, 1024);
      tc::mma_bf16(tO, da, db, id, k > 0);
    }
    tc::mma_commit(barO);
  };
  // softmax of this thread's tile row (called by whole warps: the TMEM loads are
  // warp-collective); writes P' = exp(x - m) * f into the P tile when `valid`.
  // mult_after_l: f = mult / l, else f = mult.  Returns m (log2-domain max) and l.
  auto softmax_row = [&](int t, bool valid, int jmax, float mult, bool mult_after_l, float& m_out,
                         float& l_out) {
    float s[64];
    tc::tmem_ld32(tS + lane_off, s);
    tc::tmem_ld32(tS + lane_off + 32, s + 32);
    tc::tmem_wait_ld();
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      s[j] = j <= jmax ? s[j] * sc2 : -INFINITY;  // log2 domain
      m = fmaxf(m, s[j]);
    }
    float l = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      s[j] = exp2f(s[j] - m);
      l += s[j];
    }
    const float f = mult_after_l ? mult / l : mult;
    if (valid) {
      unsigned char* prow = sm + L.p;
#pragma unroll
      for (int j = 0; j < 64; j += 8) {
        uint4 pk;
        pk.x = tc::pack_bf16x2(s[j] * f, s[j + 1] * f);
        pk.y = tc::pack_bf16x2(s[j + 2] * f, s[j + 3] * f);
        pk.z = tc::pack_bf16x2(s[j + 4] * f, s[j + 5] * f);
        pk.w = tc::pack_bf16x2(s[j + 6] * f, s[j + 7] * f);
        *reinterpret_cast<uint4*>(prow + tc::sw128_chunk(t, j >> 3)) = pk;
      }
    }
    m_out = m;
    l_out = l;
  };
  // waits for an MMA group; a timeout is recorded and aborts the CTA
  auto wait_bar = [&](uint32_t bar) {
    if (!tc::mbar_wait(bar, phase)) {
      set_error(a.err, kErrTimeout);
      failed = true;
    }
  };

  // ---------------- own (causal) chunks: LSE_own, fusion constants, O init ----------------
  const int oc_first = q0 / kChunk, oc_last = (q0 + nq - 1) / kChunk;
  for (int oc = oc_first; oc <= oc_last && !failed; ++oc) {
    const int qa = max(q0, oc * kChunk) - q0, qb = min(q0 + nq, oc * kChunk + kChunk) - q0;
    load_kv(oc, min(kChunk, N - oc * kChunk));
    for (int t0 = qa * G; t0 < qb * G; t0 += 128) {
      const int n_rows = min(128, qb * G - t0);
      if (tid < n_rows) s_tile[tid] = (uint32_t)(t0 + tid);
      __syncthreads();
      gather_q(n_rows);
      tc::cp_async_wait_all();
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) issue_s();
      wait_bar(barS);
      if (__syncthreads_or(failed)) { failed = true; break; }
      tc::fence_after_sync();
      float m = 0.f, l = 1.f;
      const bool row_ok = tid < n_rows;
      const bool warp_ok = warp * 32 < n_rows;
      const int r = row_ok ? t0 + tid : 0;
      const int qo = r / G, hh = r % G, i = q0 + qo;
      if (warp_ok) softmax_row(tid, row_ok, row_ok ? i - oc * kChunk : 63, 1.0f, false, m, l);
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) issue_pv();
      wait_bar(barO);
      if (__syncthreads_or(failed)) { failed = true; break; }
      tc::fence_after_sync();
      if (warp_ok) {
        // m, l are in the log2 domain: LSE_own = (m + log2 l) / log2(e)
        const float lse = (m + log2f(l)) / kLog2e;
        float M = lse;
        const int32_t* ir = idxg + (size_t)i * K;
        const float* sr = sselg + ((size_t)hh * N + i) * K;
        const int kk = row_ok ? K : 0;
        for (int s = 0; s < kk; ++s) {
          const int c = ir[s];
          if (c >= 0 && c < i / kChunk) M = fmaxf(M, sr[s]);
        }
        float Z = expf(lse - M);
        for (int s = 0; s < kk; ++s) {
          const int c = ir[s];
          if (c >= 0 && c < i / kChunk) Z += expf(sr[s] - M);
        }
        if (row_ok) {
          s_rowm[r] = M;
          s_rowz[r] = 1.0f / Z;
        }
        // own term: exp(LSE_own - M)/Z' * (sum_j p_j v_j)/l = exp(m_nat - M)/Z' * sum_j p_j v_j
        const float w = expf(m / kLog2e - M) / Z;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tc::tmem_ld32(tO + lane_off + c0, o);
          tc::tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *o_row_f4(sm, L.o, r, (c0 + j) >> 2, D) =
                  make_float4(o[j] * w, o[j + 1] * w, o[j + 2] * w, o[j + 3] * w);
          }
        }
      }
      tc::fence_before_sync();
      __syncthreads();
      phase ^= 1u;
    }
  }

  // ---------------- selected chunks ----------------
  for (int c = 0; c < n_cand && !failed; ++c) {
    const int base = s_off[c], cnt = s_off[c + 1] - base;
    if (cnt == 0) continue;
    load_kv(c, kChunk);
    const int total = cnt * G;
    for (int t0 = 0; t0 < total; t0 += 128) {
      const int n_rows = min(128, total - t0);
      if (tid < n_rows) {
        const int x = t0 + tid;
        const uint32_t e = s_list[base + x / G];
        const int qo = (int)(e & 511u), s = (int)(e >> 9);
        s_tile[tid] = (uint32_t)(qo * G + x % G) | ((uint32_t)s << 16);
      }
      __syncthreads();
      gather_q(n_rows);
      tc::cp_async_wait_all();
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) issue_s();
      wait_bar(barS);
      if (__syncthreads_or(failed)) { failed = true; break; }
      tc::fence_after_sync();
      int r = 0;
      const bool row_ok = tid < n_rows;
      const bool warp_ok = warp * 32 < n_rows;
      if (warp_ok) {
        float alpha = 0.f;
        if (row_ok) {
          const uint32_t e = s_tile[tid];
          r = (int)(e & 0xffffu);
          const int s = (int)(e >> 16), qo = r / G, hh = r % G;
          const float sh = sselg[((size_t)hh * N + q0 + qo) * K + s];
          alpha = expf(sh - s_rowm[r]) * s_rowz[r];
        }
        float m, l;
        softmax_row(tid, row_ok, 63, alpha, true, m, l);
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) issue_pv();
      wait_bar(barO);
      if (__syncthreads_or(failed)) { failed = true; break; }
      tc::fence_after_sync();
      if (warp_ok) {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tc::tmem_ld32(tO + lane_off + c0, o);
          tc::tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4* p = o_row_f4(sm, L.o, r, (c0 + j) >> 2, D);
              float4 v = *p;
              v.x += o[j]; v.y += o[j + 1]; v.z += o[j + 2]; v.w += o[j + 3];
              *p = v;
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncthreads();
      phase ^= 1u;
    }
  }

  // ---------------- write the block's rows ----------------
  if (!failed) {
    for (int x = tid; x < nq * G * (D / 4); x += kThreads) {
      const int r = x / (D / 4), j4 = x % (D / 4);
      const int qo = r / G, hh = r % G;
      const float4 v = *o_row_f4(sm, L.o, r, j4, D);
      uint2 pk;
      pk.x = tc::pack_bf16x2(v.x, v.y);
      pk.y = tc::pack_bf16x2(v.z, v.w);
      *reinterpret_cast<uint2*>(a.out + (((size_t)bi * a.h + head0 + hh) * N + q0 + qo) * D + j4 * 4) = pk;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// Queries per CTA for a shape, or 0 when the shared-memory plan does not fit.
static int pick_qb(int D, int G, int K, int N, size_t* smem_out) {
  const int rows_target = D == 64 ? 512 : 256;
  int qb = rows_target / G;
  const int n_cand_max = N / kChunk;
  while (qb >= 16) {
    const TcSmem L = tc_layout(D, G, qb, K, n_cand_max);
    const size_t need = (size_t)L.total + 1024;
    if (need <= 227 * 1024 - 512) {  // leave room for the static shared variables
      *smem_out = need;
      return qb;
    }
    qb >>= 1;
  }
  return 0;
}

bool attend_tc_supported(int d, int G, int K, int N) {
  size_t smem;
  return (d == 64 || d == 128) && K <= 64 && pick_qb(d, G, K, N, &smem) > 0;
}

template <int D, int G>
static cudaError_t launch_tc(TcAttendArgs a, cudaStream_t st) {
  size_t smem = 0;
  const int qb = pick_qb(D, G, a.top_k, a.n, &smem);
  if (qb == 0) return cudaErrorInvalidConfiguration;
  a.qb = qb;
  a.n_cand_max = a.n / kChunk;
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
  return d == 64 ? tc_by_group<64>(a, st) : tc_by_group<128>(a, st);
}

}  // namespace hils
