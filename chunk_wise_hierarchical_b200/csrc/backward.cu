// Backward pass of HiLS-Attention: gradients of the prefill forward with
// respect to Q, K, V and the landmark queries, the Top-K selection held fixed
// (HiLS notes, section 5.3: the hierarchical softmax lets the loss reach the
// selector; Tide digest, Figure 3 caption: gradients reach the compressed
// key).
//
// Per query row i (head h) with fusion weights w (local branch l, selected
// chunks c), output o, row normaliser lse = log Zhat and D = dO . o:
//   local branch:     P_ij = exp(s_ij - lse),            ds_ij = P_ij (u_ij - D)
//   selected chunk c: p_ij = exp(s_ij - LSE_c) (intra-chunk softmax),
//                     w_c  = exp(shat_c - lse),  P_ij = w_c p_ij,
//                     delta_c = sum_j p_ij u_ij, ds_ij = P_ij (u_ij - delta_c),
//                     dshat_c = w_c (delta_c - D)
// with s_ij = scale q_i . k_j and u_ij = dO_i . v_j; then
//   dV_j += P_ij dO_i,  dK_j += scale ds_ij q_i,  dQ_i += scale ds_ij k_j,
//   dQ_i += scale dshat_c kbar_c,  dkbar_c += scale dshat_c q_i,  dH_c += dshat_c,
// and the chain through the landmark summary (notes section 5.1:
// pi = softmax(scale l_c . k_j), kbar = sum pi_j k_j, H = -sum pi_j log pi_j):
//   dpi_j = dkbar . k_j - dH (log pi_j + 1),  dsigma_j = pi_j (dpi_j - sum_m pi_m dpi_m),
//   dK_j += pi_j dkbar + scale dsigma_j l_c,  dL_c = scale sum_j dsigma_j k_j.
//
// Three kernels:
//   bwd_lists_kernel   per (sequence, KV head): inverts the selection into
//                      per-chunk lists of the (row, slot) pairs that chose the chunk
//   bwd_rowdot_kernel  D = dO . o per row, and dQ cleared (it is accumulated)
//   bwd_chunk_kernel   per (sequence, KV head, chunk): K_c and V_c stay in shared
//                      memory while the CTA walks every row that reads the chunk
//                      (the rows that selected it, and the rows whose local branch
//                      covers it), 16 (row, head) units at a time.  S = Q K_c^T and
//                      U = dO V_c^T, then dV_c += P^T dO, dK_c += dS^T Q and
//                      dQ_rows = dS K_c run on the tensor cores (bf16 x bf16 -> fp32
//                      warp MMA tiles of 16x16x16); the softmax algebra runs in
//                      fp32.  dK_c, dV_c and dL_c are written once by their CTA; dQ
//                      rows collect their chunks' terms with fp32 vector atomics.
#include <mma.h>

#include "common.cuh"
#include "kernels.cuh"

namespace hils {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kUnits = 16;  // (row, head) units per tensor-core step

// ---------------------------------------------------------------------------
// Inverse selection lists: entries (row << 6) | slot of chunk c at
// list[off[c] .. off[c + 1]) of this (sequence, KV head); off has C + 1 entries.
__global__ void __launch_bounds__(1024) bwd_lists_kernel(BwdArgs a) {
  extern __shared__ int s_cnt[];  // [C + 1] counts, then cursors
  const int bg = blockIdx.x;
  const int C = a.n / kChunk, K = a.top_k, N = a.n;
  int* cur = s_cnt + (C + 1);
  const int32_t* idx = a.idx + (size_t)bg * N * K;
  int* off = a.list_off + (size_t)bg * (C + 1);
  int* list = a.list + (size_t)bg * N * K;
  for (int c = threadIdx.x; c <= C; c += blockDim.x) s_cnt[c] = 0;
  __syncthreads();
  const long long total = (long long)N * K;
  for (long long e = threadIdx.x; e < total; e += blockDim.x) {
    const int c = idx[e];
    const int i = (int)(e / K);
    if (c >= 0 && c < n_candidates(i, a.n_local, C)) atomicAdd(&s_cnt[c], 1);
    else if (c >= 0) set_error(a.err, kErrBadPage);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // C <= 32767: a serial scan is a few microseconds
    int run = 0;
    for (int c = 0; c < C; ++c) {
      const int x = s_cnt[c];
      s_cnt[c] = run;
      cur[c] = run;
      run += x;
    }
    s_cnt[C] = run;
  }
  __syncthreads();
  for (int c = threadIdx.x; c <= C; c += blockDim.x) off[c] = s_cnt[c];
  for (long long e = threadIdx.x; e < total; e += blockDim.x) {
    const int c = idx[e];
    const int i = (int)(e / K);
    if (c >= 0 && c < n_candidates(i, a.n_local, C)) {
      const int pos = atomicAdd(&cur[c], 1);
      list[pos] = (i << 6) | (int)(e % K);
    }
  }
}

// D = dO . o per (sequence, head, row), one warp per row; dQ rows cleared.
template <int D>
__global__ void __launch_bounds__(256) bwd_rowdot_kernel(BwdArgs a) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)a.b * a.h * a.n;
  if (row >= rows) return;
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(a.out) + row * D;
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(a.dout) + row * D;
  float s = 0.f;
#pragma unroll
  for (int e = lane; e < D; e += 32) s += __bfloat162float(o[e]) * __bfloat162float(g[e]);
  s = warp_sum(s);
  if (lane == 0) a.drow[row] = s;
#pragma unroll
  for (int e = lane; e < D; e += 32) a.dq[row * D + e] = 0.f;
}

template <int D>
struct BwdSmem {
  static constexpr int LDK = D + 8;   // bf16 row pitch of K, V, Q, dO tiles
  static constexpr int LDS = 64 + 4;  // fp32 pitch of S, U
  static constexpr int LDP = 64 + 8;  // bf16 pitch of P, dS
  static constexpr int LDQ = D + 4;   // fp32 pitch of the dQ tile
  static constexpr size_t kK = 0;
  static constexpr size_t kV = kK + 64 * LDK * 2;
  static constexpr size_t kQ = kV + 64 * LDK * 2;
  static constexpr size_t kdO = kQ + kUnits * LDK * 2;
  static constexpr size_t kS = kdO + kUnits * LDK * 2;
  static constexpr size_t kU = kS + kUnits * LDS * 4;
  static constexpr size_t kP = kU + kUnits * LDS * 4;
  static constexpr size_t kdS = kP + kUnits * LDP * 2;
  static constexpr size_t kdQ = kdS + kUnits * LDP * 2;
  static constexpr size_t kEnd = kdQ + kUnits * LDQ * 4;
  // the final dK / dV staging (64 x D fp32 each) reuses the space from kQ on
  static constexpr size_t kStageK = kQ;
  static constexpr size_t kStageV = kQ + 64 * (D + 4) * 4;
  static constexpr size_t kTotal = (kStageV + 64 * (D + 4) * 4 > kEnd) ? kStageV + 64 * (D + 4) * 4 : kEnd;
};

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kBwdThreads) bwd_chunk_kernel(BwdArgs a) {
  using namespace nvcuda;
  using SM = BwdSmem<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem + SM::kK);
  __nv_bfloat16* Vs = reinterpret_cast<__nv_bfloat16*>(smem + SM::kV);
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem + SM::kQ);
  __nv_bfloat16* dOs = reinterpret_cast<__nv_bfloat16*>(smem + SM::kdO);
  float* Ss = reinterpret_cast<float*>(smem + SM::kS);
  float* Us = reinterpret_cast<float*>(smem + SM::kU);
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(smem + SM::kP);
  __nv_bfloat16* dSs = reinterpret_cast<__nv_bfloat16*>(smem + SM::kdS);
  float* dQs = reinterpret_cast<float*>(smem + SM::kdQ);
  __shared__ float kbarS[G][D], dkbarS[G][D], lmS[G][D];
  __shared__ float piS[G][64], dhS[G], dsigS[G][64];
  __shared__ int u_row[kUnits], u_head[kUnits], u_jmax[kUnits];
  __shared__ float u_lse[kUnits], u_D[kUnits], u_w[kUnits], u_dsh[kUnits];
  __shared__ int s_nsel;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.n, K = a.top_k;
  const int C = N / kChunk, CA = (N + kChunk - 1) / kChunk;
  const int c = blockIdx.x % CA;
  const int gi = (blockIdx.x / CA) % a.g;
  const int bi = blockIdx.x / (CA * a.g);
  const int h0 = gi * G;
  const bool complete = c < C;
  const float sc = a.scale;
  const int c_rows = min(kChunk, N - c * kChunk);  // keys of this chunk

  // ---- K_c, V_c (rows past N zero), landmark rows of the group's heads
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k) + (((size_t)bi * a.g + gi) * N + (size_t)c * kChunk) * D;
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v) + (((size_t)bi * a.g + gi) * N + (size_t)c * kChunk) * D;
  for (int x = tid; x < 64 * D / 8; x += kBwdThreads) {
    const int r = x / (D / 8), e = (x % (D / 8)) * 8;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (r < c_rows) {
      kv = *reinterpret_cast<const uint4*>(kg + (size_t)r * D + e);
      vv = *reinterpret_cast<const uint4*>(vg + (size_t)r * D + e);
    }
    *reinterpret_cast<uint4*>(Ks + r * SM::LDK + e) = kv;
    *reinterpret_cast<uint4*>(Vs + r * SM::LDK + e) = vv;
  }
  for (int x = tid; x < G * D; x += kBwdThreads) {
    const int hh = x / D, e = x % D;
    lmS[hh][e] = complete ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.landmark)[(((size_t)bi * a.h + h0 + hh) * C + c) * D + e]) : 0.f;
    dkbarS[hh][e] = 0.f;
    kbarS[hh][e] = 0.f;  // stays zero for the trailing partial chunk (no summary)
  }
  if (tid < G) dhS[tid] = 0.f;
  if (tid == 0) s_nsel = complete ? a.list_off[((size_t)bi * a.g + gi) * (C + 1) + c + 1] - a.list_off[((size_t)bi * a.g + gi) * (C + 1) + c] : 0;
  __syncthreads();
  // ---- the chunk's summaries per head: pi = softmax(scale l . k_j) and kbar (complete chunks)
  if (complete) {
    for (int hh = warp; hh < G; hh += kBwdThreads / 32) {
      float s2[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = lane + 32 * u;
        float acc = 0.f;
        for (int e = 0; e < D; ++e) acc = fmaf(lmS[hh][e], __bfloat162float(Ks[j * SM::LDK + e]), acc);
        s2[u] = acc * sc;
      }
      const float m = warp_max(fmaxf(s2[0], s2[1]));
      const float e0 = expf(s2[0] - m), e1 = expf(s2[1] - m);
      const float z = warp_sum(e0 + e1);
      piS[hh][lane] = e0 / z;
      piS[hh][lane + 32] = e1 / z;
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += kBwdThreads) {
      const int hh = x / D, e = x % D;
      float acc = 0.f;
      for (int j = 0; j < 64; ++j) acc = fmaf(piS[hh][j], __bfloat162float(Ks[j * SM::LDK + e]), acc);
      kbarS[hh][e] = acc;
    }
  }

  // ---- work units: (row, head) pairs reading this chunk
  //   [0, nsel * G): selected entries of the inverse list, G heads each
  //   then the local rows: rows whose local branch (chunks own+1-n_local .. own) covers c
  const int nsel = s_nsel;
  const int loc_lo = c * kChunk;                                         // first local row
  const int loc_hi = min(N, (c + a.n_local) * kChunk);                   // one past the last
  const int n_loc = loc_hi - loc_lo;
  const int n_units = (nsel + n_loc) * G;
  const int* list = a.list + ((size_t)bi * a.g + gi) * (size_t)N * K;
  const int list0 = complete ? a.list_off[((size_t)bi * a.g + gi) * (C + 1) + c] : 0;

  // dV / dK accumulators: warp w owns (matrix, 16-column tile) pairs w and w + 8
  constexpr int NT = D / 16;           // column tiles per matrix
  constexpr int PAIRS = 2 * NT;        // dV tiles then dK tiles
  constexpr int PPW = (PAIRS + 7) / 8; // pairs per warp
  wmma::fragment<wmma::accumulator, 16, 16, 16, float> acc[PPW][4];
#pragma unroll
  for (int p = 0; p < PPW; ++p)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) wmma::fill_fragment(acc[p][mt], 0.f);

  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* dog = static_cast<const __nv_bfloat16*>(a.dout);
  __syncthreads();
  for (int u0 = 0; u0 < n_units; u0 += kUnits) {
    // (a) unit metadata
    if (tid < kUnits) {
      const int uu = u0 + tid;
      int row = -1, hh = 0, jmax = 63;
      float lse = 0.f, Dv = 0.f, w = -1.f;  // w < 0: local branch
      if (uu < n_units) {
        const int e = uu / G;
        hh = uu % G;
        const size_t hq = (size_t)bi * a.h + h0 + hh;
        if (e < nsel) {
          const int ent = list[list0 + e];
          row = ent >> 6;
          const int slot = ent & 63;
          lse = a.lse[hq * N + row];
          w = expf(a.ssel[(hq * N + row) * K + slot] - lse);
        } else {
          row = loc_lo + (e - nsel);
          lse = a.lse[hq * N + row];
          jmax = row / kChunk == c ? row - c * kChunk : 63;  // causal inside the own chunk
        }
        Dv = a.drow[hq * N + row];
      }
      u_row[tid] = row;
      u_head[tid] = hh;
      u_jmax[tid] = jmax;
      u_lse[tid] = lse;
      u_D[tid] = Dv;
      u_w[tid] = w;
    }
    __syncthreads();
    // (b) gather the units' q and dO rows
    for (int x = tid; x < kUnits * D / 8; x += kBwdThreads) {
      const int r = x / (D / 8), e = (x % (D / 8)) * 8;
      const int row = u_row[r];
      uint4 qv = make_uint4(0, 0, 0, 0), gv = make_uint4(0, 0, 0, 0);
      if (row >= 0) {
        const size_t off = (((size_t)bi * a.h + h0 + u_head[r]) * N + row) * D + e;
        qv = *reinterpret_cast<const uint4*>(qg + off);
        gv = *reinterpret_cast<const uint4*>(dog + off);
      }
      *reinterpret_cast<uint4*>(Qs + r * SM::LDK + e) = qv;
      *reinterpret_cast<uint4*>(dOs + r * SM::LDK + e) = gv;
    }
    __syncthreads();
    // (c) S = Q K^T (warps 0-3, key tile = warp) and U = dO V^T (warps 4-7)
    {
      const int nt = warp & 3;
      const __nv_bfloat16* A = warp < 4 ? Qs : dOs;
      const __nv_bfloat16* B = warp < 4 ? Ks : Vs;
      wmma::fragment<wmma::accumulator, 16, 16, 16, float> f;
      wmma::fill_fragment(f, 0.f);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        wmma::fragment<wmma::matrix_a, 16, 16, 16, __nv_bfloat16, wmma::row_major> fa;
        wmma::fragment<wmma::matrix_b, 16, 16, 16, __nv_bfloat16, wmma::col_major> fb;
        wmma::load_matrix_sync(fa, A + kk * 16, SM::LDK);
        // B[k][n] = K[key n][dim k]: column-major view of the row-major key tile
        wmma::load_matrix_sync(fb, B + (nt * 16) * SM::LDK + kk * 16, SM::LDK);
        wmma::mma_sync(f, fa, fb, f);
      }
      wmma::store_matrix_sync((warp < 4 ? Ss : Us) + nt * 16, f, SM::LDS, wmma::mem_row_major);
    }
    __syncthreads();
    // (d) softmax algebra in fp32: two units per warp, lanes own keys lane and lane + 32
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp * 2 + rr;
      const bool valid = u_row[r] >= 0;
      const float w = u_w[r], lse = u_lse[r], Dv = u_D[r];
      const int jmax = u_jmax[r];
      float P[2], dS[2];
      float s[2], uu[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int j = lane + 32 * q;
        s[q] = Ss[r * SM::LDS + j] * sc;
        uu[q] = Us[r * SM::LDS + j];
      }
      float dsh = 0.f;
      if (w >= 0.f) {  // selected chunk: intra-chunk softmax, weight w
        const float m = warp_max(fmaxf(s[0], s[1]));
        const float e0 = expf(s[0] - m), e1 = expf(s[1] - m);
        const float inv = 1.0f / warp_sum(e0 + e1);
        const float p0 = e0 * inv, p1 = e1 * inv;
        const float delta = warp_sum(p0 * uu[0] + p1 * uu[1]);
        P[0] = w * p0;
        P[1] = w * p1;
        dS[0] = P[0] * (uu[0] - delta);
        dS[1] = P[1] * (uu[1] - delta);
        dsh = w * (delta - Dv);
      } else {  // local branch: the final weights directly, causal in the own chunk
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = lane + 32 * q;
          P[q] = j <= jmax && j < c_rows ? expf(s[q] - lse) : 0.f;
          dS[q] = P[q] * (uu[q] - Dv);
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int j = lane + 32 * q;
        Ps[r * SM::LDP + j] = __float2bfloat16_rn(valid ? P[q] : 0.f);
        dSs[r * SM::LDP + j] = __float2bfloat16_rn(valid ? dS[q] * sc : 0.f);
      }
      if (lane == 0) u_dsh[r] = valid ? dsh : 0.f;
    }
    __syncthreads();
    // (e) dV[:, tile] += P^T dO[:, tile]; dK[:, tile] += dS^T Q[:, tile]
#pragma unroll
    for (int p = 0; p < PPW; ++p) {
      const int pair = warp + 8 * p;
      if (pair < PAIRS) {
        const bool is_v = pair < NT;
        const int nt = is_v ? pair : pair - NT;
        const __nv_bfloat16* At = is_v ? Ps : dSs;   // [unit][key]: read as [key][unit] (column-major)
        const __nv_bfloat16* Bt = is_v ? dOs : Qs;   // [unit][dim]
        wmma::fragment<wmma::matrix_b, 16, 16, 16, __nv_bfloat16, wmma::row_major> fb;
        wmma::load_matrix_sync(fb, Bt + nt * 16, SM::LDK);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          wmma::fragment<wmma::matrix_a, 16, 16, 16, __nv_bfloat16, wmma::col_major> fa;
          wmma::load_matrix_sync(fa, At + mt * 16, SM::LDP);
          wmma::mma_sync(acc[p][mt], fa, fb, acc[p][mt]);
        }
      }
    }
    // (f) dQ tile = dS K (scale already in dS)
    if (warp < NT) {
      wmma::fragment<wmma::accumulator, 16, 16, 16, float> f;
      wmma::fill_fragment(f, 0.f);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        wmma::fragment<wmma::matrix_a, 16, 16, 16, __nv_bfloat16, wmma::row_major> fa;
        wmma::fragment<wmma::matrix_b, 16, 16, 16, __nv_bfloat16, wmma::row_major> fb;
        wmma::load_matrix_sync(fa, dSs + kk * 16, SM::LDP);
        wmma::load_matrix_sync(fb, Ks + (kk * 16) * SM::LDK + warp * 16, SM::LDK);
        wmma::mma_sync(f, fa, fb, f);
      }
      wmma::store_matrix_sync(dQs + warp * 16, f, SM::LDQ, wmma::mem_row_major);
    }
    __syncthreads();
    // (g) dQ rows += dQ tile + scale dshat kbar (fp32 vector atomics); dkbar, dH
    for (int x = tid; x < kUnits * D / 4; x += kBwdThreads) {
      const int r = x / (D / 4), e = (x % (D / 4)) * 4;
      const int row = u_row[r];
      if (row < 0) continue;
      const int hh = u_head[r];
      const float dsh = u_dsh[r] * sc;
      float4 v;
      v.x = dQs[r * SM::LDQ + e] + dsh * kbarS[hh][e];
      v.y = dQs[r * SM::LDQ + e + 1] + dsh * kbarS[hh][e + 1];
      v.z = dQs[r * SM::LDQ + e + 2] + dsh * kbarS[hh][e + 2];
      v.w = dQs[r * SM::LDQ + e + 3] + dsh * kbarS[hh][e + 3];
      atomicAdd(reinterpret_cast<float4*>(a.dq + (((size_t)bi * a.h + h0 + hh) * N + row) * D + e), v);
    }
    for (int x = tid; x < G * D; x += kBwdThreads) {
      const int hh = x / D, e = x % D;
      float acc1 = 0.f;
#pragma unroll 4
      for (int r = 0; r < kUnits; ++r)
        if (u_row[r] >= 0 && u_head[r] == hh) acc1 = fmaf(u_dsh[r], __bfloat162float(Qs[r * SM::LDK + e]), acc1);
      dkbarS[hh][e] += acc1 * sc;
    }
    if (tid < G) {
      float acc1 = 0.f;
      for (int r = 0; r < kUnits; ++r)
        if (u_row[r] >= 0 && u_head[r] == tid) acc1 += u_dsh[r];
      dhS[tid] += acc1;
    }
    __syncthreads();
  }

  // ---- dK, dV staged in fp32, the summary chain added to dK, then written once
  float* dKs = reinterpret_cast<float*>(smem + SM::kStageK);
  float* dVs = reinterpret_cast<float*>(smem + SM::kStageV);
  constexpr int LDF = D + 4;
#pragma unroll
  for (int p = 0; p < PPW; ++p) {
    const int pair = warp + 8 * p;
    if (pair < PAIRS) {
      const bool is_v = pair < NT;
      const int nt = is_v ? pair : pair - NT;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        wmma::store_matrix_sync((is_v ? dVs : dKs) + (mt * 16) * LDF + nt * 16, acc[p][mt], LDF, wmma::mem_row_major);
    }
  }
  __syncthreads();
  if (complete) {
    // dpi_j = dkbar . k_j - dH (log pi_j + 1); dsigma_j = pi_j (dpi_j - sum_m pi_m dpi_m)
    // (log pi_j = sigma_j - LSE(sigma) is finite even where pi_j underflows)
    float* dsig = &dsigS[0][0];  // [G][64]; logits first, then dsigma
    for (int hh = warp; hh < G; hh += kBwdThreads / 32) {
      float dpi[2], pj[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int j = lane + 32 * q;
        float acc1 = 0.f;
        for (int e = 0; e < D; ++e) acc1 = fmaf(dkbarS[hh][e], __bfloat162float(Ks[j * SM::LDK + e]), acc1);
        pj[q] = piS[hh][j];
        float s1 = 0.f;  // the logit sigma_j; log pi_j = sigma_j - LSE(sigma)
        for (int e = 0; e < D; ++e) s1 = fmaf(lmS[hh][e], __bfloat162float(Ks[j * SM::LDK + e]), s1);
        dpi[q] = acc1;
        dsig[hh * 64 + j] = s1 * sc;
      }
      // LSE of the logits
      const float m = warp_max(fmaxf(dsig[hh * 64 + lane], dsig[hh * 64 + lane + 32]));
      const float lse = m + logf(warp_sum(expf(dsig[hh * 64 + lane] - m) + expf(dsig[hh * 64 + lane + 32] - m)));
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int j = lane + 32 * q;
        dpi[q] -= dhS[hh] * ((dsig[hh * 64 + j] - lse) + 1.0f);
      }
      const float mean = warp_sum(pj[0] * dpi[0] + pj[1] * dpi[1]);
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 2; ++q) dsig[hh * 64 + lane + 32 * q] = pj[q] * (dpi[q] - mean);
    }
    __syncthreads();
    for (int x = tid; x < 64 * D; x += kBwdThreads) {
      const int j = x / D, e = x % D;
      float add = 0.f;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) add += piS[hh][j] * dkbarS[hh][e] + sc * dsig[hh * 64 + j] * lmS[hh][e];
      dKs[j * LDF + e] += add;
    }
    // dL = scale sum_j dsigma_j k_j
    for (int x = tid; x < G * D; x += kBwdThreads) {
      const int hh = x / D, e = x % D;
      float acc1 = 0.f;
      for (int j = 0; j < 64; ++j) acc1 = fmaf(dsig[hh * 64 + j], __bfloat162float(Ks[j * SM::LDK + e]), acc1);
      a.dlandmark[(((size_t)bi * a.h + h0 + hh) * C + c) * D + e] = acc1 * sc;
    }
  }
  __syncthreads();
  float* dkg = a.dk + (((size_t)bi * a.g + gi) * N + (size_t)c * kChunk) * D;
  float* dvg = a.dv + (((size_t)bi * a.g + gi) * N + (size_t)c * kChunk) * D;
  for (int x = tid; x < c_rows * D / 4; x += kBwdThreads) {
    const int j = x / (D / 4), e = (x % (D / 4)) * 4;
    *reinterpret_cast<float4*>(dkg + (size_t)j * D + e) = *reinterpret_cast<const float4*>(dKs + j * LDF + e);
    *reinterpret_cast<float4*>(dvg + (size_t)j * D + e) = *reinterpret_cast<const float4*>(dVs + j * LDF + e);
  }
}

template <int D, int G>
static cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t st) {
  const size_t smem = BwdSmem<D>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(bwd_chunk_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long ca = (a.n + kChunk - 1) / kChunk;
  bwd_chunk_kernel<D, G><<<(unsigned)(ca * a.g * a.b), kBwdThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t bwd_by_group(const BwdArgs& a, cudaStream_t st) {
  switch (a.h / a.g) {
    case 1: return launch_bwd<D, 1>(a, st);
    case 2: return launch_bwd<D, 2>(a, st);
    case 4: return launch_bwd<D, 4>(a, st);
    case 8: return launch_bwd<D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_backward(const BwdArgs& a, cudaStream_t st) {
  if (a.b * a.g == 0 || a.n == 0) return cudaSuccess;
  const int C = a.n / kChunk;
  // 1. inverse selection lists
  if (a.top_k > 0 && C > 0) {
    const size_t smem = (size_t)(2 * (C + 1)) * 4;
    cudaError_t e = cudaFuncSetAttribute(bwd_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_lists_kernel<<<a.b * a.g, 1024, smem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if (C > 0) {
    cudaError_t e = cudaMemsetAsync(a.list_off, 0, (size_t)a.b * a.g * (C + 1) * 4, st);
    if (e != cudaSuccess) return e;
  }
  // 2. D = dO . o and dQ cleared
  const long long rows = (long long)a.b * a.h * a.n;
  if (a.d == 64)
    bwd_rowdot_kernel<64><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a);
  else
    bwd_rowdot_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. per-chunk gradients
  return a.d == 64 ? bwd_by_group<64>(a, st) : bwd_by_group<128>(a, st);
}

}  // namespace hils
