// Host-side launch interface of the HiLS kernels (one struct per kernel family).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include <cuda_bf16.h>

namespace hils {

struct SummarizeArgs {
  const void* k;          // [b,g,N,d] or pages [P,g,B,d]
  const void* lm;         // [b,h,C,d] or pages [P,h,d]
  void* kbar;             // [b,h,C,d] or [P,h,d]: fp32, or bf16 when kbar_bf16 (paged only)
  float* hbias;           // [b,h,C]   or [P,h]
  int b, h, g, n, d, n_chunks;
  float scale;
  bool bf16;
  const int32_t* page_ids;  // nullptr: contiguous mode
  bool kbar_bf16;
  int n_listed, n_pages;
};
cudaError_t run_summarize(const SummarizeArgs& a, cudaStream_t st);

struct SelectArgs {
  const void* q;          // [b,h,N,d]
  const float* kbar;      // [b,h,C,d]
  const float* hbias;     // [b,h,C]
  int32_t* idx;           // [b,g,N,K]
  float* score;           // [b,h,N,K] or nullptr
  unsigned* err;          // sticky error word or nullptr
  int b, h, g, n, d, n_chunks, top_k;
  int n_local;            // chunks in the local branch (1: own chunk; W / B for a window)
  float scale;
  bool bf16;
  uint32_t poll;          // polls of a bounded wait before it gives up (tensor-core kernel)
};
cudaError_t run_select_simt(const SelectArgs& a, cudaStream_t st);
// Tensor-core scores + group Top-K for G = 2, 4, 8 query heads per KV head (bf16, K <= 32):
// the summaries are split into bf16 hi + lo copies (kbar_hi / kbar_lo, workspace) first.
struct alignas(64) GtcArgs {
  CUtensorMap tmap_q;          // Q as [b*h][N][d], 64 x 128 boxes (set by the launcher)
  CUtensorMap tmap_hi;         // kbar_hi as [b*h][C][d], 64 x 64 boxes
  CUtensorMap tmap_lo;
  const __nv_bfloat16* q;      // [b,h,N,d]
  const float* kbar;           // [b,h,C,d]
  __nv_bfloat16* kbar_hi;      // [b,h,C,d] workspace
  __nv_bfloat16* kbar_lo;
  const float* hbias;          // [b,h,C]
  int32_t* idx;                // [b,g,N,K]
  float* score;                // [b,h,N,K] or nullptr
  unsigned* err;
  int b, h, g, n, d, n_chunks, top_k, n_local;
  float scale;
  uint32_t poll;
};
bool select_gtc_supported(int d, int G, int K, bool bf16);
size_t gtc_split_bytes(int b, int h, int n_chunks, int d);  // bytes of one of kbar_hi / kbar_lo
cudaError_t run_select_gtc(GtcArgs a, cudaStream_t st);
// Tensor-core scores + Top-K (bf16, one query head per KV head).
bool select_tc_supported(int d, int G, int K, bool bf16);
cudaError_t run_select_tc(const SelectArgs& a, cudaStream_t st);

// Paged decode: split scan + Top-K (last CTA merges), then per-chunk attention
// with a last-CTA fusion, chained by programmatic dependent launch.
struct DecodeArgs {
  const void* q;               // [b,h,d]
  const void* k_pages;         // [P,g,B,d]
  const void* v_pages;
  const void* kbar_pages;      // [P,h,d] fp32, or bf16 when kbar_bf16
  const float* hbias_pages;    // [P,h]
  const int32_t* block_table;  // [b,max_chunks]
  const int32_t* seq_lens;     // [b]
  void* out;                   // [b,h,d]
  int32_t* idx;                // [b,g,K]
  int32_t* sel_page;           // [b,g,K] reserved (the attention kernel looks pages up itself)
  float* ssel;                 // [b,h,K]
  unsigned long long* part_keys;  // [b,g,nsplit,K] per-range Top-K lists
  float* part_att;             // [b,g,2(K+n_local),G,d+2]: per half chunk (max, sum, unnormalised output)
  unsigned* scan_ticket;       // [b,g] reserved (the scan takes no ticket)
  unsigned* att_ticket;        // [b,g]
  unsigned* err;
  bool kbar_bf16;              // compact summary cache (bf16 models only)
  int b, h, g, d, top_k, max_chunks, n_pages;
  int n_local;                 // local-branch chunks (1: own chunk; W / B for a window), <= 16
  int nsplit, range, att_ctas; // set by the launcher: scan ranges per sequence, chunks per range
  float scale;
  bool bf16;
};
int decode_splits(int batch, int max_chunks);
bool decode_supported(int h, int d);  // the scan holds a page's summaries of all heads: h * d <= 8192
// whether the Top-K merge of the scan's range lists fits the attention kernel's shared memory
bool decode_merge_supported(int batch, int max_chunks, int top_k);
cudaError_t run_decode(DecodeArgs a, cudaStream_t st);

// Row-wise attention + fusion (one warp per query and KV group).
struct AttendRowsArgs {
  const void* q;               // prefill [b,h,N,d]; decode [b,h,d]
  const void* k;               // prefill [b,g,N,d]; decode pages [P,g,B,d]
  const void* v;
  const int32_t* idx;          // prefill [b,g,N,K]; decode [b,g,K]
  const float* ssel;           // prefill [b,h,N,K]; decode [b,h,K]
  void* out;                   // like q
  float* lse;                  // prefill [b,h,N] log Zhat, or nullptr
  const int32_t* block_table;  // decode only
  const int32_t* seq_lens;     // decode only
  unsigned* err;
  int b, h, g, n, d, top_k, max_chunks, n_pages;
  int n_local;                 // chunks in the local branch (1: own chunk)
  float scale;
  bool bf16;
  bool paged;                  // decode mode
};
cudaError_t run_attend_rows(const AttendRowsArgs& a, cudaStream_t st);

// Tensor-core prefill attention + fusion for a given selection (bf16 only).
struct alignas(64) TcAttendArgs {
  CUtensorMap tmap_k;          // K as [b*g][N][d], 64x64 boxes, 128B swizzle (set by the launcher)
  CUtensorMap tmap_v;          // V, likewise
  const __nv_bfloat16* q;      // [b,h,N,d]
  const __nv_bfloat16* k;      // [b,g,N,d]
  const __nv_bfloat16* v;
  const int32_t* idx;          // [b,g,N,K]
  const float* ssel;           // [b,h,N,K]
  __nv_bfloat16* out;          // [b,h,N,d]
  float* lse;                  // [b,h,N] log Zhat, or nullptr
  unsigned* err;
  int b, h, g, n, top_k;
  float scale;
  int qb;                      // queries per CTA (set by the launcher)
  int n_cand_max;              // N / chunk (set by the launcher)
  uint32_t poll;               // polls of a bounded wait before it gives up
};
// Backward pass (bf16 inputs, fp32 gradients) for a forward's selection and row normaliser.
struct BwdArgs {
  const void* q;          // [b,h,N,d] bf16
  const void* k;          // [b,g,N,d]
  const void* v;
  const void* landmark;   // [b,h,C,d]
  const void* out;        // [b,h,N,d] forward output
  const void* dout;       // [b,h,N,d] upstream gradient
  const float* lse;       // [b,h,N] log Zhat of the forward
  const int32_t* idx;     // [b,g,N,K]
  const float* ssel;      // [b,h,N,K] shat of the selected chunks
  float* dq;              // [b,h,N,d] (accumulated: cleared by the launcher)
  float* dk;              // [b,g,N,d]
  float* dv;
  float* dlandmark;       // [b,h,C,d]
  float* drow;            // workspace [b,h,N]: dO . o
  int* list_off;          // workspace [b,g,C+1]
  int* list;              // workspace [b,g,N*K]
  unsigned* err;
  int b, h, g, n, d, top_k, n_local;
  float scale;
};
cudaError_t run_backward(const BwdArgs& a, cudaStream_t st);

// Chunk-major prefill attention (bf16, d = 64 or 128, G in {1, 2, 4, 8}): every
// (query, selected chunk) pair of the whole sequence is bucketed by chunk into full
// 128-row tiles; each tile's normalised chunk output is stored as a bf16 partial and
// a fusion pass combines a row's partials with the inter-chunk softmax.
struct alignas(64) CmArgs {
  CUtensorMap tmap_k;          // K as [b*g][N][d], 64x64 boxes, 128B swizzle
  CUtensorMap tmap_v;          // V, likewise
  const __nv_bfloat16* q;      // [b,h,N,d]
  const __nv_bfloat16* k;      // [b,g,N,d]
  const __nv_bfloat16* v;
  const int32_t* idx;          // [b,g,N,K]
  const float* ssel;           // [b,h,N,K]
  __nv_bfloat16* out;          // [b,h,N,d]
  float* lse;                  // [b,h,N] log Zhat, or nullptr
  unsigned* err;
  // workspace (see cm_scratch_bytes)
  int* cnt;                    // [b*g*c_sel] selections per (sequence, KV head, chunk)
  int* cur;                    // [b*g*c_sel] scatter cursors
  int* toff;                   // [b*g*c_sel + 1] first selected tile of each bucket
  int* n_sel;                  // number of selected tiles
  int* abort_flag;             // set when the tile kernel gave up (the fusion then writes nothing)
  int4* desc;                  // per selected tile: (b*g + KV head, chunk, first entry, rows)
  int* ent_q;                  // per selected tile: 128 / G entries, the Q row (of [b*h*N]) of the group's first head, -1 padding
  int* pos;                    // [b,g,N,K] partial row of each selection (head 0 of the group), -1 if none
  __nv_bfloat16* part;         // [tiles][128][d] normalised chunk outputs
  float* plse;                 // [local tiles][128] log-mass of each local-branch chunk
  int b, h, g, n, d, top_k, n_local;
  int c_sel;                   // N / B: complete chunks (selectable)
  int c_all;                   // ceil(N / B): chunks with a local bucket
  int tl;                      // tiles per local bucket
  int n_lt;                    // local tiles = b * g * c_all * tl
  int max_sel;                 // capacity of the selected-tile arrays
  float scale;
  uint32_t poll;               // polls of a bounded wait before it gives up
};
bool cm_shape_supported(int d, int G, int K, int N, int n_local);
bool cm_kernel_ready(int d, int G);  // compiled to the register budget its warp roles assume
// Bytes of scratch the chunk-major path needs, and its offsets from a 256-byte aligned base.
struct CmScratch {
  size_t cnt, cur, toff, n_sel, abort_flag, desc, ent_q, pos, part, plse, total;
  int c_sel, c_all, tl, n_lt, max_sel;
};
CmScratch cm_scratch(int b, int h, int g, int n, int d, int K, int n_local);
cudaError_t run_attend_cm(CmArgs a, cudaStream_t st);
bool encode_kv_tensor_map(CUtensorMap* m, const void* base, int D, int N, int bg);

bool attend_tc_supported(int d, int G, int K, int N);
cudaError_t run_attend_tc(const TcAttendArgs& a, int d, cudaStream_t st);
// Head dim 64: Q rows in tensor memory, conflict-free accumulation order (tensor maps set).
bool attend_tc3_supported(int d, int G, int K, int N);
cudaError_t run_attend_tc3(const TcAttendArgs& a, cudaStream_t st);

}  // namespace hils
