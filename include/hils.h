/*
 * hils.h -- C ABI of libhils.so: the HiLS-Attention (Hierarchical Landmark
 * Sparse Attention) forward pass on one NVIDIA B200 (sm_100a).
 *
 * The operation is defined on the HiLS pages ("Hierarchical Sparse Attention
 * Done Right: Toward Infinite Context Modeling", reading notes, sections 5.1
 * to 5.4, and the Tide digest of the same paper, Figure 3).  Each entry point
 * below names the passage it implements.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory   All tensor pointers are DEVICE pointers owned by the caller
 *          (allocate them with any allocator, e.g. torch).  The library never
 *          allocates, frees or keeps a pointer after the call returns.
 * Layout   Dense row-major, no padding.  Prefill tensors are BHND:
 *          q [batch, heads_q, seq_len, head_dim], k and v
 *          [batch, heads_kv, seq_len, head_dim], each (batch, head) one
 *          contiguous seq_len x head_dim block.
 * Chunks   chunk = B keys (only 64 is supported).  C = seq_len / B (rounded
 *          down) complete chunks; a trailing partial chunk is never a
 *          candidate, it only serves as the own chunk of its queries.
 * Local    shape.window selects the local branch whose exact mass joins the
 *          fusion (notes section 5.3).  0 or B: the query's own causal
 *          partial chunk, keys [floor(i/B)*B, i]; a multiple W of B: a
 *          chunk-aligned sliding window (notes section 5.2), the own chunk
 *          and the W/B - 1 complete chunks before it.  The remote candidates
 *          of query i are the complete chunks before its local branch,
 *          c < floor(i/B) + 1 - W/B.
 * Dtype    shape.dtype gives the element type of q, k, v, landmark
 *          queries and out: HILS_BF16 or HILS_F32.  Summaries (kbar,
 *          hbias) and scores are always fp32; indices int32.
 * Scale    shape.scale multiplies every logit; 0 selects 1/sqrt(head_dim).
 * Streams  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *          stream).  Calls only enqueue work: they return before the GPU
 *          finishes, and perform no host-device synchronisation (except
 *          hils_device_status).
 * Errors   Arguments are checked on the host before anything is launched;
 *          a failed check returns a status and launches nothing.  A launch
 *          failure returns HILS_ERR_CUDA.  Kernels that read indices supplied
 *          by the caller (page ids, block tables) check them on the device;
 *          an out-of-range entry is skipped and recorded in the workspace's
 *          error word, which hils_device_status() reads.  No entry point
 *          aborts, traps or throws.
 * Threads  Re-entrant; the only global state is per-device kernel attribute
 *          set-up done once under a lock.
 * Limits   head_dim in {64, 128}; chunk == 64; 0 <= top_k <= 64;
 *          heads_q % heads_kv == 0 and heads_q / heads_kv in {1, 2, 4, 8}.
 */
#ifndef HILS_H_
#define HILS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HILS_API __attribute__((visibility("default")))
#else
#define HILS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARG = 1,     /* null pointer, negative or inconsistent size */
  HILS_ERR_UNSUPPORTED = 2,     /* valid but outside the limits above */
  HILS_ERR_WORKSPACE = 3,       /* workspace missing or smaller than required */
  HILS_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  HILS_ERR_DEVICE_CHECK = 5,    /* a kernel met an out-of-range index */
  HILS_ERR_DEVICE_TIMEOUT = 6   /* a bounded device wait gave up */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

/* Operations whose workspace size can be queried. */
typedef enum {
  HILS_OP_SELECT = 0,
  HILS_OP_ATTEND = 1,
  HILS_OP_DECODE = 2,
  HILS_OP_ATTEND_SELECTED = 3,
  HILS_OP_BACKWARD = 4
} hils_op;

typedef struct {
  int32_t batch;     /* sequences */
  int32_t heads_q;   /* query heads h */
  int32_t heads_kv;  /* key/value heads g (GQA group G = h / g) */
  int32_t head_dim;  /* d */
  int32_t seq_len;   /* N (prefill); the largest sequence length (decode) */
  int32_t chunk;     /* B, keys per chunk */
  int32_t top_k;     /* K, remote chunks kept per query */
  float scale;       /* logit scale; 0 => 1/sqrt(d) */
  int32_t dtype;     /* hils_dtype */
  int32_t window;    /* local branch: 0 or chunk = own chunk; W = k*chunk =
                        sliding window of k chunks (see "Local" above) */
} hils_shape;

/* Static English text for a status code; never NULL. */
HILS_API const char* hils_status_string(int status);

/* ABI version, currently 3 (1 had no window field and no lse_out; 2 had no
 * hils_set_wait_limit). */
HILS_API int32_t hils_abi_version(void);

/* Default of hils_set_wait_limit: about a second or more of polling. */
#define HILS_DEFAULT_WAIT_LIMIT (1u << 26)

/*
 * hils_set_wait_limit -- sets how many times an ordinary bounded wait of the
 * tensor-core kernels (select, prefill attention) polls its mbarrier before the
 * kernel gives up.  A kernel that gives up sets the timeout bit of the error
 * word (hils_device_status then returns HILS_ERR_DEVICE_TIMEOUT), stops issuing
 * work, waits for the copies and MMAs it has already issued (those drain waits
 * always use HILS_DEFAULT_WAIT_LIMIT), releases its tensor memory and returns
 * without writing its outputs; a later call on the same context runs normally.
 * The limit is process-wide and read when a call launches its kernels (a CUDA
 * graph keeps the value it was captured with).  0 makes every ordinary wait
 * give up at its first poll: that is how the give-up path is exercised.
 * Returns the previous limit.  Not a pages' operation; no error status.
 */
HILS_API uint32_t hils_set_wait_limit(uint32_t polls);

/* Bytes of device workspace `op` needs for `shape`, written to *bytes.
 * HILS_OP_DECODE reads shape.seq_len as the largest cache length and
 * shape.batch as the number of sequences. */
HILS_API hils_status hils_workspace_size(const hils_shape* shape, int32_t op, size_t* bytes);

/*
 * hils_summarize -- landmark summaries of every complete chunk
 * (notes section 5.1: s_j = l_c.k_j * scale, p = softmax(s),
 *  kbar_c = sum_j p_j k_j, H_c = -sum_j p_j log p_j; section 5.2: the
 *  landmark token's query is l_c).
 *   k           [batch, heads_kv, seq_len, head_dim]      (dtype)
 *   landmark_q  [batch, heads_q, C, head_dim]             (dtype), one
 *               landmark query per (chunk, query head)
 *   kbar        [batch, heads_q, C, head_dim]  fp32, written
 *   hbias       [batch, heads_q, C]            fp32, written
 * Query head h summarises the keys of KV head h / G.
 */
HILS_API hils_status hils_summarize(const hils_shape* shape, const void* k, const void* landmark_q,
                           float* kbar, float* hbias, void* stream);

/*
 * hils_summarize_paged -- the same summaries for pages of a paged chunk
 * cache (one page = one chunk of B tokens).
 *   k_pages         [n_pages, heads_kv, B, head_dim]   (dtype)
 *   landmark_pages  [n_pages, heads_q, head_dim]       (dtype)
 *   page_ids        [n_listed] int32: pages to summarise
 *   kbar_pages      [n_pages, heads_q, head_dim] fp32: rows of the listed
 *                   pages are written, others untouched
 *   hbias_pages     [n_pages, heads_q] fp32, likewise
 * shape.batch and shape.seq_len are ignored.  A page id outside
 * [0, n_pages) is skipped.
 */
HILS_API hils_status hils_summarize_paged(const hils_shape* shape, const void* k_pages,
                                 const void* landmark_pages, const int32_t* page_ids,
                                 int32_t n_listed, int32_t n_pages, float* kbar_pages,
                                 float* hbias_pages, void* stream);

/*
 * hils_select -- chunk scores and Top-K (notes section 5.2:
 *  shat_{i,c} = q_i.kbar_c * scale + H_c, I_i = the K best candidates;
 *  section 5.4: under GQA the selection key is the max over the group's
 *  query heads).  Candidates of query i are the complete chunks before
 *  its local branch, c < n_i = floor(i/B) + 1 - W/B (n_i = floor(i/B) for
 *  the own-chunk branch); K_eff = min(K, max(n_i, 0)).  Ties go to the
 *  lower chunk index.
 *   q           [batch, heads_q, seq_len, head_dim] (dtype)
 *   kbar, hbias as written by hils_summarize
 *   topk_idx    [batch, heads_kv, seq_len, top_k] int32, written in
 *               descending key order; slots >= K_eff hold -1
 *   topk_score  [batch, heads_q, seq_len, top_k] fp32 or NULL: each head's
 *               own shat of the selected chunks (-inf in unused slots)
 *   ws          workspace of hils_workspace_size(HILS_OP_SELECT) bytes,
 *               zero-filled before first use: it holds the sticky error
 *               word read by hils_device_status and, for the grouped
 *               tensor-core path below, the bf16 hi and lo parts of the
 *               summaries (rewritten by every call)
 * kbar must be 16-byte aligned.  For bf16 the scores run on the tensor
 * cores with the fp32 summaries split into two bf16 parts (score error
 * near 2^-17 |q||kbar|) when heads_q == heads_kv, and when heads_q /
 * heads_kv is 2, 4 or 8 with top_k <= 16 (up to 32 where the candidate
 * records fit in shared memory), C >= 64 and seq_len >= 128;
 * other shapes score on the CUDA cores in fp32.
 */
HILS_API hils_status hils_select(const hils_shape* shape, const void* q, const float* kbar,
                        const float* hbias, int32_t* topk_idx, float* topk_score, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * hils_attend -- the whole prefill forward pass: summaries, scores, Top-K,
 * intra-chunk softmax attention over each selected chunk and over the
 * query's own causal partial chunk, and the inter-chunk fusion (notes
 * section 5.3: w_ij = exp(s_ij)/Z_{i,c(j)} * Zhat_{i,c(j)}/Zhat_i with
 * Zhat_{i,c} = exp(shat_{i,c}); Tide Figure 3).  The own chunk enters Zhat_i
 * with its exact mass exp(LSE_own).
 *   q, k, v      prefill layout (dtype)
 *   landmark_q   [batch, heads_q, C, head_dim] (dtype)
 *   out          [batch, heads_q, seq_len, head_dim] (dtype), written
 *   lse_out      [batch, heads_q, seq_len] fp32 or NULL: log Zhat_i, the
 *                log-sum-exp of the row's fusion logits (the selected
 *                chunks' shat and the local branch's exact log-mass), the
 *                row statistic a backward pass needs
 *   topk_idx_out [batch, heads_kv, seq_len, top_k] int32 or NULL
 *   ws           workspace of hils_workspace_size(HILS_OP_ATTEND) bytes,
 *                zero-filled before first use: the error word, the
 *                summaries, the selection and its scores, the select
 *                scratch of hils_select and the chunk-major scratch of
 *                hils_attend_selected (all rewritten by every call)
 */
HILS_API hils_status hils_attend(const hils_shape* shape, const void* q, const void* k, const void* v,
                        const void* landmark_q, void* out, float* lse_out, int32_t* topk_idx_out,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * hils_attend_selected -- the attention half of hils_attend for a selection
 * the caller already holds (for instance from hils_select, or from scores
 * computed with a separate scoring query): intra-chunk softmax attention over
 * each listed chunk and over the own causal partial chunk, fused with the
 * inter-chunk softmax of notes section 5.3 (own chunk at its exact mass).
 *   q, k, v      prefill layout (dtype)
 *   topk_idx     [batch, heads_kv, seq_len, top_k] int32; -1 = unused slot;
 *                an entry that is not a remote candidate of row i (outside
 *                [0, floor(i/B) + 1 - W/B)) is skipped and flagged in the
 *                error word
 *   topk_score   [batch, heads_q, seq_len, top_k] fp32: shat of each listed
 *                chunk for each query head
 *   out          [batch, heads_q, seq_len, head_dim] (dtype), written
 *   lse_out      [batch, heads_q, seq_len] fp32 or NULL: log Zhat_i as in
 *                hils_attend
 *   ws           workspace of hils_workspace_size(HILS_OP_ATTEND_SELECTED)
 *                bytes, zero-filled before first use: the error word and,
 *                for bf16 shapes that take the chunk-major path (the
 *                selections bucketed by chunk into 128-row tiles, a bf16
 *                partial output per selection, fused per row afterwards),
 *                its bucket counts, tile list, selection positions and
 *                partials; other shapes use the error word only
 */
HILS_API hils_status hils_attend_selected(const hils_shape* shape, const void* q, const void* k,
                                          const void* v, const int32_t* topk_idx,
                                          const float* topk_score, void* out, float* lse_out,
                                          void* ws, size_t ws_bytes, void* stream);

/*
 * hils_backward -- gradients of the prefill forward pass (hils_attend) with
 * respect to q, k, v and the landmark queries, for an upstream gradient dout
 * (notes section 5.3: the hierarchical softmax carries the loss into the
 * chunk scores, so the selector is trained by it; Tide Figure 3 caption: the
 * gradients reach the compressed key).  The Top-K selection of the forward is
 * held fixed; every other step is differentiated exactly: the intra-chunk and
 * local softmaxes, the inter-chunk softmax over shat and the local log-mass,
 * shat = q.kbar * scale + H, and the landmark softmax that makes kbar and H
 * (notes section 5.1).  Unselected chunks receive gradient only through the
 * local branches that contain them.
 *   q, k, v, landmark_q   the forward's inputs (bf16 only: HILS_ERR_UNSUPPORTED
 *                         for HILS_F32)
 *   out                   [batch, heads_q, seq_len, head_dim] bf16, the forward's output
 *   lse                   [batch, heads_q, seq_len] fp32, the forward's lse_out
 *   topk_idx, topk_score  the forward's selection and each head's shat of it
 *                         (hils_select's outputs); may be NULL when top_k == 0
 *   dout                  [batch, heads_q, seq_len, head_dim] bf16
 *   dq                    [batch, heads_q, seq_len, head_dim] fp32, written
 *   dk, dv                [batch, heads_kv, seq_len, head_dim] fp32, written
 *   dlandmark             [batch, heads_q, C, head_dim] fp32, written
 *   ws                    workspace of hils_workspace_size(HILS_OP_BACKWARD)
 * Selection entries outside row i's candidates are skipped and flagged.
 */
HILS_API hils_status hils_backward(const hils_shape* shape, const void* q, const void* k, const void* v,
                          const void* landmark_q, const void* out, const float* lse,
                          const int32_t* topk_idx, const float* topk_score, const void* dout,
                          float* dq, float* dk, float* dv, float* dlandmark, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * hils_decode -- one decode step per sequence over a paged chunk cache.
 * The new query of sequence b sits at position seq_lens[b]-1 and its key and
 * value are already in the cache.  Own chunk = floor((seq_lens[b]-1)/B);
 * the local branch is the own chunk (shape.window 0 or B) or the last
 * window/B chunks up to the new token; candidates are the complete chunks
 * before the local branch, scored with the cached summaries; then the same
 * intra-chunk attention and fusion as hils_attend.
 *   q            [batch, heads_q, head_dim] (dtype)
 *   k_pages,
 *   v_pages      [n_pages, heads_kv, B, head_dim] (dtype)
 *   kbar_pages   [n_pages, heads_q, head_dim] fp32 (hils_summarize_paged)
 *   hbias_pages  [n_pages, heads_q] fp32
 *   block_table  [batch, max_chunks] int32: page of chunk c of sequence b
 *   seq_lens     [batch] int32, each <= max_chunks * B and <= shape.seq_len;
 *                a sequence with seq_lens[b] <= 0 gets a zero output
 *   out          [batch, heads_q, head_dim] (dtype), written
 *   topk_idx_out [batch, heads_kv, top_k] int32 or NULL
 *   ws           workspace of hils_workspace_size(HILS_OP_DECODE) bytes
 * Page ids outside [0, n_pages) are skipped and flagged in the error word.
 * max_chunks is limited to about 2^24 / top_k (the Top-K merge of the
 * scan's per-range lists runs in shared memory); beyond it the call returns
 * HILS_ERR_UNSUPPORTED.
 */
HILS_API hils_status hils_decode(const hils_shape* shape, const void* q, const void* k_pages,
                        const void* v_pages, const float* kbar_pages, const float* hbias_pages,
                        const int32_t* block_table, int32_t max_chunks, const int32_t* seq_lens,
                        int32_t n_pages, void* out, int32_t* topk_idx_out, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * hils_decode_static -- hils_decode with no workspace argument.  The HiLS
 * notes have no counterpart: this is a plumbing variant for callers that
 * cannot hand the library a device buffer, e.g. an engine whose device memory
 * is carved up once at start-up, or a loop that must not call cudaMalloc or
 * cudaFree, which can synchronise the whole device and stall its other
 * streams.  The call itself allocates and frees nothing: its scratch is one
 * fixed device array of HILS_DECODE_STATIC_SCRATCH_BYTES bytes inside
 * libhils.so.
 *   Arguments as for hils_decode, except:
 *   status_word  NULL, or a 4-byte-aligned device word, zero-filled by the
 *                caller, into which the kernels OR their error bits (read
 *                and clear it with hils_device_status(status_word, stream));
 *                with NULL, device-side errors are not reported
 * Returns HILS_ERR_WORKSPACE, without launching anything, when the shape
 * needs more scratch than the array holds (batch * heads_kv > 4096, or
 * roughly 256 + 32 KiB + what hils_workspace_size(HILS_OP_DECODE) reports
 * beyond its own 256-byte header > HILS_DECODE_STATIC_SCRATCH_BYTES).
 * The first call on each device looks up the array's device address (this
 * may load the library's device code onto that device): make it before any
 * stream capture starts.
 * Every call on a device uses the same array: calls whose kernels may run at
 * the same time (different streams with no ordering between them, or
 * different host threads) race on it and corrupt each other's results; order
 * them on one stream or with events.  Its ticket counters (taken by the
 * attention kernel's CTAs, the last of each (sequence, KV head) resetting
 * its own) must start at zero: they are zero when the library's device code
 * is loaded, and each call whose attention kernel runs to completion leaves
 * them at zero again.  A call whose second launch fails (HILS_ERR_CUDA after
 * the first kernel was enqueued) touches no ticket; an attention kernel that
 * starts but does not complete can leave tickets non-zero, and later calls
 * on that device then return wrong results until the library's device code
 * is loaded again (a new process).
 * kbar_pages must be the fp32 summary cache (this entry point has no
 * summary_dtype argument).
 */
#define HILS_DECODE_STATIC_SCRATCH_BYTES (4u << 20)
HILS_API hils_status hils_decode_static(const hils_shape* shape, const void* q, const void* k_pages,
                        const void* v_pages, const float* kbar_pages, const float* hbias_pages,
                        const int32_t* block_table, int32_t max_chunks, const int32_t* seq_lens,
                        int32_t n_pages, void* out, int32_t* topk_idx_out, unsigned* status_word,
                        void* stream);

/*
 * hils_summarize_paged_ex, hils_decode_ex -- hils_summarize_paged and
 * hils_decode with the cached summaries kbar_pages stored in summary_dtype:
 * HILS_F32 (the plain entry points) or HILS_BF16, a compact cache that
 * halves the bytes the decode scan reads (the summaries of a 512K context
 * are most of a decode step's memory traffic).  Scores from bf16 summaries
 * carry the bf16 rounding of kbar (relative error up to 2^-9 per element,
 * about 2^-9 |q||kbar| * scale on a score), so their Top-K may differ from
 * the fp32 cache's where candidate keys lie that close.  H stays fp32.
 * HILS_BF16 summaries require shape.dtype == HILS_BF16 (HILS_ERR_UNSUPPORTED
 * otherwise); an unknown summary_dtype is HILS_ERR_INVALID_ARG.  The HiLS
 * pages fix no storage precision for kbar; the bf16 cache is an option of
 * this library.
 */
HILS_API hils_status hils_summarize_paged_ex(const hils_shape* shape, const void* k_pages,
                                    const void* landmark_pages, const int32_t* page_ids,
                                    int32_t n_listed, int32_t n_pages, void* kbar_pages,
                                    int32_t summary_dtype, float* hbias_pages, void* stream);
HILS_API hils_status hils_decode_ex(const hils_shape* shape, const void* q, const void* k_pages,
                           const void* v_pages, const void* kbar_pages, int32_t summary_dtype,
                           const float* hbias_pages, const int32_t* block_table,
                           int32_t max_chunks, const int32_t* seq_lens, int32_t n_pages,
                           void* out, int32_t* topk_idx_out, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * hils_device_status -- synchronises `stream`, reads and clears the error
 * word at the start of a hils_attend / hils_attend_selected / hils_decode
 * workspace, and returns HILS_OK, HILS_ERR_DEVICE_CHECK or
 * HILS_ERR_DEVICE_TIMEOUT.  The word is sticky: kernels only set bits, so it
 * reports every error since the last read.  A new workspace must be
 * zero-filled once before its first use.
 */
HILS_API hils_status hils_device_status(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H_ */
