/*
 * lserve.h -- C ABI of the unified block-sparse attention library (liblserve.so).
 *
 * One library serves both phases of LServe-style unified sparse attention
 * (mlsanity, "LServe: Efficient Long-sequence LLM Serving with Unified Sparse
 * Attention", Abstract: structured sparsity for prefilling and decoding in one
 * framework, computations on less important tokens skipped block-wise):
 *
 *   prefill  causal flash attention that skips whole 64x64 KV tiles; dense KV
 *            heads keep every causal tile (optionally ANDed with a block mask),
 *            streaming KV heads keep only the Lambda support (sink tokens plus a
 *            local window)  -- LServe + SampleAttention blog post, "LServe -
 *            Prefill Phase", Fig. 1(a)/(b);
 *   decode   per-logical-page key min/max summaries, an upper-bound page score,
 *            the max over the logical pages of each physical page, top-k pages
 *            within a token budget, then split-KV paged attention over only those
 *            pages and a log-sum-exp merge -- same blog post, "LServe - Decode
 *            Phase", Fig. 2; the summary/bound follow Quest (listed under
 *            "Builds on" on the mlsanity LServe page).
 *
 * Conventions (all entry points):
 *   - Every tensor pointer is DEVICE memory owned by the caller; the library
 *     never allocates, frees or keeps a pointer past the call.  Workspaces are
 *     caller-provided; query their size with the *_workspace_size functions.
 *     Workspace contents on entry are ignored; on return they are undefined.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream; none synchronises the host except
 *     lserve_get_device_status.
 *   - Argument errors are detected on the host and returned before anything is
 *     launched.  Launch failures return LSERVE_ERR_CUDA.  Errors found by the
 *     kernels themselves (an out-of-range page id, a bounded wait that ran out)
 *     are recorded in a per-device status word, read by lserve_get_device_status.
 *   - bf16 means IEEE bfloat16 stored as uint16; all tensors are dense,
 *     row-major, in the layout given (last index fastest), 16-byte aligned.
 *   - Supported: head_dim d in {64, 128}; Hq a multiple of Hkv; physical page
 *     64 tokens, logical page 16 tokens, prefill tile 64x64.  Anything else
 *     returns LSERVE_ERR_UNSUPPORTED.  There is no fallback path.
 *   - No exception crosses the ABI.  The library keeps no state between calls
 *     except the device status word, the thread-local error string and the
 *     fixed scratch array of lserve_decode_noalloc.
 */
#ifndef LSERVE_H_
#define LSERVE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lserve_status {
  LSERVE_OK = 0,
  LSERVE_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad sink/local/budget   */
  LSERVE_ERR_UNSUPPORTED = 2,     /* shape outside the supported set (see above)          */
  LSERVE_ERR_WORKSPACE = 3,       /* workspace pointer null/misaligned or too small       */
  LSERVE_ERR_CUDA = 4,            /* a CUDA runtime call or kernel launch failed          */
  LSERVE_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait ran out (device status)      */
  LSERVE_ERR_DEVICE_BOUNDS = 6    /* an out-of-range index, or an INT4 operand past fp16 (device status) */
} lserve_status;

#define LSERVE_PAGE 64            /* tokens per physical KV page                          */
#define LSERVE_LOGICAL_PAGE 16    /* tokens per logical page (granularity of the summary) */
#define LSERVE_TILE 64            /* prefill tile: 64 query rows x 64 keys                */

/* Head kinds (uint8 per KV head). */
#define LSERVE_HEAD_DENSE 0       /* retrieval head: all causal tiles / top-k pages       */
#define LSERVE_HEAD_STREAMING 1   /* streaming head: Lambda support (sink + local window) */

/* ------------------------------------------------------------------ prefill */

typedef struct lserve_shape {
  int32_t B;      /* batch                                                         */
  int32_t S;      /* sequence length, a positive multiple of 64                    */
  int32_t Hq;     /* query heads                                                   */
  int32_t Hkv;    /* KV heads; query head h reads KV head h / (Hq / Hkv)           */
  int32_t d;      /* head dim, 64 or 128                                           */
  float scale;    /* softmax scale; <= 0 selects 1/sqrt(d)                         */
  int32_t lambda_tiles; /* 0: token-level Lambda support of streaming heads;
                           1: tile-level (whole 64x64 tiles, see lserve_prefill) */
} lserve_shape;

/*
 * Bytes of workspace lserve_prefill needs for `shape` (0 on an invalid shape).
 * It holds the kept-tile lists (CSR), the longest-first work order and
 * counters; it is sized for the worst case (every causal tile kept).
 */
size_t lserve_prefill_workspace_size(const lserve_shape* shape);

/*
 * Block-sparse causal prefill attention.
 *
 * Kept set of query row i (token position within its sequence) for query head
 * h, KV head g = h / (Hq/Hkv):
 *   dense g      (head_kind[g] == 0):  { j <= i : block_mask[b,g,i/64,j/64] != 0 }
 *                                       (every j <= i when block_mask == NULL)
 *   streaming g  (head_kind[g] == 1):  { j <= i : j < sink  or  i - j < local }
 *   streaming g, shape->lambda_tiles == 1 (the tile-level reading of the blog's
 *                "no partial blocks", Fig. 1(b)): every causal key of every
 *                64x64 tile that meets that support,
 *                { j <= i : 64 (j/64) < sink  or  max(64 (i/64) - 64 (j/64) - 63, 0) < local }
 * out[b,i,h,:] = sum_j softmax_j(scale * q.k_j) v_j over the kept set; a row
 * whose kept set is empty gets out = 0 and lse = -inf.  A 64x64 tile with no
 * kept element is never read (whole-tile skipping, blog "LServe - Prefill
 * Phase", Fig. 1(a)); elements inside kept tiles are masked exactly.
 *
 *   q          bf16 [B, S, Hq, d]
 *   k, v       bf16 [B, S, Hkv, d]
 *   head_kind  uint8 [Hkv]                    (device)
 *   sink,local >= 0 tokens                    (used by streaming heads only)
 *   block_mask uint8 [B, Hkv, S/64, S/64] or NULL; read for dense heads only,
 *              ANDed with causality (entries above the diagonal are ignored)
 *   out        bf16 [B, S, Hq, d]             (written)
 *   lse        fp32 [B, Hq, S] or NULL        (natural-log LSE of the kept logits)
 *   workspace  >= lserve_prefill_workspace_size(shape) bytes, 256-byte aligned
 */
lserve_status lserve_prefill(const lserve_shape* shape, const void* q, const void* k,
                             const void* v, const uint8_t* head_kind, int32_t sink,
                             int32_t local, const uint8_t* block_mask, void* out,
                             float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * The tile-list step of lserve_prefill on its own, for inspection: the kept
 * KV tiles of every (b, kvh, qt) row as a CSR.  Row r = (b*Hkv + kvh)*(S/64) + qt.
 *   row_offsets int32 [B*Hkv*(S/64) + 1]      (written; row_offsets[0] = 0)
 *   tile_cols   uint16 [max_nnz]              (written; kt ascending within a row)
 *   max_nnz     capacity of tile_cols; B*Hkv*n*(n+1)/2 with n = S/64 always fits.
 *               If the kept tiles exceed it the call records LSERVE_ERR_DEVICE_BOUNDS
 *               in the device status and writes nothing past the capacity.
 * Same tile rule as lserve_prefill: dense rows keep kt <= qt (ANDed with the
 * block mask); streaming rows keep kt <= qt with 64*kt < sink or
 * max(64*qt - 64*kt - 63, 0) < local.
 */
lserve_status lserve_prefill_tile_lists(const lserve_shape* shape, const uint8_t* head_kind,
                                        int32_t sink, int32_t local,
                                        const uint8_t* block_mask, int32_t* row_offsets,
                                        uint16_t* tile_cols, int64_t max_nnz,
                                        void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- page summaries */

/*
 * Per-logical-page key summaries for the decode selector (blog "LServe - Decode
 * Phase": every page scored from a summary vector; Quest min/max summary).
 *
 * For every sequence b, every physical page i < ceil(seq_lens[b]/64) of its
 * page table, every DENSE KV head g and every logical page l in 0..3 whose
 * sequence-wide index 4*i + l >= first_logical_page:
 *   stats[p,g,l,0,c] = min over the valid tokens t (t < seq_lens[b]) of the
 *                      logical page of k[t,g,c];  stats[p,g,l,1,c] = max.
 *   A logical page without a valid token gets min = +inf, max = -inf.
 * p = page_table[b*maxP + i].  Min/max of bf16 values are exact: results are
 * bit-identical to any correct implementation.  Streaming heads and pages not
 * reached are left untouched.
 *
 *   k_pages     bf16 [num_pages, Hkv, 64, d]
 *   page_table  int32 [B, maxP]; entries must lie in [0, num_pages)
 *               (an entry outside records LSERVE_ERR_DEVICE_BOUNDS and is skipped)
 *   seq_lens    int32 [B], 0 <= seq_lens[b] <= 64*maxP (device)
 *   first_logical_page  0 = full rebuild; > 0 = refresh only logical pages at or
 *               past this index (after appending tokens)
 *   head_kind   uint8 [Hkv] (device)
 *   stats       bf16 [num_pages, Hkv, 4, 2, d] (written)
 */
lserve_status lserve_update_page_stats(int32_t B, int32_t Hkv, int32_t d, int32_t num_pages,
                                       const void* k_pages, const int32_t* page_table,
                                       int32_t maxP, const int32_t* seq_lens,
                                       int32_t first_logical_page, const uint8_t* head_kind,
                                       void* stats, void* stream);

/*
 * lserve_build_vslash_mask -- a vertical-slash block mask for the dense heads,
 * built from sampled queries.
 *
 * LServe + SampleAttention blog post, "SampleAttention - Column Pattern" and
 * "Slash Pattern" (Fig. 3), with "CRA - The Accuracy Proxy" (Fig. 4): column
 * and slash candidates are added until the worst-kept query keeps a share tau
 * of its causal softmax mass.  The post leaves the estimator to its paper; this
 * library's reading, at the 64 x 64 tile grain of lserve_prefill:
 *   sampled queries  the last row of query tiles nQT-1, nQT-1-stride, ... (>= 0),
 *                    each for the Hq/Hkv query heads of the KV head
 *   tile masses      r[s,h,kt] = that row's causal softmax weights (exact, over
 *                    all keys <= the row) summed over the keys of tile kt
 *   candidates       column kt (tiles (qt, kt), qt >= kt), score sum_{s,h} r[s,h,kt];
 *                    slash delta (tiles (qt, qt - delta)), score sum_{s,h} r[s,h,qt(s)-delta]
 *   greedy           the diagonal slash (delta = 0) first, always; then by score,
 *                    descending (equal scores: columns first, then the lower
 *                    index); stop as soon as min over (s, h) of the retained mass
 *                    (r summed over the row's covered tiles) is >= tau
 *   mask             block_mask[b,g,qt,kt] = 1 for kt <= qt covered by a taken
 *                    column or slash, else 0
 * Streaming heads get an all-zero mask (lserve_prefill ignores it for them),
 * cra 0 and no candidates.  The mask is ready to pass to lserve_prefill and
 * lserve_cra.
 *
 *   q, k           bf16 [B, S, Hq, d], [B, S, Hkv, d]; S a multiple of 64, d in {64, 128}
 *   head_kind      uint8 [Hkv]                   (device)
 *   sample_stride  >= 1; (S/64 - 1)/stride + 1 rows sampled per (sequence, KV head);
 *                  rows x Hq/Hkv at most 16384, Hq/Hkv at most 8, S/64 at most 8192
 *   tau            in [0, 1]
 *   block_mask     uint8 [B, Hkv, S/64, S/64]     (written)
 *   cra            fp32 [B, Hkv] or NULL: the sampled rows' minimum retained mass
 *   n_columns, n_slashes  int32 [B, Hkv] or NULL: candidates taken (the diagonal counts as a slash)
 *   workspace      >= lserve_vslash_workspace_size(shape, stride) bytes, 256-byte
 *                  aligned (the tile masses: B*Hkv*rows*Hq/Hkv*S/64 floats)
 * Errors: LSERVE_ERR_INVALID_ARG (shape, stride < 1, tau outside [0, 1], null or
 * misaligned pointers), LSERVE_ERR_UNSUPPORTED (d, S, Hq/Hkv or sample count past
 * the limits above), LSERVE_ERR_WORKSPACE.  Asynchronous on the stream.
 */
size_t lserve_vslash_workspace_size(const lserve_shape* shape, int32_t sample_stride);
lserve_status lserve_build_vslash_mask(const lserve_shape* shape, const void* q, const void* k,
                                       const uint8_t* head_kind, int32_t sample_stride, float tau,
                                       uint8_t* block_mask, float* cra, int32_t* n_columns,
                                       int32_t* n_slashes, void* workspace, size_t ws_bytes,
                                       void* stream);

/*
 * lserve_cra -- cumulative residual attention of a sparse prefill mask.
 *
 * LServe + SampleAttention blog post, "CRA - The Accuracy Proxy", Fig. 4: for
 * every query row i, the share r_i of its causal softmax probability mass that
 * the sparse mask keeps, and CRA = the minimum of r_i over the rows -- the
 * worst-kept query, which a mask is judged by.  The mask is given exactly as to
 * lserve_prefill (head_kind, sink, local, block_mask, shape->lambda_tiles).  Computed from two LSE-only
 * passes of the prefill kernel (causal, and the sparse mask; no output written):
 * r_i = exp(lse_sparse(i) - lse_causal(i)); a row that keeps nothing retains 0.
 *
 *   retained  fp32 [B, Hq, S] or NULL: r_i of every row
 *   cra       fp32 [B, Hq]: min_i r_i
 *   workspace >= lserve_cra_workspace_size(shape) bytes, 256-byte aligned
 * Errors and stream behaviour as for lserve_prefill.
 */
size_t lserve_cra_workspace_size(const lserve_shape* shape);
lserve_status lserve_cra(const lserve_shape* shape, const void* q, const void* k, const void* v,
                         const uint8_t* head_kind, int32_t sink, int32_t local,
                         const uint8_t* block_mask, float* retained, float* cra, void* workspace,
                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------- decode */

typedef struct lserve_decode_args {
  int32_t B, Hq, Hkv, d;
  int32_t num_pages;          /* physical pages in the pool                              */
  int32_t maxP;               /* row length of page_table                                */
  const void* q;              /* bf16 [B, Hq, d]: one query token per sequence            */
  const void* k_pages;        /* bf16 [num_pages, Hkv, 64, d]                            */
  const void* v_pages;        /* bf16 [num_pages, Hkv, 64, d]                            */
  const int32_t* page_table;  /* int32 [B, maxP]                                         */
  const int32_t* seq_lens;    /* int32 [B]: tokens in the cache, the query's own included */
  const void* stats;          /* bf16 [num_pages, Hkv, 4, 2, d] from lserve_update_page_stats */
  const uint8_t* head_kind;   /* uint8 [Hkv]                                             */
  int32_t sink, local;        /* streaming heads: tokens t < sink or t >= seq_len - local */
  int32_t token_budget;       /* dense heads keep k = min(budget/64, n_pages) pages; >= 64 */
  float scale;                /* <= 0 selects 1/sqrt(d)                                  */
} lserve_decode_args;

/* Capacity (pages) of one selection row: max(min(budget/64, maxP), streaming pages). */
int32_t lserve_decode_max_selected(const lserve_decode_args* args);

/* Bytes of workspace lserve_decode needs (page scores, selection, partition,
 * per-warp partials); lserve_decode_reuse needs the same, and may ask with
 * stats = NULL, and so does lserve_decode_int4.  It depends on the current
 * device's SM count (the attention grid is one wave of SMs x 2 CTAs, x 3 for
 * INT4 pages) or, when the environment variable LSERVE_DECODE_GRID holds a
 * positive integer, on that grid size; ask again after changing either. */
size_t lserve_decode_workspace_size(const lserve_decode_args* args);

/*
 * One sparse decode step for B sequences.
 *
 * Dense KV head g of sequence b (n = ceil(seq_len/64) pages):
 *   bound of query head h on logical page l:  s_h(l) = sum_c max(q_h,c*kmax_c, q_h,c*kmin_c)
 *   group score    s(l) = max over the Hq/Hkv query heads of g of s_h(l)
 *   page score     max of s(l) over the logical pages holding a valid token
 *   selection      the k = min(token_budget/64, n) highest-scoring pages, ties to
 *                  the lower page index, listed in ascending page order
 *   attention      softmax(scale * q.k_t) over every valid token t of the
 *                  selected pages.  All units' selected pages are dealt out
 *                  evenly to one wave of CTAs; the partial results of a unit
 *                  are merged by log-sum-exp.
 * Streaming KV head: the pages holding tokens [0, sink) and
 * [seq_len - local, seq_len), attending to exactly those tokens.
 * The query is at position seq_len - 1 (its own key/value are in the cache).
 *
 *   out      bf16 [B, Hq, d] (written)
 *   lse      fp32 [B, Hq] or NULL
 *   sel_out  int32 [B, Hkv, lserve_decode_max_selected(args)] or NULL: selected
 *            page indices (within the sequence, ascending; unused slots -1)
 *   sel_n    int32 [B, Hkv] or NULL: number of selected pages
 *   workspace >= lserve_decode_workspace_size(args) bytes, 256-byte aligned
 */
lserve_status lserve_decode(const lserve_decode_args* args, void* out, float* lse,
                            int32_t* sel_out, int32_t* sel_n, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * lserve_decode_noalloc -- lserve_decode for callers that cannot allocate.
 *
 * The paper has no counterpart to this entry point; it exists for deployment.
 * Some callers must not allocate device memory at all once they are running:
 * serving loops that fix their memory budget at start-up and keep the
 * allocator (and its implicit synchronisation) off the per-token path, and
 * plugin hosts that own every device allocation and hand a kernel library only
 * its input and output buffers.  Such callers cannot provide the workspace
 * lserve_decode needs.  This variant computes exactly what lserve_decode
 * computes, with the same arguments except the workspace, and takes its
 * scratch (page scores, selections, split partials) from a fixed array of
 * LSERVE_NOALLOC_SCRATCH_BYTES that is part of the library image on every
 * device that loads it, held until the process exits.  It calls no cudaMalloc,
 * cudaFree or any other allocating routine.
 *
 *   - The first call in each CUDA context of a device looks up that array's
 *     device address (with that device current) and caches it; make that first
 *     call before any stream capture.  After cudaDeviceReset the next call
 *     looks it up again.
 *   - The split partials of the attention grid grow with its width.  When a
 *     full wave's would not fit in the array, the call narrows the grid to the
 *     widest one whose scratch fits; the result is the same attention, merged
 *     from fewer splits (equal to lserve_decode's within rounding; the page
 *     selection is identical).  Only a batch whose scratch exceeds
 *     LSERVE_NOALLOC_SCRATCH_BYTES even on a one-CTA grid (page scores and
 *     selections of B * Hkv rows of maxP pages, mostly) is rejected, with
 *     LSERVE_ERR_WORKSPACE, before anything is launched.
 *     lserve_decode_workspace_size gives the need of lserve_decode's full-wave
 *     grid, an upper bound of this call's.
 *   - All calls on a device share the one array and it keeps whatever the last
 *     call left in it (nothing in it needs to start at zero).  Calls whose
 *     kernels overlap on the GPU -- on different streams, or from different
 *     host threads -- race on it; serialise them on one stream.
 */
#define LSERVE_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB per device */
lserve_status lserve_decode_noalloc(const lserve_decode_args* args, void* out, float* lse,
                                    int32_t* sel_out, int32_t* sel_n, void* stream);

/*
 * lserve_quantize_pages_int4 -- INT4 KV pages for lserve_decode_int4.
 *
 * LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2: INT4
 * KV quantization cuts the bytes of every page read.  The pages name no scheme;
 * this one is asymmetric INT4 with one step s and offset lo per (page, KV
 * head, channel) for keys (over the page's valid tokens) and per (page, KV
 * head, token) for values (over the d channels), in float32:
 *   s = (hi - lo) / 15,  code = clamp(rint((x - lo) / s), 0, 15) (0 when s == 0),
 *   dequantised value = fma(code, s, lo) in float32.
 * The pages sequence b holds from page index first_page onward (0: all) are
 * quantised from the bf16 pools, and the page summaries of dense heads are
 * written from the dequantised keys, minimum rounded down and maximum rounded
 * up to bf16 (so they bound what lserve_decode_int4 attends to).  Rows past seq_len get code 0 (values: s = lo = 0).
 *
 *   k_pages, v_pages  bf16 [num_pages, Hkv, 64, d] (read)
 *   kq                uint8 [num_pages, Hkv, 64, d/2] (written): one key row per
 *                     token, its codes in the order of the decode step's operand
 *                     fragments: four chunks of d/8 bytes; word w of chunk t holds
 *                     nibbles n = j + 4e (nibble n in bits 4n..4n+3) of channels
 *                     16 (r/2) + 8 (r%2) + 2t + e, r = 4w + j
 *   vq                uint8 [num_pages, Hkv, 64 * d/2] (written): four slices of
 *                     16 tokens, each 32 chunks of d/4 bytes; word m of chunk
 *                     4g + t holds nibbles n = j + 4e of channel 16m + g + 8 (j%2),
 *                     token 16 slice + 2t + 8 (j/2) + e
 *   kpar              fp32 [num_pages, Hkv, 2, d] (written): s, then lo, each in
 *                     four chunks of d/4 channels, entry i of chunk t being
 *                     channel 16 (i/4) + 8 ((i/2)%2) + 2t + i%2
 *   vpar              fp32 [num_pages, Hkv, 64, 2] (written): (s, lo) per token
 *   stats             bf16 [num_pages, Hkv, 4, 2, d] (dense heads written)
 * All device memory, owned by the caller; k_pages, v_pages, kq, vq and stats
 * 16-byte aligned.  The call is asynchronous on the stream.
 * Errors: LSERVE_ERR_INVALID_ARG (sizes, null or misaligned pointers),
 * LSERVE_ERR_UNSUPPORTED (d not 64 or 128); a page_table entry outside
 * [0, num_pages) is skipped and reported as LSERVE_ERR_DEVICE_BOUNDS by
 * lserve_get_device_status.
 */
lserve_status lserve_quantize_pages_int4(int32_t B, int32_t Hkv, int32_t d, int32_t num_pages,
                                        const void* k_pages, const void* v_pages,
                                        const int32_t* page_table, int32_t maxP,
                                        const int32_t* seq_lens, int32_t first_page,
                                        const uint8_t* head_kind, void* kq, float* kpar, void* vq,
                                        float* vpar, void* stats, void* stream);

/*
 * lserve_decode_int4 -- lserve_decode over INT4 pages.
 *
 * LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2: the
 * same selection and attention as lserve_decode, with every K and V row read
 * as INT4 codes: keys s_c code + lo_c, values s_t code + lo_t (the values
 * lserve_quantize_pages_int4 defines).  The steps are folded into the other
 * operand: the tensor cores multiply the integer codes, exact in fp16, by s q
 * (carried as the sum of two fp16 parts, so about 2^-22 of each product is
 * lost) and by s p (one fp16 part, 2^-11).  The offsets go into one fp32 term
 * per head; no dequantised value is ever rounded to a 16-bit format.  Range:
 * each |s_c q_c| and |s_t| must stay within the fp16 range (65504); a page
 * whose key steps times q exceed it is reported as LSERVE_ERR_DEVICE_BOUNDS by
 * lserve_get_device_status (its output is then not meaningful).
 * args->k_pages / args->v_pages point at the code pools kq / vq and args->stats
 * at the summaries that lserve_quantize_pages_int4 wrote (so the bound holds for
 * the dequantised keys).
 *
 *   kpar   fp32 [num_pages, Hkv, 2, d], 16-byte aligned (read)
 *   vpar   fp32 [num_pages, Hkv, 64, 2], 16-byte aligned (read)
 *   out, lse, sel_out, sel_n, workspace: as lserve_decode (the same
 *   lserve_decode_workspace_size).
 * Errors: LSERVE_ERR_INVALID_ARG for a null or misaligned kpar / vpar, every
 * error lserve_decode returns, and the device-reported range error above.
 */
lserve_status lserve_decode_int4(const lserve_decode_args* args, const float* kpar,
                                 const float* vpar, void* out, float* lse, int32_t* sel_out,
                                 int32_t* sel_n, void* workspace, size_t ws_bytes, void* stream);

/*
 * lserve_decode_reuse -- a decode step that keeps an earlier page selection.
 *
 * LServe + SampleAttention blog post, "LServe - Decode Phase": selection
 * results are reused across a small window of decode steps, so that the page
 * scoring is not paid on every token.  This call computes lserve_decode's
 * attention with each dense head's page set taken from sel_in / sel_n_in
 * instead of being scored and selected; the page summaries are not read
 * (args->stats may be NULL) and no scoring kernel runs.
 *
 *   sel_in    int32 [B, Hkv, lserve_decode_max_selected(args)]: page indices
 *             within each sequence (ascending), as lserve_decode wrote them to
 *             sel_out at an earlier step of the same batch (same B, Hkv, maxP,
 *             token_budget, sink, local).  Only the rows of dense heads are read.
 *   sel_n_in  int32 [B, Hkv]: valid entries of each row (clamped to the row
 *             capacity).
 *
 * A dense head of sequence b attends to every token t < seq_lens[b] of those
 * pages: tokens appended since the selection count where they fall in a
 * selected page, not elsewhere.  A streaming head takes its sink and local
 * window from the current seq_lens, as in lserve_decode.  A page index outside
 * [0, maxP) is recorded as LSERVE_ERR_DEVICE_BOUNDS and its tokens are skipped.
 * out, lse, sel_out, sel_n and the workspace are as for lserve_decode (the same
 * workspace size suffices); sel_out / sel_n may be sel_in / sel_n_in (the dense
 * rows are copied onto themselves, the streaming rows refreshed).
 */
lserve_status lserve_decode_reuse(const lserve_decode_args* args, const int32_t* sel_in,
                                  const int32_t* sel_n_in, void* out, float* lse, int32_t* sel_out,
                                  int32_t* sel_n, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ status */

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word: LSERVE_OK, LSERVE_ERR_DEVICE_TIMEOUT or LSERVE_ERR_DEVICE_BOUNDS (the
 * first error recorded since the last read), or LSERVE_ERR_CUDA if the
 * synchronisation itself failed.
 */
lserve_status lserve_get_device_status(void* stream);

/* Message of the last error returned on the calling thread ("" if none). */
const char* lserve_last_error_string(void);

/* Library version, e.g. "0.1.0". */
const char* lserve_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LSERVE_H_ */
