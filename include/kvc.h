/*
 * kvc.h -- C ABI of libkvc: observation-window token scoring, top-k selection
 * that always keeps the window, and compaction (gather) of K/V rows and hidden
 * states, as used by window-based KV-cache compression at prefill.
 *
 * The operations are the ones described in
 *   [FastKV]   "FastKV: Decoupling of Context Reduction and KV Cache
 *              Compression for Prefill-Decoding Acceleration"
 *              (gist.science, 2502.01068), sections 2.A (Token-Selective
 *              Propagation) and 2.B (decoupled KV retention), and its abstract
 *              (chatpaper.ai, "FastKV: KV Cache Compression for Fast
 *              Long-Context Processing with Token-Selective Propagation":
 *              GQA-aware KV compression);
 *   [StructKV] "StructKV: Preserving the Structural Skeleton for Scalable
 *              Long-Context Inference" (gist.science, 2604.06746), sections
 *              2.A (global in-degree centrality) and 2.B (entropy, sparsity
 *              and variance monitoring).
 *
 * Conventions (apply to every entry point unless stated otherwise)
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or synchronises device memory or streams; scratch
 *    space is the caller's `ws` buffer, sized by the matching *_workspace_size
 *    call.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  A returned KVC_OK means "validated and
 *    launched", not "finished".
 *  - bf16 tensors are passed as `uint16_t*` holding raw bf16 bit patterns.
 *  - Strides are in ELEMENTS (not bytes).  The innermost dimension (head_dim
 *    or hidden) must be contiguous.  K/Q pointers must be 16-byte aligned and
 *    their token/head strides multiples of 8 elements (16 bytes).
 *  - Arguments are validated on the host before any launch; an invalid call
 *    returns an error status and launches nothing.  kvc_last_error() then
 *    gives a one-line reason (thread-local).
 *  - Errors that only the device can see (a gather index out of range, a
 *    cu_seqlens entry that is not monotone or a sequence shorter than the
 *    window) are reported by OR-ing bits into the optional device word
 *    `dev_err` (int32, may be NULL); affected outputs are written as zeros /
 *    -1 instead of reading out of bounds.  Bits: KVC_DEV_ERR_*.
 *  - Sizes: head_dim in {64, 128}; G*w (window rows per KV head) <= 256;
 *    token counts < 2^31.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVC_ABI_VERSION 1

typedef enum kvc_status {
  KVC_OK = 0,
  KVC_ERR_INVALID_ARG = 1, /* bad pointer, size, stride or alignment */
  KVC_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96) */
  KVC_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  KVC_ERR_WORKSPACE = 4    /* ws NULL/too small/misaligned (256 B) */
} kvc_status;

/* Device-side error bits (OR-ed into *dev_err when dev_err != NULL). */
#define KVC_DEV_ERR_INDEX 1   /* gather index outside [-1, n) */
#define KVC_DEV_ERR_SEQLENS 2 /* cu_seqlens malformed (not monotone, past the total) or a sequence shorter than w */
#define KVC_DEV_ERR_TIMEOUT 4 /* an internal pipeline wait hit its bound (a bug): outputs invalid */
#define KVC_DEV_ERR_ORDER 8   /* kvc_pivot_update: a layer folded in out of order */

/* Scoring geometry shared by the score entry points. */
typedef struct kvc_score_params {
  int32_t num_heads;    /* H: query heads */
  int32_t num_kv_heads; /* Hkv: KV heads; H % Hkv == 0, G = H / Hkv */
  int32_t head_dim;     /* d in {64, 128} */
  int32_t window;       /* w >= 1: observation-window queries (the last w tokens) */
  float scale;          /* softmax scale applied to q.k (usually 1/sqrt(d)) */
} kvc_score_params;

/* Version / diagnostics -------------------------------------------------- */

/* KVC_ABI_VERSION of the loaded library. */
int32_t kvc_abi_version(void);

/* Static string for a status code. */
const char* kvc_status_string(kvc_status s);

/* Reason of the last non-OK status returned on the calling thread ("" if none). */
const char* kvc_last_error(void);

/* Number of kernels this library has launched in this process (all threads). */
int64_t kvc_launch_count(void);

/* Scoring ---------------------------------------------------------------- */

/*
 * Workspace bytes needed by kvc_score (batch = 1, total_tokens = n) or
 * kvc_score_varlen (batch = B, total_tokens = packed token count).
 */
kvc_status kvc_score_workspace_size(const kvc_score_params* p, int32_t batch,
                                    int64_t total_tokens, size_t* bytes);

/*
 * Window-attention aggregate of one sequence  [FastKV 2.A; FastKV abstract
 * (GQA-aware); StructKV 2.A for `accum`].
 *
 * For KV head g, query head h of its group (h / G == g), window row i
 * (position n - w + i) and key j <= n - w + i:
 *     P[h, i, j] = softmax_j( scale * q[i, h, :] . k[j, g, :] )
 *     scores[g * n + j] = sum_{h in g} sum_{i : j <= n - w + i} P[h, i, j]
 * (keys after a window row's own position are masked: causal inside the
 * window; every prefix key is visible to every window row.)
 *
 *  q_win  [w][H][d] bf16, element (i, h, c) at q_win[i*q_stride_w + h*q_stride_h + c]
 *  k      [n][Hkv][d] bf16, element (j, g, c) at k[j*k_stride_n + g*k_stride_h + c]
 *  n      context tokens, w <= n < 2^31
 *  scores [Hkv][n] fp32 out, contiguous
 *  tsp    [n] fp32 out or NULL: tsp[j] = sum_g scores[g*n + j] (TSP aggregate)
 *  accum  [Hkv][n] fp32 in/out or NULL: accum += scores (cross-layer C_global)
 *  ws     workspace of kvc_score_workspace_size(p, 1, n) bytes, 256-B aligned
 *  dev_err device int32 or NULL (KVC_DEV_ERR_TIMEOUT only)
 * Summation is in fp32 from bf16 products; results are deterministic.
 */
kvc_status kvc_score(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h,
                     const uint16_t* k, int64_t k_stride_n, int64_t k_stride_h, int64_t n,
                     const kvc_score_params* p, float* scores, float* tsp, float* accum,
                     void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/*
 * kvc_score with the window rows' softmax normalisers supplied by the
 * caller  [FastKV 2.A: the TSP layer runs full attention over the prompt, so
 * every window query's normaliser already exists when the token scores are
 * formed; the softmax definition then gives each probability from its logit
 * and that normaliser alone].
 *
 *  lse  fp32, element (i, h) at lse[i*lse_stride_w + h*lse_stride_h]:
 *       ln sum_{j <= n - w + i} exp(scale * q[i, h, :] . k[j, g, :]), the
 *       natural-log log-sum-exp that a causal prefill attention returns for
 *       the query at position n - w + i (e.g. its [H][seqlen] output viewed
 *       at columns n - w .. n - 1: lse_stride_w = 1, lse_stride_h = seqlen).
 *       Finite values; strides >= 0.
 *     scores[g * n + j] = sum_{h in g} sum_{i : j <= n - w + i}
 *                         exp(scale * q[i, h, :] . k[j, g, :] - lse[i, h])
 *  which equals kvc_score's result when lse is the true log-sum-exp.  Only
 *  the second pass over K runs (one read of K instead of two).  Every other
 *  argument, the workspace (kvc_score_workspace_size(p, 1, n)) and the
 *  error behaviour are those of kvc_score.
 */
kvc_status kvc_score_lse(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h,
                         const uint16_t* k, int64_t k_stride_n, int64_t k_stride_h, int64_t n,
                         const kvc_score_params* p, const float* lse, int64_t lse_stride_w,
                         int64_t lse_stride_h, float* scores, float* tsp, float* accum, void* ws,
                         size_t ws_bytes, int32_t* dev_err, void* stream);

/*
 * Ragged batch version of kvc_score.  Sequence b occupies packed tokens
 * [cu_seqlens[b], cu_seqlens[b+1]); its window is its own last w tokens.
 *  q_win       [B][w][H][d] bf16 (q_stride_b, q_stride_w, q_stride_h)
 *  k           [total][Hkv][d] bf16, packed
 *  cu_seqlens  DEVICE int32 [B+1], cu_seqlens[0] == 0, cu_seqlens[B] == total
 *  batch       1..1024
 *  max_seqlen  an upper bound of the longest sequence (host value)
 *  scores      [Hkv][total] fp32 out (packed like k); tsp [total]; accum [Hkv][total]
 *  dev_err     KVC_DEV_ERR_SEQLENS if cu_seqlens is malformed or a sequence
 *              is shorter than w (that sequence's scores are left zero)
 */
kvc_status kvc_score_varlen(const uint16_t* q_win, int64_t q_stride_b, int64_t q_stride_w,
                            int64_t q_stride_h, const uint16_t* k, int64_t k_stride_n,
                            int64_t k_stride_h, const int32_t* cu_seqlens, int32_t batch,
                            int64_t total, int64_t max_seqlen, const kvc_score_params* p,
                            float* scores, float* tsp, float* accum, void* ws, size_t ws_bytes,
                            int32_t* dev_err, void* stream);

/*
 * kvc_score for callers that cannot allocate.  The paper has no counterpart:
 * this is a deployment variant of kvc_score, same arguments minus the
 * workspace, same results.
 *
 * Some callers cannot hand the library a workspace: an operator running
 * inside another runtime's plugin interface that offers no scratch buffer,
 * or a serving loop that must not call cudaMalloc once it is running
 * (cudaMalloc can synchronise the device and stall every other stream).
 * This entry point takes its scratch from a static device array of
 * KVC_NOALLOC_SCRATCH_BYTES inside the library instead, and itself calls no
 * cudaMalloc, cudaFree or other allocating routine.  The array exists on
 * every GPU that loads the library and is held until the process exits.
 *  - Size limit: a call whose scratch need (kvc_score_workspace_size(p, 1, n))
 *    exceeds KVC_NOALLOC_SCRATCH_BYTES is rejected with KVC_ERR_WORKSPACE and
 *    launches nothing (8 KV heads x 128 window rows fit up to ~330K tokens).
 *  - First call on a device: it looks up (once per device, with that device
 *    current) the device address of the array.  Make the first call on each
 *    device before any stream capture.  A device reset (cudaDeviceReset)
 *    ends the context the address belongs to; the next call then looks it
 *    up again, so after a reset, too, make one call before any capture.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    previous call's contents (nothing in it needs to start at zero: each
 *    call writes every entry it later reads).  Calls that may overlap on the
 *    GPU -- on different streams, or from different threads -- race on the
 *    array and give wrong results; serialise them (one stream).
 */
#define KVC_NOALLOC_SCRATCH_BYTES (8u << 20)
kvc_status kvc_score_noalloc(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h,
                             const uint16_t* k, int64_t k_stride_n, int64_t k_stride_h, int64_t n,
                             const kvc_score_params* p, float* scores, float* tsp, float* accum,
                             int32_t* dev_err, void* stream);

/* Selection -------------------------------------------------------------- */

/* Workspace bytes for kvc_select_topk(_varlen) with `out_rows` ranking rows. */
kvc_status kvc_select_workspace_size(int32_t out_rows, int32_t batch, int64_t total_tokens,
                                     size_t* bytes);

/*
 * Top-k that always keeps the window  [FastKV 2.A: the window tokens go
 * forward with the selected ones; FastKV 2.B: the TSP rate and the KV
 * retention rate are two independent budgets over the same scores].
 *
 * Output row o ranks  R_o[j] = sum_{r = o*row_group}^{o*row_group+row_group-1} scores[r*row_stride + j]
 * (row_group = 1: one set per KV head; row_group = Hkv: one TSP set over all
 * heads).  With L = n - w prefix positions and h = pool_kernel / 2:
 *     S_o[j] = (1/pool_kernel) * sum_{t=-h}^{h} R_o[j + t],  R_o = 0 outside [0, L)
 * The output is the k - w prefix positions with the largest S (equal S: the
 * lower position wins) together with the window n-w..n-1, in ascending
 * order.  If k >= n all n positions are output.
 *  scores     [rows][row_stride] fp32; rows % row_group == 0
 *  pool_kernel odd >= 1 (1 = no pooling)
 *  k          budget including the window, k >= w
 *  idx        [rows/row_group][idx_row_stride] int32 out; the first min(k, n)
 *             entries of each row are written
 *  pooled     [rows/row_group][n - w] fp32 out or NULL: the ranking scores S
 *  ws         kvc_select_workspace_size(rows/row_group, 1, n) bytes
 */
kvc_status kvc_select_topk(const float* scores, int32_t rows, int64_t row_stride,
                           int32_t row_group, int64_t n, int32_t window, int32_t pool_kernel,
                           int64_t k, int32_t* idx, int64_t idx_row_stride, float* pooled,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Ragged batch version of kvc_select_topk.  Row r of sequence b is
 * scores[r*row_stride + cu_seqlens[b] .. + len_b).  For each sequence and
 * output row, min(k, len_b) LOCAL positions (0-based within the sequence)
 * are written to idx[(b*out_rows + o)*k ...] and the rest of the k entries
 * are set to -1.  counts [B] int32 out (or NULL) receives min(k, len_b).
 * max_seqlen must bound every sequence length: a longer sequence is not
 * ranked (its row is -1, counts 0) and sets KVC_DEV_ERR_SEQLENS.
 */
kvc_status kvc_select_topk_varlen(const float* scores, int32_t rows, int64_t row_stride,
                                  int32_t row_group, const int32_t* cu_seqlens, int32_t batch,
                                  int64_t total, int64_t max_seqlen, int32_t window,
                                  int32_t pool_kernel, int64_t k, int32_t* idx, int32_t* counts,
                                  void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Gathers ---------------------------------------------------------------- */

/*
 * Compacted KV cache  [FastKV 2.B: entries retained per layer; FastKV
 * abstract: one set per KV head].  Bit copy:
 *     k_out[(g*kk + r)*d + c] = k[idx[g*idx_row_stride + r]*stride_n + g*stride_h + c]
 * and the same for v -> v_out (v / v_out may both be NULL).
 *  idx_row_stride 0 broadcasts one index row to every KV head.
 *  An index of -1 writes a zero row (padding); any other index outside
 *  [0, n) writes a zero row and sets KVC_DEV_ERR_INDEX.
 *  k_out, v_out [Hkv][kk][d] contiguous, 16-byte aligned.
 */
kvc_status kvc_gather_kv(const uint16_t* k, const uint16_t* v, int64_t stride_n, int64_t stride_h,
                         int64_t n, int32_t num_kv_heads, int32_t head_dim, const int32_t* idx,
                         int64_t idx_row_stride, int64_t kk, uint16_t* k_out, uint16_t* v_out,
                         int32_t* dev_err, void* stream);

/*
 * Ragged batch version: idx [B][Hkv][kk] holds LOCAL positions (as written
 * by kvc_select_topk_varlen, -1 padded); source row = cu_seqlens[b] + idx.
 * Outputs [B][Hkv][kk][d].  An index >= len_b sets KVC_DEV_ERR_INDEX.
 */
kvc_status kvc_gather_kv_varlen(const uint16_t* k, const uint16_t* v, int64_t stride_n,
                                int64_t stride_h, const int32_t* cu_seqlens, int32_t batch,
                                int64_t total, int32_t num_kv_heads, int32_t head_dim,
                                const int32_t* idx, int64_t kk, uint16_t* k_out, uint16_t* v_out,
                                int32_t* dev_err, void* stream);

/*
 * Token-Selective Propagation of hidden states  [FastKV 2.A: only the
 * selected tokens' states (plus the window) go on to the later layers].
 *     out[r*hidden + c] = x[idx[r]*stride_n + c]
 *  x [n][hidden] bf16 (stride_n >= hidden), hidden % 8 == 0, 16-B aligned
 *  out [kk][hidden] contiguous; idx -1 -> zero row; out of range -> zero row
 *  and KVC_DEV_ERR_INDEX.
 */
kvc_status kvc_gather_hidden(const uint16_t* x, int64_t stride_n, int64_t n, int64_t hidden,
                             const int32_t* idx, int64_t kk, uint16_t* out, int32_t* dev_err,
                             void* stream);

/* Decode over the compacted cache ---------------------------------------- */

/* Workspace bytes for kvc_decode_attention (host only). */
kvc_status kvc_decode_workspace_size(int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int64_t kk,
                                     size_t* bytes);

/*
 * Attention of one decode query per query head over the compacted cache
 * [FastKV 2.B: the retained entries of every KV head are the cache the later
 * decoding steps read; FastKV 1: decoding is bound by reading that cache].
 * For query head h of KV head g = h / G (G = num_heads / num_kv_heads) and
 * the kk retained entries of g:
 *     s_j = scale * q[h, :] . k_c[g, j, :]
 *     out[h, :] = sum_j exp(s_j - max s) v_c[g, j, :] / sum_j exp(s_j - max s)
 * every retained entry visible (the decode query follows all of them).
 *  q        [H][d] bf16, row h at q + h * q_stride_h (q_stride_h >= d)
 *  k_c, v_c [Hkv][kk][d] bf16, contiguous (as kvc_gather_kv writes them),
 *           16-byte aligned; kk >= 1, kk * Hkv < 2^31
 *  out      [H][d] fp32, contiguous, 16-byte aligned
 *  ws       kvc_decode_workspace_size(H, Hkv, d, kk) bytes, 256-B aligned,
 *           ZERO-FILLED before its first use: it starts with one counter per
 *           KV head (chunks of that head done), which every call returns to
 *           zero, also when a wait timed out; one call at a time per workspace
 *  dev_err  device int32 or NULL (KVC_DEV_ERR_TIMEOUT only)
 * head_dim in {64, 128}; at most 16 query heads per KV head.  fp32
 * accumulation from the bf16 values; deterministic.  At head_dim 128 with up
 * to 8 query heads per KV head both contractions run on the tensor cores
 * (the probabilities enter the second one as two bf16 terms, hi + lo, good
 * to ~2^-17 of each) in one launch; otherwise on the CUDA cores, with a
 * second launch that merges the chunk partials.
 */
kvc_status kvc_decode_attention(const uint16_t* q, int64_t q_stride_h, const uint16_t* k_c, const uint16_t* v_c,
                                int64_t kk, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                                float* out, void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* Causal prefill attention with the rows' log-sum-exp ------------------- */

/*
 * Causal attention of one sequence over itself, returning every query row's
 * log-sum-exp  [FastKV (gist.science 2502.01068) 1: during prefill every
 * layer runs full attention over the prompt; 2.A: at the TSP layer this is
 * the attention whose window rows' normalisers the token scores use --
 * kvc_score_lse takes lse[n - w .. n) and reads K once; FastKV abstract:
 * grouped-query heads, h reads KV head h / G].  Query i sees keys j <= i:
 *     s_ij     = scale * q[i, h, :] . k[j, g, :]
 *     lse[i,h] = ln sum_{j <= i} exp(s_ij)
 *     out[i,h] = sum_{j <= i} exp(s_ij - lse[i,h]) v[j, g, :]
 * The same call is the attention of the later layers over the TSP-propagated
 * tokens (their positions ascend, so the causal order carries over).
 *  q        [n][H][d] bf16, contiguous, 16-byte aligned
 *  k, v     [n][Hkv][d] bf16, contiguous, 16-byte aligned
 *  out      [n][H][d] bf16 out, 16-byte aligned, or NULL (log-sum-exp only)
 *  lse      [n][H] fp32 out, or NULL
 *  dev_err  device int32 or NULL (KVC_DEV_ERR_TIMEOUT only)
 * head_dim 128; 1 <= n < 2^31.  Both contractions run on the tensor cores
 * (bf16 operands, fp32 accumulation); the probabilities enter the output
 * contraction as bf16 and the output is normalised by the sum of those
 * rounded probabilities (a convex combination of V rows: |error| <= ~6e-3 of
 * max |v|), while the log-sum-exp sums the fp32 probabilities in fp64
 * (relative error ~1e-6).  Deterministic.
 */
kvc_status kvc_prefill_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t n,
                                 int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                                 uint16_t* out, float* lse, int32_t* dev_err, void* stream);

/* Residual vector quantisation of retained rows --------------------------- */

/*
 * Residual VQ codes of retained K or V rows  [VQKV (gist.science 2603.16435)
 * 2: each cached vector becomes indices into codebooks; the first codebook
 * encodes the vector, each later one the residual the earlier ones leave].
 * For row t and stages s = 0 .. S-1 with codebooks C[s] ([M][d] each):
 *     r_0 = x[t]
 *     codes[t][s] = argmin_m ||r_s - C[s][m]||^2   (equal distances: lowest m)
 *     r_{s+1}     = r_s - C[s][codes[t][s]]
 *  x          [n][d] bf16, row t at x + t * x_stride (x_stride >= d); e.g. a
 *             compacted cache [Hkv][kk][d] as n = Hkv * kk rows
 *  codebooks  [S][M][d] fp32, contiguous, 16-byte aligned
 *  codes      [n][S] int32 out
 *  residual   [n][d] fp32 out or NULL: r_S, the row minus its reconstruction
 *  dev_err    device int32 or NULL (KVC_DEV_ERR_TIMEOUT only)
 * head_dim in {64, 128}; 16 <= M <= 256 with M % 16 == 0; 1 <= S <= 16.
 * The scores r . C[s][m] are a tf32 tensor-core contraction; every codeword
 * whose score lies within the bound of that rounding from the best one is
 * re-scored as an fp32 distance, so a code departs from the exact argmin only
 * where fp32 rounding of two nearly equal distances decides it.  The
 * residual is carried in fp32.
 */
kvc_status kvc_rvq_encode(const uint16_t* x, int64_t x_stride, int64_t n, int32_t head_dim, const float* codebooks,
                          int32_t stages, int32_t codebook_size, int32_t* codes, float* residual, int32_t* dev_err,
                          void* stream);

/* Statistics ------------------------------------------------------------- */

/* Workspace bytes for kvc_layer_stats over `rows` rows. */
kvc_status kvc_stats_workspace_size(int32_t rows, int64_t n, size_t* bytes);

/*
 * Per-row attention statistics  [StructKV 2.B: attention entropy,
 * sparsity and variance].  With a[j] = scores[r*row_stride + j] / mass_norm
 * over all n keys (mass_norm = w*G makes a sum to 1):
 *     out[3r+0] = -sum_j a[j] ln a[j]                (entropy, nats; 0 ln 0 = 0)
 *     out[3r+1] = sum of the ceil(n/100) largest a[j] (top-1% mass)
 *     out[3r+2] = (1/n) sum_j (a[j] - mean)^2         (population variance)
 */
kvc_status kvc_layer_stats(const float* scores, int32_t rows, int64_t row_stride, int64_t n,
                           float mass_norm, float* out, void* ws, size_t ws_bytes, void* stream);

/* Pivot detection ------------------------------------------------------- */

/* Device-resident state of the online pivot rule; zero it before layer 1. */
typedef struct kvc_pivot_state {
  double prev_entropy;  /* head-mean entropy of the last layer folded in */
  double prev_sparsity; /* head-mean top-1% mass of the last layer folded in */
  int32_t pivot;        /* 0 until decided, then the pivot layer (1-based) */
  int32_t layers_seen;  /* last layer folded in (0: none) */
} kvc_pivot_state;

/*
 * Dynamic pivot detection, online, one layer per call  [StructKV 2.B: the
 * per-layer attention entropy, sparsity and variance are watched; the pivot
 * is where the entropy falls sharply while the sparsity rises].  The page
 * fixes neither the per-layer statistic nor the threshold; the rule is:
 *     E_l = (1/rows) sum_g stats[3g + 0],  S_l = (1/rows) sum_g stats[3g + 1]
 * (float64, heads in order), and the pivot is the first layer l with
 * l_min <= l <= l_max, l >= 2, E_{l-1} - E_l >= tau * E_{l-1} and
 * S_l > S_{l-1}; if none qualifies, l_max (decided when layer l_max is
 * folded in).  Variance (stats[3g + 2]) is not part of the rule.
 *  stats  [rows][3] fp32 device: kvc_layer_stats' output for this layer
 *  layer  1-based; calls must come in order 1, 2, 3, ... on one state; a call
 *         whose layer is not state->layers_seen + 1 changes nothing and sets
 *         KVC_DEV_ERR_ORDER in dev_err
 *  state  device kvc_pivot_state (zeroed before layer 1); state->pivot holds
 *         the decision once made, later layers leave it unchanged
 *  tau >= 0, 1 <= l_min <= l_max
 * The decision stays on the device (no host synchronisation); read
 * state->pivot whenever convenient.
 */
kvc_status kvc_pivot_update(const float* stats, int32_t rows, int32_t layer, double tau, int32_t l_min,
                            int32_t l_max, kvc_pivot_state* state, int32_t* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
