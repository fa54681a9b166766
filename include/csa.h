/*
 * csa.h -- C ABI of the B200 (sm_100a) Compressed Sparse Attention (CSA) /
 * Heavily Compressed Attention (HCA) decode/prefill hot path.
 *
 * The method (DeepSeek-V4's million-token attention) is described in prose
 * on "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V",
 * section "The attention: compress, then select" (CSA and HCA bullets, and
 * the three details that follow them) and section "The skeleton, and what's
 * kept"; on "The Exchange Rates of a Million Tokens", section 3 ("Rate #2");
 * and on "DeepSeek V4: How It Made Million-Token AI", section "The Memory
 * Problem Nobody Wanted to Solve".  Each entry point below cites the passage
 * it realises and states the reading taken where the prose leaves a step
 * open.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers owned by the caller.  The library allocates
 *    no device memory; where scratch is needed the caller passes a workspace
 *    sized by the matching *_workspace_size query.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  A return of CSA_OK means the work was enqueued.
 *  - Tensors are dense, row-major, with the innermost dimension contiguous;
 *    every float tensor pointer must be 16-byte aligned.  `dt` gives the
 *    element type of every float tensor of the call (CSA_F32: float;
 *    CSA_BF16: bfloat16); lengths, positions and indices are int32.
 *  - Arithmetic is fp32 (bf16 inputs are multiplied on the tensor cores with
 *    fp32 accumulation); outputs are rounded to `dt`, nearest-even.
 *  - Arguments are validated on the host before anything is launched; a
 *    failing call returns a negative status, launches nothing and leaves a
 *    message for csa_last_error().  Values that live in device memory
 *    (lengths, positions, indices) are checked by the kernels: an invalid
 *    query writes a zero output row and raises the device error word, read
 *    (and cleared) by csa_check_device_error().  Nothing traps or exits.
 *  - Query positions: q_pos[b][tq] is the 0-based position t of query
 *    (b, tq) in sequence b; with q_pos == NULL, t = lens[b] - Tq + tq (the
 *    last Tq tokens: t = lens[b]-1 for a decode step).  Valid: 0 <= t <
 *    lens[b].
 *  - Visibility ("three details": an entry is formed only once its block is
 *    complete): a query at position t sees compressed entries
 *    i < floor((t+1)/m) (m = 4 for CSA), plus the window tokens
 *    max(0, t-window+1) .. t.
 *  - The one host-side resource the library creates is the second stream
 *    and two events of csa_hca_pair_decode, once per device.
 *
 * Entry points, by role
 *  - compression: csa_compress, hca_compress; at decode, one entry per
 *    completed block: csa_compress_step, hca_compress_step;
 *  - selection: csa_index_topk (= csa_index_scores + csa_topk), the
 *    allocation-free csa_index_topk_noalloc, and over MXFP4 indexer keys
 *    csa_quantize_mxfp4 + csa_index_topk_mxfp4;
 *  - attention: csa_attend, hca_attend (optional sink); with QK-norm and
 *    partial RoPE fused, csa_attend_rope, hca_attend_rope, and the cache
 *    pass csa_norm_rope; over FP8 entries, csa_quantize_fp8_entries +
 *    csa_attend_fp8, hca_attend_fp8;
 *  - scheduling: csa_hca_pair_decode, one decode step of a CSA + HCA layer
 *    pair as one call.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

/* status codes */
#define CSA_OK 0
#define CSA_ERR_NULL (-1)        /* a required pointer is NULL                    */
#define CSA_ERR_ALIGN (-2)       /* a tensor pointer is not 16-byte aligned       */
#define CSA_ERR_SHAPE (-3)       /* a size is out of range or inconsistent        */
#define CSA_ERR_DTYPE (-4)       /* dt is not a csa_dtype                         */
#define CSA_ERR_UNSUPPORTED (-5) /* outside the supported set (see each call)     */
#define CSA_ERR_WORKSPACE (-6)   /* workspace NULL or smaller than required       */
#define CSA_ERR_LAUNCH (-7)      /* a kernel launch failed                        */
#define CSA_ERR_DEVICE (-8)      /* a kernel found an invalid length/position     */
#define CSA_ERR_CUDA (-9)        /* another CUDA runtime call failed              */

/* Library version, (major << 16) | minor. */
CSA_API int csa_version(void);

/* Message describing the last failing call on this host thread ("" if none).
 * The string is owned by the library and valid until the next call on the
 * same thread. */
CSA_API const char *csa_last_error(void);

/* Synchronise `stream`, then return CSA_ERR_DEVICE if any kernel of this
 * library on the current device has raised the device error word since the
 * last check (clearing it), else CSA_OK.  CSA_ERR_CUDA if the stream itself
 * reports an error. */
CSA_API int csa_check_device_error(void *stream);

/* Per-kernel timing for performance analysis.  While enabled (per host
 * thread), every entry point records a pair of CUDA events on its stream
 * around each kernel it launches; this serialises those kernels.
 * csa_kernel_timing() waits for the last call's events, writes up to
 * max_kernels durations (ms, in launch order) and returns the number of
 * kernels that call launched (or a negative status). */
CSA_API int csa_set_kernel_timing(int enable);
CSA_API int csa_kernel_timing(float *ms, int max_kernels);

/* ------------------------------------------------------------------------
 * csa_compress -- CSA overlapping compressor (stride 4, 8-token windows).
 *
 * Anatomy page, CSA bullet: every 4 tokens become one cache entry, a learned
 * softmax-weighted pooling of their key-value vectors computed per channel
 * with learned position biases; each entry pools 8 tokens, its own block and
 * the one before.  Exchange Rates page, section 3: two series C^a / C^b
 * overlapping across block boundaries under one joint softmax.  Reading:
 * entry i pools tokens s = 4(i-1)+j, j = 0..7; slots j < 4 (block i-1) use
 * W_a, slots j >= 4 (block i) use W_b:
 *     z_s[c] = sum_e x_s[e] W[e][c] + bias8[j][c]
 *     out_i[c] = sum_s softmax_s(z_s[c]) x_s[c]
 * over the tokens with 0 <= s < lens[b] (others masked: entry 0 pools 4
 * tokens, a trailing partial block pools what exists).  The same call builds
 * the indexer-key cache from per-token indexer keys with their own params.
 *
 *   x      [B][n_max][d]   per-token key-value vectors (or indexer keys)
 *   lens   [B]             tokens of each sequence, 0 <= lens[b] <= n_max
 *   W_a,W_b [d][d]         logit weights, indexed [in][out]
 *   bias8  [8][d]          position biases
 *   out    [B][ceil(n_max/4)][d]; rows i >= ceil(lens[b]/4) are set to 0.
 * Supported: d in {32, 64, 128}; B >= 0, n_max >= 0.
 * ---------------------------------------------------------------------- */
CSA_API int csa_compress(const void *x, const int32_t *lens, int B, int n_max, int d, const void *W_a,
                 const void *W_b, const void *bias8, csa_dtype dt, void *out, void *stream);

/* ------------------------------------------------------------------------
 * hca_compress -- HCA compressor (stride m, no overlap).
 *
 * Anatomy page, HCA bullet: every 128 tokens become one entry, without
 * overlap; Million-Token AI page, "The Memory Problem": every 128 tokens
 * collapse into a single entry.  Reading: the same per-channel softmax
 * pooling with one series, block i = tokens m*i .. m*i+m-1:
 *     z_s[c] = sum_e x_s[e] W[e][c] + bias[s - m*i][c]
 *     out_i[c] = sum_s softmax_s(z_s[c]) x_s[c],   s < lens[b].
 *   x [B][n_max][d], W [d][d] ([in][out]), bias [m][d],
 *   out [B][ceil(n_max/m)][d]; rows i >= ceil(lens[b]/m) are set to 0.
 * Supported: d in {32, 64, 128}; 1 <= m <= 4096.
 * ---------------------------------------------------------------------- */
CSA_API int hca_compress(const void *x, const int32_t *lens, int B, int n_max, int d, int m,
                 const void *W, const void *bias, csa_dtype dt, void *out, void *stream);

/* ------------------------------------------------------------------------
 * csa_compress_step / hca_compress_step -- the compressors at decode: the
 * one entry that the newest token completes.
 *
 * Anatomy page, "The attention: compress, then select", first of the three
 * details: an entry is formed only once its block is complete (until then
 * its tokens are reached through the sliding window).  For each sequence b
 * with lens[b] > 0 and lens[b] a multiple of the stride (4, or m), the entry
 * i = lens[b]/stride - 1 is computed exactly as csa_compress / hca_compress
 * compute it (CSA: tokens 4i-4 .. 4i+3, entry 0 masked to its own block;
 * HCA: tokens m*i .. m*i+m-1) and written to cache[b][i]; every other row
 * and every other sequence is left untouched.  The tokens are read from the
 * ring the decode step keeps for the window: token s at row s % n_tok of
 * x_tok[b], which must hold the entry's tokens (n_tok >= min(8, lens[b])
 * for CSA, >= m for HCA; otherwise the device error word is set).
 *
 *   x_tok  [B][n_tok][d]   token ring (key-value vectors or indexer keys)
 *   lens   [B]             tokens of each sequence, newest included
 *   W_a, W_b, bias8 / W, bias   as for csa_compress / hca_compress
 *   cache  [B][nc_max][d]  the compressed cache, updated in place
 * Supported: d in {32, 64, 128}; 1 <= m <= 4096.
 * ---------------------------------------------------------------------- */
CSA_API int csa_compress_step(const void *x_tok, int n_tok, const int32_t *lens, int B, int d,
                              const void *W_a, const void *W_b, const void *bias8, csa_dtype dt,
                              void *cache, int nc_max, void *stream);

CSA_API int hca_compress_step(const void *x_tok, int n_tok, const int32_t *lens, int B, int d, int m,
                              const void *W, const void *bias, csa_dtype dt, void *cache, int nc_max,
                              void *stream);

/* ------------------------------------------------------------------------
 * csa_index_topk -- lightning-indexer scores and per-query top-k.
 *
 * Anatomy page, CSA bullet: a small lightning indexer (64 heads of 128
 * dimensions) ranks the compressed blocks for each query, and each query
 * attends only to the most relevant 1,024 (Flash: 512).  Exchange Rates
 * page, section 3: ReLU-gated dot products, then top-k.  Reading:
 *     I[t,i] = sum_h w[t,h] * max(0, q_idx[t,h,:] . k_idx[i,:])
 * for visible entries i < floor((t+1)/4).  The selected set S_t is the k
 * visible entries first in the order (score descending, index ascending):
 * ties go to the lower index and -0.0 ranks as +0.0.  If fewer than k are
 * visible, all are selected.
 *
 *   q_idx  [B][Tq][HI][dI]   indexer queries
 *   w      [B][Tq][HI]       per-head indexer weights
 *   k_idx  [B][nc_max][dI]   indexer-key cache (one key per entry)
 *   lens, q_pos              see conventions (q_pos may be NULL)
 *   idx_out [B][Tq][k] int32 S_t in ascending index order, padded with -1
 *   scores_out [B][Tq][nc_max] float, optional (NULL: kept in workspace):
 *                            I[t,i] for visible i, -inf for the rest
 *   workspace, ws_bytes      >= csa_index_topk_workspace_size(...), 16-byte
 *                            aligned; may be NULL when that size is 0 (it
 *                            holds the scores when scores_out is NULL)
 * Inputs must be finite.  Supported: (HI, dI) with HI in [1, 128] and dI in
 * {32, 64, 128}; 1 <= k <= 4096; nc_max <= 327680 (1.31M tokens).
 * ---------------------------------------------------------------------- */
CSA_API size_t csa_index_topk_workspace_size(int B, int Tq, int nc_max, int has_scores_out);

CSA_API int csa_index_topk(const void *q_idx, const void *w, const void *k_idx, const int32_t *lens,
                   const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max, int k,
                   csa_dtype dt, int32_t *idx_out, float *scores_out, void *workspace,
                   size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * csa_index_scores / csa_topk -- the two halves of csa_index_topk, for
 * callers that want the scores themselves or select over their own scores.
 * csa_index_topk(...) is exactly csa_index_scores into its scores buffer
 * followed by csa_topk on it.
 *
 * csa_index_scores writes scores_out [B][Tq][nc_max] (float, required):
 * I[t,i] for visible i < floor((t+1)/4), -inf for the rest.
 * csa_topk reads such a score array (visible entries must be finite) and
 * writes idx_out [B][Tq][k] with the selection rule of csa_index_topk.
 * Supported sets as for csa_index_topk.
 * ---------------------------------------------------------------------- */
CSA_API int csa_index_scores(const void *q_idx, const void *w, const void *k_idx,
                             const int32_t *lens, const int32_t *q_pos, int B, int Tq, int HI,
                             int dI, int nc_max, csa_dtype dt, float *scores_out, void *stream);

CSA_API int csa_topk(const float *scores, const int32_t *lens, const int32_t *q_pos, int B, int Tq,
                     int nc_max, int k, int32_t *idx_out, void *stream);

/* ------------------------------------------------------------------------
 * csa_index_topk_noalloc -- csa_index_topk without a caller workspace.
 *
 * The paper has no counterpart: this is a library convenience.  It serves
 * callers that may not allocate device memory during a call (a serving
 * engine whose memory pool already holds nearly all of the GPU, a custom
 * allocator that forbids allocations outside its pool, code where
 * cudaMalloc / cudaFree would synchronise the device).  It allocates
 * nothing: the scores live in a fixed 8 MiB array of device memory that the
 * library holds on every GPU that loads it, until the process exits.
 *
 * Arguments, supported sets, selection rule and idx_out as for
 * csa_index_topk with scores_out NULL.  In addition:
 *   - B * Tq * nc_max must not exceed csa_index_topk_noalloc_max_elems()
 *     (2,097,152, e.g. 8 decode queries at 1M tokens); larger calls fail
 *     with CSA_ERR_WORKSPACE and leave idx_out untouched.
 *   - The first call on a device looks up the array's device address (it
 *     may load the library's GPU code): make it before any stream capture.
 *   - Every call shares the array: calls that overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the
 *     caller.  Nothing left in it by an earlier call affects a result.
 * ---------------------------------------------------------------------- */
CSA_API size_t csa_index_topk_noalloc_max_elems(void);

CSA_API int csa_index_topk_noalloc(const void *q_idx, const void *w, const void *k_idx,
                                   const int32_t *lens, const int32_t *q_pos, int B, int Tq,
                                   int HI, int dI, int nc_max, int k, csa_dtype dt,
                                   int32_t *idx_out, void *stream);

/* ------------------------------------------------------------------------
 * csa_quantize_mxfp4 / csa_index_topk_mxfp4 -- the indexer over FP4 keys.
 *
 * Anatomy page, "The KV cache, recomputed": the indexer key is 128 numbers
 * in FP4 plus one byte of scale per 32 (68 bytes); CSA bullet: the lightning
 * indexer runs in FP4.  Format (the OCP microscaling layout): per block of 32
 * elements a power-of-two scale 2^X stored as the byte X + 127, X =
 * floor(log2 amax) - 2 (-127 for an all-zero block); per element an E2M1
 * code (sign bit 3; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6: nearest to
 * x / 2^X, ties to the even code, saturating at 6), two per byte, element 2j
 * in the low nibble.
 *   csa_quantize_mxfp4: k_idx [B][nc_max][dI] (bf16 or fp32) -> codes
 *     [B][nc_max][dI/2] uint8, scales [B][nc_max][dI/32] uint8.
 *   csa_index_topk_mxfp4: csa_index_topk with the key cache given as codes
 *     and scales; the scores are those of csa_index_topk over the
 *     dequantised keys (sign * magnitude * 2^X, each a bf16 number).  q_idx
 *     and w bf16; codes 16-byte aligned, scales 4-byte aligned; other
 *     arguments, workspace and selection as for csa_index_topk.
 * Supported: dI in {64, 128}; HI in [1, 128].
 * ---------------------------------------------------------------------- */
CSA_API int csa_quantize_mxfp4(const void *k_idx, int B, int nc_max, int dI, csa_dtype dt, uint8_t *codes,
                               uint8_t *scales, void *stream);

CSA_API int csa_index_topk_mxfp4(const void *q_idx, const void *w, const uint8_t *codes,
                                 const uint8_t *scales, const int32_t *lens, const int32_t *q_pos, int B,
                                 int Tq, int HI, int dI, int nc_max, int k, int32_t *idx_out,
                                 float *scores_out, void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * csa_attend -- sparse MQA attention over the selected entries + window.
 *
 * Anatomy page, "The skeleton": one key-value head is shared by every query
 * head, and each cached entry is both the key and the value.  CSA bullet:
 * each query attends to its selected entries.  First of the three details:
 * every CSA layer also attends to the last 128 tokens directly.  Reading:
 * for each head h, one joint softmax over
 *     { kv_c[b][i] : i in idx[b][tq][:], 0 <= i < floor((t+1)/4) }
 *   + { token s : max(0, t-window+1) <= s <= t }
 * with logits scale * (q[t,h] . v) and output sum softmax * v.  -1 padding
 * and indices that are not visible contribute nothing; a repeated index
 * contributes once per occurrence.
 *
 *   q      [B][Tq][H][d]      queries (already normalised / rotated)
 *   kv_c   [B][nc_max][d]     compressed KV cache
 *   kv_tok [B][n_tok][d]      window tokens, a ring: token s at row
 *                             s % n_tok; each query's window must fit
 *                             (min(window, t+1) <= n_tok)
 *   idx    [B][Tq][k] int32   selected entries (csa_index_topk output)
 *   scale  softmax scale; <= 0 means 1/sqrt(d)
 *   sink   [H] float or NULL: per-head sink logit s_h (second of the three
 *          details: a learned logit whose exponential joins the softmax
 *          denominator; it carries no value), in the units of the scaled
 *          logits: o = sum_j e^{l_j} v_j / (sum_j e^{l_j} + e^{s_h})
 *   out    [B][Tq][H][d]
 * Supported: d in {64, 128}; 1 <= H <= 128; 1 <= k <= 4096;
 * 1 <= window <= 4096.
 * ---------------------------------------------------------------------- */
CSA_API int csa_attend(const void *q, const void *kv_c, const void *kv_tok, int n_tok, const int32_t *idx,
               const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
               int k, int window, float scale, const float *sink, csa_dtype dt, void *out,
               void *stream);

/* ------------------------------------------------------------------------
 * hca_attend -- dense MQA attention over every visible HCA entry + window.
 *
 * Anatomy page, HCA bullet: queries attend to all compressed entries
 * densely (about 8,000 at a million tokens).  Same reading as csa_attend
 * with the selected set replaced by every visible entry i < floor((t+1)/m).
 *   kv_c [B][nc_max][d] HCA cache (nc_max may be 0), other arguments as for
 *   csa_attend.  Supported: d in {64, 128}; 1 <= H <= 128; 1 <= m <= 4096;
 *   1 <= window <= 4096; nc_max <= 65536.
 * ---------------------------------------------------------------------- */
CSA_API int hca_attend(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
               const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
               int m, int window, float scale, const float *sink, csa_dtype dt, void *out,
               void *stream);

/* ------------------------------------------------------------------------
 * QK-norm and partial RoPE.
 *
 * Anatomy page, "The attention: compress, then select", third of the three
 * details: queries and compressed entries are RMS-normalised per head, RoPE
 * turns only the last dims of each vector (64 of 512 there), and because
 * the cached entry is also the value, each attention output is turned back
 * by its own query's position, leaving only relative position.  Reading
 * (the pages give no formula), per head vector of d dims:
 *   CSA_NR_NORM    y = x / sqrt(mean(x^2) + eps) * gamma (gamma [d] in dt,
 *                  or NULL for ones)
 *   CSA_NR_ROTATE  after the norm, the adjacent pairs (d-r+2j, d-r+2j+1)
 *                  of the last r = rope_dim dims turned by the angle
 *                  p * rope_base^(-2j/r):  (a, b) -> (a cos - b sin,
 *                  a sin + b cos)   (textbook RoPE frequencies)
 *   CSA_NR_INVERSE with CSA_NR_ROTATE: the angle -p (undoes the rotation)
 * Positions: a query at t (the attention's decode rule), a window token at
 * its own position s, compressed entry i of stride m at m * i (the first
 * token of its own block).
 * ---------------------------------------------------------------------- */
#define CSA_NR_NORM 1
#define CSA_NR_ROTATE 2
#define CSA_NR_INVERSE 4

/* csa_norm_rope -- y = the flags' steps applied to x, per head vector.
 *   x, y   [R][G][d] in dt (y may be x: in place; 16-byte aligned)
 *   G      heads sharing one position (H for queries, 1 for caches)
 *   position of row group r, first rule that applies:
 *     pos    [R] int32 (explicit positions), else
 *     lens   [R / Tq] int32: lens[r / Tq] - Tq + r % Tq (decode queries:
 *            the attention's rule for q_pos == NULL), else
 *     pos_stride * (r % Tq) + pos_offset  (a cache [B][Tq = nc_max][d] of
 *            stride m: pos_stride = m; a token array [B][Tq = n][d]:
 *            pos_stride = 1)
 *   eps    >= 0; rope_dim even, 0 <= rope_dim <= d; rope_base > 0
 * Supported: d in {64, 128}; R * G < 2^31.  Caller owns every buffer;
 * nothing is allocated; asynchronous on `stream`.
 * ---------------------------------------------------------------------- */
CSA_API int csa_norm_rope(const void *x, void *y, long R, int G, int d, const int32_t *pos,
                          const int32_t *lens, int Tq, int pos_stride, int pos_offset, const void *gamma,
                          float eps, int rope_dim, float rope_base, int flags, csa_dtype dt, void *stream);

/* csa_attend_rope / hca_attend_rope -- csa_attend / hca_attend with the
 * query's QK-norm and RoPE and the output's inverse rotation fused into the
 * attention kernel:
 *   q' = csa_norm_rope(q) at the query's position t with `flags`
 *        (CSA_NR_NORM and/or CSA_NR_ROTATE; q_gamma, eps, rope_dim,
 *        rope_base as there), rounded to dt as a stored q' would be;
 *   o  = the attention of q' over the entries and window tokens, which the
 *        caller has normalised and rotated at their own positions (e.g. by
 *        csa_norm_rope when they are formed);
 *   out = o turned back by -t when CSA_NR_ROTATE is set.
 * Other arguments, supported sets and errors as csa_attend / hca_attend;
 * CSA_NR_INVERSE is rejected (CSA_ERR_UNSUPPORTED).
 * ---------------------------------------------------------------------- */
CSA_API int csa_attend_rope(const void *q, const void *kv_c, const void *kv_tok, int n_tok, const int32_t *idx,
                            const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
                            int k, int window, float scale, const float *sink, const void *q_gamma, float eps,
                            int rope_dim, float rope_base, int flags, csa_dtype dt, void *out, void *stream);
CSA_API int hca_attend_rope(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
                            const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
                            int m, int window, float scale, const float *sink, const void *q_gamma, float eps,
                            int rope_dim, float rope_base, int flags, csa_dtype dt, void *out, void *stream);

/* ------------------------------------------------------------------------
 * FP8 cache entries.
 *
 * Anatomy page, "The KV cache, recomputed": an entry keeps its 64 RoPE
 * dimensions in BF16 and the others in FP8 with one-byte UE8M0 scales (448
 * numbers and 7 scales: one per 64).  Reading: E4M3 codes (largest finite
 * 448); per block of 64 elements the scale 2^X with X = floor(log2 amax) - 8
 * clamped to [-127, 127] (-127 for an all-zero block), stored as the byte
 * X + 127; each element x / 2^X rounded to the nearest E4M3 value, ties to
 * even, saturating at 448.  The pages pack one record per entry; here the
 * entry is held in three planes:
 *   fp8    [rows][d - rope_dim]         E4M3 codes
 *   scales [rows][(d - rope_dim) / 64]  UE8M0 bytes
 *   rope   [rows][rope_dim]             the last rope_dim dims, unchanged
 * A dequantised element (code value * 2^X) is exact in bf16.
 * ---------------------------------------------------------------------- */

/* csa_quantize_fp8_entries -- kv [rows][d] (dt) into the three planes.
 * Supported: d - rope_dim a positive multiple of 64 (or 0), rope_dim even;
 * rows < 2^31.  kv and rope 16-byte aligned, fp8 2-byte aligned. */
CSA_API int csa_quantize_fp8_entries(const void *kv, long rows, int d, int rope_dim, csa_dtype dt, uint8_t *fp8,
                                     uint8_t *scales, void *rope, void *stream);

/* csa_attend_fp8 / hca_attend_fp8 -- csa_attend / hca_attend over a cache
 * of FP8 entries (planes of csa_quantize_fp8_entries with rows = B * nc_max,
 * d = 128, rope_dim = 64): the attention over the entries' dequantised
 * values.  The tensor-core kernel widens the codes in shared memory as the
 * tiles land.  Window tokens stay bf16.  Supported: bf16, d = 128,
 * nc_max % 4 == 0 (the scales are fetched in aligned 4-byte words); other
 * arguments as csa_attend / hca_attend.
 * ---------------------------------------------------------------------- */
CSA_API int csa_attend_fp8(const void *q, const uint8_t *kv_fp8, const uint8_t *kv_scales, const void *kv_rope,
                           const void *kv_tok, int n_tok, const int32_t *idx, const int32_t *lens,
                           const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max, int k, int window,
                           float scale, const float *sink, csa_dtype dt, void *out, void *stream);
CSA_API int hca_attend_fp8(const void *q, const uint8_t *kv_fp8, const uint8_t *kv_scales, const void *kv_rope,
                           const void *kv_tok, int n_tok, const int32_t *lens, const int32_t *q_pos, int B, int Tq,
                           int H, int d, int nc_max, int m, int window, float scale, const float *sink,
                           csa_dtype dt, void *out, void *stream);

/* ------------------------------------------------------------------------
 * csa_hca_pair_decode -- one decode step of an interleaved CSA + HCA layer
 * pair (Anatomy page, "The attention: compress, then select": V4
 * interleaves the two kinds of layer), both layers' queries given, issued as
 * one call:
 *   idx_out = csa_index_topk(q_idx, w, k_idx, ...)          (CSA, m = 4)
 *   out_csa = csa_attend(q_csa, kv_csa, kv_tok, idx_out, ...)
 *   out_hca = hca_attend(q_hca, kv_hca, kv_tok, ..., m)     (HCA)
 * with one query row per sequence (Tq = 1, decode positions lens[b] - 1),
 * bf16, default softmax scale, no sink.  The results are those of the three
 * calls.  Scheduling: the HCA attention shares nothing with the CSA layer,
 * so it runs on a second (library-owned, high-priority) stream forked from
 * and joined back to `stream` by events; the persistent CSA scoring kernel
 * is launched on all but min(B, SMs / 4) SMs so that the HCA rows run beside
 * it.  Capturable into a CUDA graph (fork and join are event edges).
 *   q_csa, q_hca [B][1][H][d]; q_idx [B][1][HI][dI]; w [B][1][HI];
 *   k_idx [B][nc_max][dI]; kv_csa [B][nc_max][d]; kv_hca [B][nh_max][d];
 *   kv_tok [B][n_tok][d] (the window ring both layers read);
 *   idx_out [B][1][k]; out_csa, out_hca [B][1][H][d];
 *   workspace >= csa_index_topk_workspace_size(B, 1, nc_max, 0) bytes.
 * Supported sets: those of the three calls.  The library creates its
 * second stream and two events once per device, on the first call (before
 * any capture).
 * ---------------------------------------------------------------------- */
CSA_API int csa_hca_pair_decode(const void *q_csa, const void *q_idx, const void *w, const void *k_idx,
                                const void *kv_csa, int nc_max, int HI, int dI, int k, const void *q_hca,
                                const void *kv_hca, int nh_max, int m, const void *kv_tok, int n_tok,
                                const int32_t *lens, int B, int H, int d, int window, int32_t *idx_out,
                                void *out_csa, void *out_hca, void *workspace, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_B200_H */
