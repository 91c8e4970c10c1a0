/* lrkv: low-rank latent KV cache with decode attention over the codes.
 *
 * C ABI of the CUDA library liblrkv.so (sm_100a).  Plain pointers and sizes
 * only.  Unless a comment says "host", every pointer is DEVICE memory owned
 * by the caller; the library keeps no state between calls and allocates no
 * memory.  Every call is asynchronous on the given stream (a cudaStream_t
 * passed as void*; NULL is the legacy default stream).  Arguments are
 * checked on the host before anything is launched: a bad argument returns a
 * negative status and launches nothing.  A failed launch returns
 * LRKV_ERR_CUDA.  Errors inside a kernel surface at the caller's next
 * synchronisation; kernels never trap.
 *
 * The method (pages: "Half the Memory, None of the Answers Lost" sections
 * 04, 05 and 08; the OjaKV article; the Palu and LowRAM abstracts):
 *  - each token's post-RoPE key k and value v (128 dims per KV head) are
 *    stored as r-dim codes c_k = P_k^T k and c_v = P_v^T v under a
 *    per-(layer, KV head) basis P in R^{128 x r};
 *  - the first token (sink) and a window of the W most recent tokens stay
 *    full-rank (OjaKV: first and most recent tokens kept as anchors); a
 *    token that leaves the window is compressed with the basis passed to
 *    the call that evicts it;
 *  - decode attention runs on the codes: q~ = P_k^T q, s_t = q~ . c_k,t *
 *    scale for latent tokens, s_a = q . k_a * scale for anchors, one softmax
 *    over both, o = P_v sum_t p_t c_v,t + sum_a p_a v_a;
 *  - the basis may be refreshed online by Oja's rule with periodic QR.
 */
#ifndef LRKV_H
#define LRKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
enum {
  LRKV_OK = 0,
  LRKV_ERR_ARG = -1,         /* null pointer, bad size, misaligned pointer  */
  LRKV_ERR_UNSUPPORTED = -2, /* head_dim != 128, rank not supported, ...    */
  LRKV_ERR_CAPACITY = -3,    /* appended tokens would overflow the pages    */
  LRKV_ERR_WORKSPACE = -4,   /* workspace smaller than the size query says  */
  LRKV_ERR_CUDA = -5         /* a CUDA runtime call or launch failed        */
};

/* Element type of K/V inputs, codes, anchors, q and o.  LRKV_BF16_Q8: K/V
 * inputs, anchors, q and o are bf16, and the latent codes are stored as
 * per-token int8 with one fp32 scale per (token, KV head, side): the Palu
 * abstract (low-rank codes are quantisation-friendly) and the LowRAM
 * abstract (low-rank compression composes with quantisation) combine the
 * two; the pages give no scheme, and this one is symmetric per token,
 * s = max_j |c_j| / 127 and q_j = round-half-even(c_j / s), decided in fp32.
 * Attention reads the dequantised codes q_j s. */
enum { LRKV_BF16 = 0, LRKV_F32 = 1, LRKV_BF16_Q8 = 2, LRKV_BF16_VA = 3 };

/* LRKV_BF16_VA: value amortisation (LowRAM abstract: within a head, values
 * are largely predictable from their keys; a light per-head predictor is
 * fitted at test time and residuals are stored only for the tokens it
 * reconstructs worst).  The pages give neither the predictor's form nor the
 * selection rule; here, per (sequence, KV head), a linear map A (rank_k x
 * rank_v, fp32) predicts the value code from the key code, c_v ~ A^T c_k,
 * fitted by least squares over the prompt's latent tokens, and each 64-token
 * page keeps the value residual c_v - A^T c_k of its LRKV_VA_KEEP tokens
 * with the largest residual norm (ties: the earlier token).  No value codes
 * are stored; attention reads A^T c_k (+ the kept residual).  A slab holds
 *   [rank_k / 8][64][8] bf16 key codes, [rank_v / 8][16][8] bf16 residuals,
 *   int32 [16] page row of each residual slot (-1 empty), fp32 [16] squared
 *   residual norm of each slot,
 * 128 * rank_k + 32 * rank_v + 128 bytes in all. */
#define LRKV_VA_KEEP 16

#define LRKV_HEAD_DIM 128
#define LRKV_PAGE_TOKENS 64    /* tokens per latent code page */
#define LRKV_FULL_RANK_TILE 32 /* tokens per full-rank anchor / dense tile */
#define LRKV_MAX_BATCH 1024

/* Chunk of a stored row: 16 bytes, i.e. CE = 8 bf16 or 4 fp32 elements.
 * Every stored block is chunk-major: for each 16-byte chunk index, the
 * chunks of all tokens of the block follow each other, so one bulk copy
 * moves a block and lane t reading chunk j of token t touches consecutive
 * 16-byte words.
 *
 * Latent code pool, one slab per (page, KV head) holding the key codes'
 * chunks first, then the value codes' chunks:
 *   codes[num_pages][num_kv_heads][(rank_k + rank_v) / CE][LRKV_PAGE_TOKENS][CE]
 * Latent token j of sequence b (the j-th token that left the window) lives
 * in page block_table[b * max_pages_per_seq + j / 64], row j % 64.
 * With LRKV_BF16_Q8 a chunk holds 16 int8 codes and the slab ends with the
 * scales: [(rank_k + rank_v) / 16][64][16] int8, then [64][2] fp32 (key
 * scale, value scale per token); one slab is 64 * (rank_k + rank_v) + 512
 * bytes, and both ranks must be multiples of 16.
 *
 * Anchors (full-rank sink + window ring), chunk-major tiles of 32 slots with
 * the key's 128 dims first, then the value's:
 *   anchors[batch][num_kv_heads][anchor_tiles][256 / CE][32][CE]
 * with anchor_tiles = ceil((n_sink + window) / 32).  Slot 0 holds the sink
 * when n_sink == 1; token t >= n_sink of the window sits in slot
 * n_sink + (t - n_sink) % window.  The valid slots of a sequence of L tokens
 * are the first min(L, n_sink) + min(L - sink, window) slots.
 *
 * The block table may scatter pages over the pool in any order.  Entries
 * out of [0, num_pages) are never dereferenced: writes to them are skipped
 * and decode and re-basing set error word 2.  lrkv_compress and lrkv_rebase
 * write pages, so two entries naming one page must not both be written.
 *
 * seq_len[b] counts the tokens appended to sequence b so far; the library
 * advances it.  append_counter[b] is scratch the append kernels use to
 * advance seq_len when num_kv_heads > 8 (up to 8 the CTAs of a sequence
 * form a thread-block cluster and need no counter): zero it once when the
 * cache is created; every completed lrkv_compress leaves it zero again. */
typedef struct lrkv_cache {
  int32_t batch;             /* B, 1..LRKV_MAX_BATCH                       */
  int32_t num_kv_heads;      /* H_kv                                       */
  int32_t head_dim;          /* must be 128                                */
  int32_t rank_k, rank_v;    /* 8..128, multiples of CE (16 for Q8)        */
  int32_t dtype;             /* LRKV_BF16, LRKV_F32 or LRKV_BF16_Q8        */
  int32_t n_sink;            /* 0 or 1                                     */
  int32_t window;            /* W >= 0 full-rank recent tokens             */
  int32_t num_pages;         /* pages in the code pool                     */
  int32_t max_pages_per_seq; /* row length of block_table                  */
  void *codes;               /* code pool, layout above                    */
  const int32_t *block_table;/* [batch][max_pages_per_seq] page ids        */
  void *anchors;             /* anchor tiles (may be NULL when n_sink+W==0)*/
  int32_t *seq_len;          /* [batch] tokens appended so far             */
  int32_t *append_counter;   /* [batch] zero-initialised scratch           */
} lrkv_cache;

/* Append new tokens to every sequence and compress the tokens that become
 * latent ("store the small r-dim codes", Half the Memory, section 04;
 * anchors and window: OjaKV article).
 *   n_tokens : rows available per sequence in k and v.
 *   n_new    : optional device [batch] counts; sequence b appends
 *              min(n_new[b], n_tokens) tokens.  NULL: every sequence appends
 *              n_tokens tokens.
 *   k, v   : post-RoPE rows in the cache dtype; token i of (b, h) starts at
 *            k + b*seq_stride + h*head_stride + i*128 (element strides).
 *   P_k    : fp32 basis [Bp][H_kv][128][rank_k] (row-major 128 x r per head);
 *            sequence b uses P_k + b*basis_batch_stride (0 = shared by all).
 *   P_v    : the same for values with rank_v.
 *   Alignment: k, v, P_k and P_v 16-byte aligned; seq_stride and
 *            head_stride multiples of 8 elements (bf16) or 4 (fp32);
 *            basis_batch_stride a multiple of 4 (LRKV_ERR_ARG otherwise).
 * The sink, window slots and codes of each sequence are written; seq_len is
 * advanced by n_tokens.  Returns LRKV_ERR_CAPACITY only when the host can see
 * the overflow (n_tokens larger than the page capacity); the kernels skip
 * (and never write) code rows beyond max_pages_per_seq pages. */
int lrkv_compress(const lrkv_cache *cache, const void *k, const void *v,
                  int32_t n_tokens, const int32_t *n_new, int64_t seq_stride,
                  int64_t head_stride,
                  const float *P_k, const float *P_v,
                  int64_t basis_batch_stride, void *stream);

/* The same append for a value-amortised cache (LRKV_BF16_VA) whose
 * predictors A [batch][num_kv_heads][rank_k][rank_v] (fp32, 16-byte
 * aligned, as lrkv_amortise wrote them) exist: key codes are stored as by
 * lrkv_compress, and the value residual e = P_v^T v - A^T c_k of each token
 * that becomes latent enters its page's residual slots when it is among the
 * page's LRKV_VA_KEEP largest so far (ties: the earlier token; a token that
 * starts a page clears the page's slots first).  lrkv_compress on such a
 * cache stores the key codes only (use it for the prompt, before
 * lrkv_amortise).  LRKV_ERR_UNSUPPORTED for other caches. */
int lrkv_compress_amortised(const lrkv_cache *cache, const void *k, const void *v,
                            int32_t n_tokens, const int32_t *n_new, int64_t seq_stride,
                            int64_t head_stride, const float *P_k, const float *P_v,
                            int64_t basis_batch_stride, const float *A, void *stream);

/* Fit the value predictors of a value-amortised cache right after its
 * prompt was appended with lrkv_compress, and fill the residual slots of the
 * prompt's pages (LowRAM abstract: a per-head predictor fitted at test
 * time; residuals kept for the tokens it reconstructs worst).
 *   v : the same prompt value rows (bf16, layout and strides as given to
 *       lrkv_compress; n_tokens rows per sequence, read from token 0).
 *   A : output [batch][num_kv_heads][rank_k][rank_v] fp32: per unit the
 *       least-squares solution of C_k A = C_v over the prompt's latent
 *       tokens (normal equations by Cholesky in fp64 with a ridge of
 *       1e-12 trace(C_k^T C_k) / rank_k), C_k the stored key codes and
 *       C_v = V P_v computed from v (value codes are never stored).
 *   workspace : at least lrkv_amortise_workspace_bytes, 16-byte aligned;
 *       the first 4 bytes are an error word (2 = a block-table entry out of
 *       range).
 * Three stream-ordered launches (partial Gram matrices, solve, residual
 * slots).  LRKV_ERR_UNSUPPORTED for other caches. */
size_t lrkv_amortise_workspace_bytes(const lrkv_cache *cache);
int lrkv_amortise(const lrkv_cache *cache, const void *v, int32_t n_tokens,
                  int64_t seq_stride, int64_t head_stride, const float *P_v,
                  int64_t basis_batch_stride, float *A, void *workspace,
                  size_t workspace_bytes, void *stream);

/* Bytes of workspace lrkv_decode_attn needs on the current device.  It
 * holds the folded queries, the split-K partial records and (first 4 bytes)
 * an error word; zero the error word when the workspace is allocated. */
size_t lrkv_decode_workspace_bytes(const lrkv_cache *cache, int32_t num_q_heads);

/* Decode attention of one query per q head over the latent cache plus the
 * full-rank anchors (Half the Memory, section 08: attend directly against
 * the codes; q folded as q~ = P_k^T q, o = P_v sum p c_v + sum p_a v_a).
 * Three stream-ordered launches (q-fold, split-K, merge).
 *   q, o  : [batch][num_q_heads][128] in the cache dtype (q post-RoPE).
 *           q head h reads KV head h / (num_q_heads / num_kv_heads).
 *   scale : softmax scale applied to q . k (1/sqrt(128) for these models).
 *   P_v must be 16-byte aligned and basis_batch_stride a multiple of 4
 *           (LRKV_ERR_ARG otherwise).
 *   workspace : at least lrkv_decode_workspace_bytes, 16-byte aligned; calls sharing a
 *           workspace must be stream-ordered.  The error word is set (1 = a
 *           bounded wait timed out, 2 = a block-table entry out of range)
 *           and never cleared by the library.
 * A sequence with no tokens gets o = 0. */
int lrkv_decode_attn(const lrkv_cache *cache, const void *q, int32_t num_q_heads,
                     const float *P_k, const float *P_v,
                     int64_t basis_batch_stride, float scale, void *o,
                     void *workspace, size_t workspace_bytes, void *stream);

/* One decode step: append one token per sequence, then decode attention
 * with the appended token in the cache.  The same results as
 * lrkv_compress(cache, k, v, 1, NULL, ...) followed by lrkv_decode_attn
 * (the folded queries agree up to fp32 rounding order), with one launch
 * fewer: the append kernel, which stages each unit's basis anyway, also
 * folds that unit's queries q~ = P_k^T q into the workspace.
 *   k, v : [batch][num_kv_heads][1][128] post-RoPE (seq_stride, head_stride
 *          in elements, as for lrkv_compress); q, o, scale, workspace as for
 *          lrkv_decode_attn (the same workspace size).
 *   Plain caches only (LRKV_BF16, LRKV_F32; LRKV_ERR_UNSUPPORTED otherwise).
 *   Arguments are checked as by the two calls; on failure nothing is
 *   launched. */
int lrkv_decode_step(const lrkv_cache *cache, const void *k, const void *v,
                     int64_t seq_stride, int64_t head_stride, const void *q,
                     int32_t num_q_heads, const float *P_k, const float *P_v,
                     int64_t basis_batch_stride, float scale, void *o,
                     void *workspace, size_t workspace_bytes, void *stream);

/* Decode attention over a value-amortised cache: as lrkv_decode_attn, with
 * each latent token's value code read as A^T c_k plus its kept residual.
 * The split-K pass sums p c_k over the key codes and p e over the residual
 * slots; the merge applies A once per unit, o = P_v (A^T sum p c_k +
 * sum p e) / l + anchors.  A as for lrkv_compress_amortised;
 * rank_k + rank_v <= 128.  lrkv_decode_attn refuses these caches
 * (LRKV_ERR_UNSUPPORTED) and this call refuses other caches. */
int lrkv_decode_attn_amortised(const lrkv_cache *cache, const void *q, int32_t num_q_heads,
                               const float *P_k, const float *P_v,
                               int64_t basis_batch_stride, const float *A, float scale,
                               void *o, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Decode attention that allocates nothing and takes no workspace.  The
 * pages have no counterpart to this entry point: it exists for callers that
 * cannot allocate device memory or hand the library a buffer -- a plugin
 * inside a host framework that owns every allocation, or code on a path
 * where cudaMalloc's device synchronisation is not allowed.
 *   Same arguments and results as lrkv_decode_attn, minus the workspace.
 *   Scratch: a fixed array of LRKV_STATIC_WORKSPACE_BYTES compiled into the
 *     library, resident on every GPU that loads it until the process exits.
 *     Configurations needing more scratch than that (see
 *     lrkv_decode_workspace_bytes) return LRKV_ERR_WORKSPACE and launch
 *     nothing.
 *   The first call on a device (with that device current) looks up the
 *     array's device address once; make that first call before any stream
 *     capture.
 *   All calls share the one array: calls whose work overlaps on the GPU
 *     (other streams, other host threads) race and give wrong results;
 *     keep them ordered on one stream.  Each call clears the parts that must
 *     start at zero.  The error word is not reported by this entry point, so
 *     its outputs are unchecked: with a block-table entry out of range or a
 *     timed-out wait it still returns LRKV_OK and o holds wrong values.
 *     Callers that need that check use lrkv_decode_attn with a workspace.
 *   The stream must belong to the current device; a device reset while the
 *     library is loaded is not supported (the kept address goes stale).
 *   A configuration the regular entry point rejects returns the same
 *     status here (bad cache or heads, or LRKV_ERR_UNSUPPORTED). */
#define LRKV_STATIC_WORKSPACE_BYTES (4u << 20)
int lrkv_decode_attn_static(const lrkv_cache *cache, const void *q,
                            int32_t num_q_heads, const float *P_k,
                            const float *P_v, int64_t basis_batch_stride,
                            float scale, void *o, void *stream);

/* Oja subspace update of S independent bases, in place (OjaKV article:
 * online PCA with Oja's algorithm during prefill and periodically during
 * decode).  For each token x of stream s in order: y = P^T x,
 * P <- P + eta (x - P y) y^T; when (tokens_seen + i + 1) % qr_every == 0
 * (qr_every > 0) P is replaced by the Q of its QR with diag(R) > 0.
 *   P  : fp32 [S] bases of [128][rank], stream s at P + s*basis_stride.
 *   x  : tokens of stream s at x + s*x_stream_stride + i*128, dtype x_dtype.
 * tokens_seen is the host-side count of tokens this basis saw before. */
int lrkv_oja_update(float *P, int32_t num_streams, int32_t rank,
                    int64_t basis_stride, const void *x, int32_t x_dtype,
                    int64_t x_stream_stride, int32_t n_tokens, float eta,
                    int32_t qr_every, int64_t tokens_seen, void *stream);

/* Chunked form of the Oja update, for the prompt pass (OjaKV article: the
 * basis adapts comprehensively during prompt prefilling; done token by token
 * that pass is one long chain of dependent steps).  The tokens of each
 * stream are taken in chunks of `chunk` (1..64); within a chunk every token's
 * update uses the basis of the chunk's start, so a chunk is
 *   Y = X P,  Z = X - Y P^T,  P <- P + eta Z^T Y,
 * the sum of the rule's per-token updates with P frozen (chunk = 1 is the
 * sequential rule; the two differ by a term of order eta^2 * chunk per
 * chunk).  A chunk ends early where (tokens_seen + tokens so far) reaches a
 * multiple of qr_every, and P is then replaced by the Q of its QR with
 * diag(R) > 0.  Same arguments as lrkv_oja_update, plus chunk; rank <= 64
 * and a multiple of 8 (LRKV_ERR_UNSUPPORTED otherwise); x 16-byte aligned
 * with x_stream_stride a multiple of 16 bytes (LRKV_ERR_ARG otherwise). */
int lrkv_oja_update_chunked(float *P, int32_t num_streams, int32_t rank,
                            int64_t basis_stride, const void *x, int32_t x_dtype,
                            int64_t x_stream_stride, int32_t n_tokens, float eta,
                            int32_t qr_every, int64_t tokens_seen, int32_t chunk,
                            void *stream);

/* Replace each basis by the Q factor of its thin QR with diag(R) > 0. */
int lrkv_qr_orthonormalize(float *P, int32_t num_streams, int32_t rank,
                           int64_t basis_stride, void *stream);

/* Re-basing of the stored codes after the bases changed.  The OjaKV page
 * adapts the basis online (its question on online subspace adaptation) but
 * does not say what becomes of codes stored under the old basis.  Here a
 * stored code c stands for its rank-r reconstruction P_old c, and every
 * latent code of every sequence and KV head is replaced by that vector's
 * code under the new basis: c' = P_new^T (P_old c).  The sink and window
 * anchors are full-rank and untouched; the decode calls that follow take
 * P_new.
 *   P_k_old, P_k_new : fp32 [Bp][H_kv][128][rank_k], 16-byte aligned, the
 *       layout and basis_batch_stride of lrkv_compress (0: one basis shared
 *       by every sequence).  Both NULL to leave the key codes as they are.
 *   P_v_old, P_v_new : the same for the value codes.
 *   workspace : at least lrkv_rebase_workspace_bytes, 16-byte aligned; the
 *       first 4 bytes are an error word (2 = a block-table entry out of
 *       range) that the library sets and never clears; zero it when the
 *       workspace is allocated.
 * Two stream-ordered launches: the per-unit r x r products P_new^T P_old in
 * fp32, then one pass over the latent pages (read on the device from
 * seq_len and the block table, so it follows the appends queued before it)
 * that rounds each new code to the cache dtype once (LRKV_BF16_Q8 caches:
 * LRKV_ERR_UNSUPPORTED).  Pages are rewritten in
 * place per (sequence, page), so no two block-table entries may name the
 * same page (no shared-prefix aliasing): an aliased page would be re-based
 * twice, or by two CTAs at once.  Returns LRKV_ERR_ARG for a half-given
 * pair, a misaligned pointer or a short workspace. */
size_t lrkv_rebase_workspace_bytes(const lrkv_cache *cache);
int lrkv_rebase(const lrkv_cache *cache, const float *P_k_old, const float *P_k_new,
                const float *P_v_old, const float *P_v_new, int64_t basis_batch_stride,
                void *workspace, size_t workspace_bytes, void *stream);

/* Dense full-rank paged KV cache: the baseline the latent cache replaces
 * (Half the Memory, section 08 compares against the full cache).  One slab
 * per (page, KV head), key chunks then value chunks:
 *   kv_pages[num_pages][num_kv_heads][256 / CE][32][CE] (chunk-major),
 *   token t of sequence b in page block_table[b*max_pages_per_seq + t/32]. */
typedef struct lrkv_dense_cache {
  int32_t batch, num_kv_heads, head_dim, dtype;
  int32_t num_pages, max_pages_per_seq;
  void *kv_pages;
  const int32_t *block_table;
  int32_t *seq_len;
  int32_t *append_counter; /* [batch] zero-initialised scratch */
} lrkv_dense_cache;

/* Append tokens to the dense cache (same k/v/n_new conventions as
 * lrkv_compress) and advance seq_len. */
int lrkv_dense_append(const lrkv_dense_cache *cache, const void *k,
                      const void *v, int32_t n_tokens, const int32_t *n_new,
                      int64_t seq_stride, int64_t head_stride, void *stream);
/* Workspace of the dense decode; the same contract as above. */
size_t lrkv_dense_decode_workspace_bytes(const lrkv_dense_cache *cache,
                                         int32_t num_q_heads);
int lrkv_dense_decode_attn(const lrkv_dense_cache *cache, const void *q,
                           int32_t num_q_heads, float scale, void *o,
                           void *workspace, size_t workspace_bytes,
                           void *stream);

/* Static text for a status code. */
const char *lrkv_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int lrkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LRKV_H */
