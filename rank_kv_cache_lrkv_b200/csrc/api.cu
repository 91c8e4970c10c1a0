// C ABI entry points: host-side argument checks, then the launchers.
#include <limits.h>

#include "common.cuh"
#include "internal.h"

using namespace lrkv;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// Elements per 16-byte chunk of the K/V inputs, anchors, q and o.
int chunk_elems(int dtype) { return dtype == LRKV_F32 ? 4 : 8; }
// Code elements per 16-byte chunk of a latent page.
int code_chunk_elems(int dtype) { return dtype == LRKV_BF16_Q8 ? 16 : chunk_elems(dtype); }

int check_rank(int r, int dtype) {
  const int ce = code_chunk_elems(dtype);
  if (r < ce || r > kHeadDim || r % ce != 0) return LRKV_ERR_UNSUPPORTED;
  return LRKV_OK;
}

int check_cache(const lrkv_cache* c) {
  if (!c) return LRKV_ERR_ARG;
  if (c->dtype != LRKV_BF16 && c->dtype != LRKV_F32 && c->dtype != LRKV_BF16_Q8 &&
      c->dtype != LRKV_BF16_VA)
    return LRKV_ERR_UNSUPPORTED;
  if (c->head_dim != kHeadDim) return LRKV_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->batch > LRKV_MAX_BATCH || c->num_kv_heads < 1) return LRKV_ERR_ARG;
  int rc = check_rank(c->rank_k, c->dtype);
  if (rc == LRKV_OK) rc = check_rank(c->rank_v, c->dtype);
  if (rc != LRKV_OK) return rc;
  // value-amortised records hold rank_k + rank_v sums per head
  if (c->dtype == LRKV_BF16_VA && c->rank_k + c->rank_v > kHeadDim) return LRKV_ERR_UNSUPPORTED;
  if (c->n_sink < 0 || c->n_sink > 1 || c->window < 0 || c->window > (1 << 20)) return LRKV_ERR_ARG;
  if (c->num_pages < 1 || c->max_pages_per_seq < 1) return LRKV_ERR_ARG;
  if (!c->codes || !c->block_table || !c->seq_len || !c->append_counter) return LRKV_ERR_ARG;
  if (!aligned16(c->codes)) return LRKV_ERR_ARG;
  if (c->n_sink + c->window > 0 && (!c->anchors || !aligned16(c->anchors))) return LRKV_ERR_ARG;
  return LRKV_OK;
}

int check_dense(const lrkv_dense_cache* c) {
  if (!c) return LRKV_ERR_ARG;
  if (c->dtype != LRKV_BF16 && c->dtype != LRKV_F32) return LRKV_ERR_UNSUPPORTED;
  if (c->head_dim != kHeadDim) return LRKV_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->batch > LRKV_MAX_BATCH || c->num_kv_heads < 1) return LRKV_ERR_ARG;
  if (c->num_pages < 1 || c->max_pages_per_seq < 1) return LRKV_ERR_ARG;
  if (!c->kv_pages || !c->block_table || !c->seq_len || !c->append_counter) return LRKV_ERR_ARG;
  if (!aligned16(c->kv_pages)) return LRKV_ERR_ARG;
  return LRKV_OK;
}

int check_heads(int H_kv, int H_q) {
  if (H_q < 1 || H_q % H_kv != 0) return LRKV_ERR_ARG;
  const int G = H_q / H_kv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return LRKV_ERR_UNSUPPORTED;
  return LRKV_OK;
}

}  // namespace

namespace lrkv {
// Why lrkv_decode_workspace_bytes returned 0: the argument check's status, or
// the planning status (LRKV_ERR_UNSUPPORTED when the ring does not fit in
// shared memory, LRKV_ERR_CUDA when the device query failed).
int decode_plan_status(const lrkv_cache* cache, int H_q) {
  int rc = check_cache(cache);
  if (rc == LRKV_OK) rc = check_heads(cache->num_kv_heads, H_q);
  if (rc != LRKV_OK) return rc;
  return decode_plan_check(cache->batch, cache->num_kv_heads, H_q, cache->rank_k,
                           cache->rank_v, true, cache->n_sink + cache->window > 0,
                           cache->dtype);
}
}  // namespace lrkv

extern "C" {

int lrkv_version(void) { return 100; }

const char* lrkv_status_string(int s) {
  switch (s) {
    case LRKV_OK: return "ok";
    case LRKV_ERR_ARG: return "invalid argument";
    case LRKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case LRKV_ERR_CAPACITY: return "cache capacity exceeded";
    case LRKV_ERR_WORKSPACE: return "workspace too small";
    case LRKV_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

// The checks of lrkv_compress and lrkv_compress_amortised, then the launch.
static int compress_checked(const lrkv_cache* cache, const void* k, const void* v,
                            int32_t n_tokens, const int32_t* n_new, int64_t seq_stride,
                            int64_t head_stride, const float* P_k, const float* P_v,
                            int64_t basis_batch_stride, const float* A, void* stream) {
  int rc = check_cache(cache);
  if (rc != LRKV_OK) return rc;
  if (n_tokens < 0) return LRKV_ERR_ARG;
  if (n_tokens == 0) return LRKV_OK;
  if (!k || !v || !P_k || !P_v || basis_batch_stride < 0) return LRKV_ERR_ARG;
  // token rows are read in 16-byte chunks and the bases four floats at a time
  const int ce = chunk_elems(cache->dtype);
  if (!aligned16(k) || !aligned16(v) || seq_stride % ce != 0 || head_stride % ce != 0 ||
      !aligned16(P_k) || !aligned16(P_v) || basis_batch_stride % 4 != 0)
    return LRKV_ERR_ARG;
  const long long cap = (long long)cache->max_pages_per_seq * kLatPage + cache->n_sink + cache->window;
  if (n_tokens > cap) return LRKV_ERR_CAPACITY;
  return compress_launch(*cache, k, v, n_tokens, n_new, seq_stride, head_stride, P_k, P_v,
                         basis_batch_stride, static_cast<cudaStream_t>(stream), A);
}

int lrkv_compress(const lrkv_cache* cache, const void* k, const void* v, int32_t n_tokens,
                  const int32_t* n_new, int64_t seq_stride, int64_t head_stride, const float* P_k,
                  const float* P_v, int64_t basis_batch_stride, void* stream) {
  return compress_checked(cache, k, v, n_tokens, n_new, seq_stride, head_stride, P_k, P_v,
                          basis_batch_stride, nullptr, stream);
}

int lrkv_compress_amortised(const lrkv_cache* cache, const void* k, const void* v,
                            int32_t n_tokens, const int32_t* n_new, int64_t seq_stride,
                            int64_t head_stride, const float* P_k, const float* P_v,
                            int64_t basis_batch_stride, const float* A, void* stream) {
  if (!cache || cache->dtype != LRKV_BF16_VA) return cache ? LRKV_ERR_UNSUPPORTED : LRKV_ERR_ARG;
  if (!A) return LRKV_ERR_ARG;
  return compress_checked(cache, k, v, n_tokens, n_new, seq_stride, head_stride, P_k, P_v,
                          basis_batch_stride, A, stream);
}

size_t lrkv_amortise_workspace_bytes(const lrkv_cache* cache) {
  if (check_cache(cache) != LRKV_OK || cache->dtype != LRKV_BF16_VA) return 0;
  return amortise_workspace_bytes(cache->batch, cache->num_kv_heads, cache->rank_k,
                                  cache->rank_v);
}

int lrkv_amortise(const lrkv_cache* cache, const void* v, int32_t n_tokens, int64_t seq_stride,
                  int64_t head_stride, const float* P_v, int64_t basis_batch_stride, float* A,
                  void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_cache(cache);
  if (rc != LRKV_OK) return rc;
  if (cache->dtype != LRKV_BF16_VA) return LRKV_ERR_UNSUPPORTED;
  if (!v || !P_v || !A || !workspace || n_tokens < 1 || basis_batch_stride < 0 ||
      !aligned16(v) || !aligned16(P_v) || !aligned16(A) || !aligned16(workspace) ||
      seq_stride % 8 != 0 || head_stride % 8 != 0 || basis_batch_stride % 4 != 0)
    return LRKV_ERR_ARG;
  if (workspace_bytes < lrkv_amortise_workspace_bytes(cache)) return LRKV_ERR_WORKSPACE;
  return amortise_launch(*cache, v, n_tokens, seq_stride, head_stride, P_v, basis_batch_stride,
                         A, workspace, static_cast<cudaStream_t>(stream));
}

size_t lrkv_decode_workspace_bytes(const lrkv_cache* cache, int32_t num_q_heads) {
  if (check_cache(cache) != LRKV_OK || check_heads(cache->num_kv_heads, num_q_heads) != LRKV_OK)
    return 0;
  return decode_workspace_bytes(cache->batch, cache->num_kv_heads, num_q_heads, cache->rank_k,
                                cache->rank_v, true, cache->n_sink + cache->window > 0,
                                cache->dtype);
}

// The checks of the decode entry points; fills the launch description.
static int decode_setup(const lrkv_cache* cache, const void* q, int32_t num_q_heads,
                        const float* P_k, const float* P_v, int64_t basis_batch_stride,
                        const float* A, float scale, void* o, void* workspace,
                        size_t workspace_bytes, DecodeLaunch& L) {
  int rc = check_cache(cache);
  if (rc != LRKV_OK) return rc;
  if ((cache->dtype == LRKV_BF16_VA) != (A != nullptr)) return LRKV_ERR_UNSUPPORTED;
  if (A && !aligned16(A)) return LRKV_ERR_ARG;
  rc = check_heads(cache->num_kv_heads, num_q_heads);
  if (rc != LRKV_OK) return rc;
  if (!q || !o || !P_k || !P_v || !workspace || basis_batch_stride < 0) return LRKV_ERR_ARG;
  // the value basis is read four floats at a time
  if (!aligned16(workspace) || !aligned16(P_v) || basis_batch_stride % 4 != 0) return LRKV_ERR_ARG;
  L.B = cache->batch; L.H_kv = cache->num_kv_heads; L.H_q = num_q_heads; L.dtype = cache->dtype;
  L.seq_len = cache->seq_len; L.n_sink = cache->n_sink; L.W = cache->window;
  L.codes = cache->codes; L.bt_lat = cache->block_table;
  L.maxp_lat = cache->max_pages_per_seq; L.rk = cache->rank_k; L.rv = cache->rank_v;
  L.num_pages_lat = cache->num_pages;
  const bool has_fr = cache->n_sink + cache->window > 0;
  L.fr = has_fr ? cache->anchors : nullptr;
  L.bt_fr = nullptr;
  L.maxp_fr = (cache->n_sink + cache->window + kFrTile - 1) / kFrTile;
  L.num_pages_fr = 0;
  L.q = q; L.P_k = P_k; L.P_v = P_v; L.basis_bs = basis_batch_stride; L.scale = scale;
  L.o = o; L.ws = workspace; L.ws_bytes = workspace_bytes; L.A = A;
  return LRKV_OK;
}

static int decode_checked(const lrkv_cache* cache, const void* q, int32_t num_q_heads,
                          const float* P_k, const float* P_v, int64_t basis_batch_stride,
                          const float* A, float scale, void* o, void* workspace,
                          size_t workspace_bytes, void* stream) {
  DecodeLaunch L;
  const int rc = decode_setup(cache, q, num_q_heads, P_k, P_v, basis_batch_stride, A, scale, o,
                              workspace, workspace_bytes, L);
  if (rc != LRKV_OK) return rc;
  return decode_launch(L, static_cast<cudaStream_t>(stream));
}

int lrkv_decode_step(const lrkv_cache* cache, const void* k, const void* v, int64_t seq_stride,
                     int64_t head_stride, const void* q, int32_t num_q_heads, const float* P_k,
                     const float* P_v, int64_t basis_batch_stride, float scale, void* o,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache) return LRKV_ERR_ARG;
  int rc = check_cache(cache);
  if (rc != LRKV_OK) return rc;
  if (cache->dtype != LRKV_BF16 && cache->dtype != LRKV_F32) return LRKV_ERR_UNSUPPORTED;
  DecodeLaunch L;
  rc = decode_setup(cache, q, num_q_heads, P_k, P_v, basis_batch_stride, nullptr, scale, o,
                    workspace, workspace_bytes, L);
  if (rc != LRKV_OK) return rc;
  // the append's arguments, as lrkv_compress checks them for one token
  const int ce = chunk_elems(cache->dtype);
  if (!k || !v || !aligned16(k) || !aligned16(v) || seq_stride % ce != 0 ||
      head_stride % ce != 0 || !aligned16(P_k))
    return LRKV_ERR_ARG;
  StepFold f;
  rc = decode_fold_targets(L, &f.qlat, &f.qfr, &f.qscale);
  if (rc != LRKV_OK) return rc;
  f.q = q;
  f.H_q = num_q_heads;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = compress_launch(*cache, k, v, 1, nullptr, seq_stride, head_stride, P_k, P_v,
                       basis_batch_stride, st, nullptr, &f);
  if (rc != LRKV_OK) return rc;
  return decode_launch(L, st, true);
}

int lrkv_decode_attn(const lrkv_cache* cache, const void* q, int32_t num_q_heads,
                     const float* P_k, const float* P_v, int64_t basis_batch_stride, float scale,
                     void* o, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_checked(cache, q, num_q_heads, P_k, P_v, basis_batch_stride, nullptr, scale, o,
                        workspace, workspace_bytes, stream);
}

int lrkv_decode_attn_amortised(const lrkv_cache* cache, const void* q, int32_t num_q_heads,
                               const float* P_k, const float* P_v, int64_t basis_batch_stride,
                               const float* A, float scale, void* o, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!A) return LRKV_ERR_ARG;
  return decode_checked(cache, q, num_q_heads, P_k, P_v, basis_batch_stride, A, scale, o,
                        workspace, workspace_bytes, stream);
}

int lrkv_oja_update(float* P, int32_t num_streams, int32_t rank, int64_t basis_stride,
                    const void* x, int32_t x_dtype, int64_t x_stream_stride, int32_t n_tokens,
                    float eta, int32_t qr_every, int64_t tokens_seen, void* stream) {
  if (!P || num_streams < 1 || rank < 1 || rank > kHeadDim || n_tokens < 0 || qr_every < 0 ||
      tokens_seen < 0 || basis_stride < (int64_t)kHeadDim * rank)
    return LRKV_ERR_ARG;
  if (x_dtype != LRKV_BF16 && x_dtype != LRKV_F32) return LRKV_ERR_UNSUPPORTED;
  if (n_tokens > 0 && !x) return LRKV_ERR_ARG;
  if (n_tokens == 0) return LRKV_OK;
  return oja_launch(P, num_streams, rank, basis_stride, x, x_dtype, x_stream_stride, n_tokens,
                    eta, qr_every, tokens_seen, static_cast<cudaStream_t>(stream));
}

int lrkv_oja_update_chunked(float* P, int32_t num_streams, int32_t rank, int64_t basis_stride,
                            const void* x, int32_t x_dtype, int64_t x_stream_stride,
                            int32_t n_tokens, float eta, int32_t qr_every, int64_t tokens_seen,
                            int32_t chunk, void* stream) {
  if (!P || num_streams < 1 || rank < 1 || rank > kHeadDim || n_tokens < 0 || qr_every < 0 ||
      tokens_seen < 0 || basis_stride < (int64_t)kHeadDim * rank || chunk < 1 || chunk > 64)
    return LRKV_ERR_ARG;
  if (x_dtype != LRKV_BF16 && x_dtype != LRKV_F32) return LRKV_ERR_UNSUPPORTED;
  if (rank > 64 || rank % 8 != 0) return LRKV_ERR_UNSUPPORTED;
  if (n_tokens > 0 && !x) return LRKV_ERR_ARG;
  if (n_tokens == 0) return LRKV_OK;
  return oja_blocked_launch(P, num_streams, rank, basis_stride, x, x_dtype, x_stream_stride,
                            n_tokens, eta, qr_every, tokens_seen, chunk,
                            static_cast<cudaStream_t>(stream));
}

int lrkv_qr_orthonormalize(float* P, int32_t num_streams, int32_t rank, int64_t basis_stride,
                           void* stream) {
  if (!P || num_streams < 1 || rank < 1 || rank > kHeadDim ||
      basis_stride < (int64_t)kHeadDim * rank)
    return LRKV_ERR_ARG;
  return qr_launch(P, num_streams, rank, basis_stride, static_cast<cudaStream_t>(stream));
}

size_t lrkv_rebase_workspace_bytes(const lrkv_cache* cache) {
  if (check_cache(cache) != LRKV_OK) return 0;
  return rebase_workspace_bytes(cache->batch, cache->num_kv_heads, cache->rank_k, cache->rank_v);
}

int lrkv_rebase(const lrkv_cache* cache, const float* P_k_old, const float* P_k_new,
                const float* P_v_old, const float* P_v_new, int64_t basis_batch_stride,
                void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_cache(cache);
  if (rc != LRKV_OK) return rc;
  // a side is re-based when both of its bases are given
  if (!P_k_old != !P_k_new || !P_v_old != !P_v_new) return LRKV_ERR_ARG;
  if (!workspace || basis_batch_stride < 0 || basis_batch_stride % 4 != 0 ||
      !aligned16(workspace) || !aligned16(P_k_old) || !aligned16(P_k_new) ||
      !aligned16(P_v_old) || !aligned16(P_v_new))
    return LRKV_ERR_ARG;
  if (workspace_bytes < lrkv_rebase_workspace_bytes(cache)) return LRKV_ERR_WORKSPACE;
  if (cache->dtype == LRKV_BF16_Q8 || cache->dtype == LRKV_BF16_VA) return LRKV_ERR_UNSUPPORTED;
  if (!P_k_old && !P_v_old) return LRKV_OK;
  return rebase_launch(*cache, P_k_old, P_k_new, P_v_old, P_v_new, basis_batch_stride, workspace,
                       static_cast<cudaStream_t>(stream));
}

int lrkv_dense_append(const lrkv_dense_cache* cache, const void* k, const void* v,
                      int32_t n_tokens, const int32_t* n_new, int64_t seq_stride, int64_t head_stride, void* stream) {
  int rc = check_dense(cache);
  if (rc != LRKV_OK) return rc;
  if (n_tokens < 0) return LRKV_ERR_ARG;
  if (n_tokens == 0) return LRKV_OK;
  if (!k || !v) return LRKV_ERR_ARG;
  if ((long long)n_tokens > (long long)cache->max_pages_per_seq * kFrTile) return LRKV_ERR_CAPACITY;
  return dense_append_launch(*cache, k, v, n_tokens, n_new, seq_stride, head_stride,
                             static_cast<cudaStream_t>(stream));
}

size_t lrkv_dense_decode_workspace_bytes(const lrkv_dense_cache* cache, int32_t num_q_heads) {
  if (check_dense(cache) != LRKV_OK || check_heads(cache->num_kv_heads, num_q_heads) != LRKV_OK)
    return 0;
  return decode_workspace_bytes(cache->batch, cache->num_kv_heads, num_q_heads, 0, 0, false, true,
                                cache->dtype);
}

int lrkv_dense_decode_attn(const lrkv_dense_cache* cache, const void* q, int32_t num_q_heads,
                           float scale, void* o, void* workspace, size_t workspace_bytes,
                           void* stream) {
  int rc = check_dense(cache);
  if (rc != LRKV_OK) return rc;
  rc = check_heads(cache->num_kv_heads, num_q_heads);
  if (rc != LRKV_OK) return rc;
  if (!q || !o || !workspace) return LRKV_ERR_ARG;
  if (!aligned16(workspace)) return LRKV_ERR_ARG;
  DecodeLaunch L;
  L.B = cache->batch; L.H_kv = cache->num_kv_heads; L.H_q = num_q_heads; L.dtype = cache->dtype;
  L.seq_len = cache->seq_len; L.n_sink = 0; L.W = INT_MAX;
  L.codes = nullptr; L.bt_lat = nullptr; L.maxp_lat = 0; L.rk = 0; L.rv = 0;
  L.num_pages_lat = 0;
  L.fr = cache->kv_pages; L.bt_fr = cache->block_table;
  L.maxp_fr = cache->max_pages_per_seq; L.num_pages_fr = cache->num_pages;
  L.q = q; L.P_k = nullptr; L.P_v = nullptr; L.basis_bs = 0; L.scale = scale;
  L.o = o; L.ws = workspace; L.ws_bytes = workspace_bytes;
  return decode_launch(L, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
