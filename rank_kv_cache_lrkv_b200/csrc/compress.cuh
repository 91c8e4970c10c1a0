// Argument block and index helpers shared by the compress kernels
// (append_kernel, the SIMT and warp-MMA prefill kernels, and the
// tensor-memory prefill kernel).
#pragma once
#include "common.cuh"

namespace lrkv {

// Tokens sequence b appends in this call.
__device__ inline int appended(const int* n_new, int n, int b) {
  if (!n_new) return n;
  const int x = n_new[b];
  return x < 0 ? 0 : (x < n ? x : n);
}

struct AppendArgs {
  int B, H_kv, rk, rv, n_sink, W, maxp, num_pages, n, anchor_tiles;
  int q8;            // codes stored as per-token int8 + fp32 scales (bf16 inputs)
  int va;            // value-amortised slabs: key codes + residual slots
  const float* A;    // value predictors [B][H_kv][rk][rv] (va; NULL: not fitted yet)
  void *codes, *anchors;
  const int* bt;
  int* seq_len;
  int* counter;
  const int* n_new;  // optional per-sequence counts (<= n)
  const void *k, *v;
  long long seq_stride, head_stride;
  const float *P_k, *P_v;
  long long basis_bs;
  // Optional query fold of a decode step (fq != nullptr), done by the CTA of
  // unit (b, kvh) from the basis it stages anyway: q [B][fH_q][128] ->
  // fqlat [B][fH_q][rk] = fqscale P_k^T q and, when fqfr != nullptr,
  // fqfr [B][fH_q][128] = fqscale q.
  const void* fq;
  int fH_q;
  float fqscale;
  float *fqlat, *fqfr;
};

// Element offset of (slot, dim d) of the key (isv = 0) or value (isv = 1)
// in the anchor tiles of unit (b, kvh).
template <typename T>
__device__ inline size_t anchor_off(const AppendArgs& a, int b, int kvh, int slot, int d, int isv) {
  constexpr int CE = Elem<T>::CE;
  const size_t tile = ((size_t)b * a.H_kv + kvh) * a.anchor_tiles + slot / kFrTile;
  const int chunk = isv * (kHeadDim / CE) + d / CE;
  return (tile * (2 * kHeadDim / CE) + chunk) * kFrTile * CE + (slot % kFrTile) * CE + d % CE;
}

// Element offset of (latent index j, code dim jj) of the key (isv = 0) or
// value (isv = 1) codes in the code pool; -1 if the page is out of range.
template <typename T>
__device__ inline long long code_off(const AppendArgs& a, int b, int kvh, int j, int jj, int isv) {
  constexpr int CE = Elem<T>::CE;
  const int pi = j / kLatPage;
  if (pi >= a.maxp) return -1;
  const int page = a.bt[(size_t)b * a.maxp + pi];
  if (page < 0 || page >= a.num_pages) return -1;
  const int nch = (a.rk + a.rv) / CE;
  const int chunk = isv * (a.rk / CE) + jj / CE;
  return ((((long long)page * a.H_kv + kvh) * nch + chunk) * kLatPage + j % kLatPage) * CE +
         jj % CE;
}

// Page of latent index j of sequence b (-1 when past the block table or
// out of the pool), and the element offset of code dim jj of that token.
__device__ inline int latent_page(const AppendArgs& a, int b, int j) {
  const int pi = j / kLatPage;
  if (pi >= a.maxp) return -1;
  const int page = a.bt[(size_t)b * a.maxp + pi];
  return page >= 0 && page < a.num_pages ? page : -1;
}
template <typename T>
__device__ inline long long code_off_in(const AppendArgs& a, int page, int kvh, int j, int jj,
                                        int isv) {
  constexpr int CE = Elem<T>::CE;
  // elements per slab: key and value codes, or (value-amortised) the key
  // codes followed by the residual slots
  const long long slab = a.va ? va_slab_bytes(a.rk, a.rv) / (long long)sizeof(T)
                              : (long long)kLatPage * (a.rk + a.rv);
  const int chunk = isv * (a.rk / CE) + jj / CE;
  return ((long long)page * a.H_kv + kvh) * slab + ((long long)chunk * kLatPage + j % kLatPage) * CE +
         jj % CE;
}

__host__ __device__ inline int round16(int x) { return (x + 15) / 16 * 16; }

// First tile of CTA c when `total` tiles are split evenly over C CTAs.
__device__ inline int bulk_range_lo(int c, int total, int C) {
  const int q = total / C, r = total - q * C;
  return c * q + (c * r) / C;
}

// Input rows of sequence b that go straight to latent: [in_lo, in_hi), relative to L0.
__device__ inline void bulk_rows(const AppendArgs& a, int b, int& L0, int& in_lo, int& in_hi) {
  L0 = __ldcg(a.seq_len + b);
  const int L1 = L0 + appended(a.n_new, a.n, b);
  const Split s0 = split_tokens(L0, a.n_sink, a.W), s1 = split_tokens(L1, a.n_sink, a.W);
  in_lo = max(L0, a.n_sink + s0.lat) - L0;
  in_hi = max(in_lo, a.n_sink + s1.lat - L0);
}

// ---- per-token int8 codes (LRKV_BF16_Q8): slab of 64 * (rk + rv) code
// bytes, 16 codes per chunk, chunk-major, then [64][2] fp32 scales.
__host__ __device__ inline int q8_slab_bytes(int rk, int rv) { return kLatPage * (rk + rv) + 512; }
// Byte offset of code jj (of side isv) of latent row j % 64 in its page.
__device__ inline long long q8_code_off(const AppendArgs& a, int page, int kvh, int j, int jj,
                                        int isv) {
  const int chunk = isv * (a.rk / 16) + jj / 16;
  return ((long long)page * a.H_kv + kvh) * q8_slab_bytes(a.rk, a.rv) +
         ((long long)chunk * kLatPage + j % kLatPage) * 16 + jj % 16;
}
// Byte offset of the scale of (row j % 64, side isv) in its page.
__device__ inline long long q8_scale_off(const AppendArgs& a, int page, int kvh, int j, int isv) {
  return ((long long)page * a.H_kv + kvh) * q8_slab_bytes(a.rk, a.rv) +
         (long long)kLatPage * (a.rk + a.rv) + ((j % kLatPage) * 2 + isv) * 4;
}
// The int8 code of c under scale s: round half to even of c / s (IEEE
// division), clamped to [-127, 127]; 0 when s == 0.
__device__ __forceinline__ int q8_code(float c, float s) {
  if (!(s > 0.f)) return 0;
  const int q = __float2int_rn(__fdiv_rn(c, s));
  return q > 127 ? 127 : (q < -127 ? -127 : q);
}

// Prefill compress of bf16 inputs on the fifth-generation tensor cores
// (compress_tc.cu); LRKV_ERR_UNSUPPORTED when the configuration does not
// fit, so the caller can take the warp-MMA kernel instead.
int bulk_compress_tc_launch(const AppendArgs& a, int sms, int optin, cudaStream_t st);

}  // namespace lrkv
