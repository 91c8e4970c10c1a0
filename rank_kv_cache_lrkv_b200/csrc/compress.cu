// Append + compress: new tokens enter the sink / window ring, and every
// token that becomes latent is projected to codes c = P^T x and written into
// its page (Half the Memory, section 04: store the small r-dim codes; OjaKV
// article: first and most recent tokens kept full-rank as anchors).
//
// For a sequence going from L0 to L1 = L0 + n tokens, with latent counts
// lat(L0) and lat(L1), the tokens n_sink + [lat(L0), lat(L1)) become latent:
// those below L0 are read from the window ring (evictions), the others come
// straight from the input.  Ring reads happen before the window writes in
// the same CTA, so a slot is never overwritten before it is compressed.
//
// Launch order per call: bulk_compress (input tokens that go straight to the
// latent pages, only for large n) then append_kernel (evictions, small-n
// input tokens, sink and window writes, and the seq_len advance).  seq_len
// is advanced by the last CTA of each sequence to finish (a per-sequence
// completion counter, reset to zero by that CTA).
#include "common.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kSmallN = 16;       // input tokens handled by append_kernel
constexpr int kBulkRows = 64;     // tokens per bulk_compress CTA

// Tokens sequence b appends in this call.
__device__ inline int appended(const int* n_new, int n, int b) {
  if (!n_new) return n;
  const int x = n_new[b];
  return x < 0 ? 0 : (x < n ? x : n);
}

struct AppendArgs {
  int B, H_kv, rk, rv, n_sink, W, maxp, num_pages, n, anchor_tiles;
  void *codes, *anchors;
  const int* bt;
  int* seq_len;
  int* counter;
  const int* n_new;  // optional per-sequence counts (<= n)
  const void *k, *v;
  long long seq_stride, head_stride;
  const float *P_k, *P_v;
  long long basis_bs;
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

// Codes of one token held in shared memory (xk, xv fp32) -> pages.  The
// 128-long dot products are split over 4 row segments so every thread has
// independent loads in flight; red holds [4][r_k + r_v] partial sums.
constexpr int kSeg = 4;
template <typename T>
__device__ void project_one(const AppendArgs& a, int b, int kvh, int j, const float* xk,
                            const float* xv, float* red) {
  const float* Pk = a.P_k + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rk;
  const float* Pv = a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rv;
  const int NJ = a.rk + a.rv;
  constexpr int rows = kHeadDim / kSeg;
  for (int task = threadIdx.x; task < kSeg * NJ; task += blockDim.x) {
    const int seg = task / NJ, o = task - seg * NJ;
    const bool isk = o < a.rk;
    const int jj = isk ? o : o - a.rk;
    const int r = isk ? a.rk : a.rv;
    const float* P = (isk ? Pk : Pv) + (size_t)seg * rows * r + jj;
    const float* x = (isk ? xk : xv) + seg * rows;
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < rows; ++i) s = fmaf(P[(size_t)i * r], x[i], s);
    red[seg * NJ + o] = s;
  }
  __syncthreads();
  for (int o = threadIdx.x; o < NJ; o += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int seg = 0; seg < kSeg; ++seg) s += red[seg * NJ + o];
    const bool isk = o < a.rk;
    const int jj = isk ? o : o - a.rk;
    const long long off = code_off<T>(a, b, kvh, j, jj, isk ? 0 : 1);
    if (off >= 0) static_cast<T*>(a.codes)[off] = from_f<T>(s);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a, int do_input_latent) {
  __shared__ float xk[kHeadDim], xv[kHeadDim];
  __shared__ float red[kSeg * 2 * kHeadDim];
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int L0 = a.seq_len[b], L1 = L0 + appended(a.n_new, a.n, b);
  const Split s0 = split_tokens(L0, a.n_sink, a.W), s1 = split_tokens(L1, a.n_sink, a.W);
  const T* kin = static_cast<const T*>(a.k) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* vin = static_cast<const T*>(a.v) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* anc = static_cast<const T*>(a.anchors);

  // 1. evictions from the ring (token index < L0), oldest first.
  const int ev_lo = a.n_sink + s0.lat, ev_hi = min(L0, a.n_sink + s1.lat);
  for (int t = ev_lo; t < ev_hi; ++t) {
    const int slot = a.n_sink + (t - a.n_sink) % a.W;
    for (int d = threadIdx.x; d < kHeadDim; d += blockDim.x) {
      xk[d] = to_f<T>(anc[anchor_off<T>(a, b, kvh, slot, d, 0)]);
      xv[d] = to_f<T>(anc[anchor_off<T>(a, b, kvh, slot, d, 1)]);
    }
    __syncthreads();
    project_one<T>(a, b, kvh, t - a.n_sink, xk, xv, red);
    __syncthreads();
  }
  // 2. input tokens that go straight to latent (small n only).
  if (do_input_latent) {
    const int in_lo = max(L0, a.n_sink + s0.lat), in_hi = a.n_sink + s1.lat;
    for (int t = in_lo; t < in_hi; ++t) {
      for (int d = threadIdx.x; d < kHeadDim; d += blockDim.x) {
        xk[d] = to_f<T>(kin[(size_t)(t - L0) * kHeadDim + d]);
        xv[d] = to_f<T>(vin[(size_t)(t - L0) * kHeadDim + d]);
      }
      __syncthreads();
      project_one<T>(a, b, kvh, t - a.n_sink, xk, xv, red);
      __syncthreads();
    }
  }
  // 3. sink and window writes (full-rank, verbatim).
  if (a.n_sink + a.W > 0) {
    T* ancw = static_cast<T*>(a.anchors);
    const int w_lo = max(L0, max(a.n_sink, L1 - a.W));
    // sink first (t < n_sink), then the window tokens [w_lo, L1)
    const int n_sink_new = max(0, min(a.n_sink, L1) - L0);
    const int n_win_new = max(0, L1 - w_lo);
    const int total = (n_sink_new + n_win_new) * kHeadDim;
    for (int x = threadIdx.x; x < total; x += blockDim.x) {
      const int q = x / kHeadDim, d = x - q * kHeadDim;
      int t, slot;
      if (q < n_sink_new) { t = L0 + q; slot = t; }
      else { t = w_lo + (q - n_sink_new); slot = a.n_sink + (t - a.n_sink) % a.W; }
      ancw[anchor_off<T>(a, b, kvh, slot, d, 0)] = kin[(size_t)(t - L0) * kHeadDim + d];
      ancw[anchor_off<T>(a, b, kvh, slot, d, 1)] = vin[(size_t)(t - L0) * kHeadDim + d];
    }
  }
  // 4. the last CTA of this sequence advances seq_len.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(&a.counter[b], 1);
    if (old == a.H_kv - 1) {
      a.seq_len[b] = L1;
      a.counter[b] = 0;
      __threadfence();
    }
  }
}

// Input tokens that become latent without passing through the window, in
// tiles of kBulkRows tokens per (tile, kv head, sequence).
template <typename T>
__global__ void __launch_bounds__(256) bulk_compress_kernel(AppendArgs a) {
  __shared__ float xs[kBulkRows][kHeadDim + 1];
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int L0 = a.seq_len[b], L1 = L0 + appended(a.n_new, a.n, b);
  const Split s0 = split_tokens(L0, a.n_sink, a.W), s1 = split_tokens(L1, a.n_sink, a.W);
  const int in_lo = max(L0, a.n_sink + s0.lat) - L0, in_hi = a.n_sink + s1.lat - L0;
  const int r0 = in_lo + blockIdx.x * kBulkRows;
  const int rows = min(kBulkRows, in_hi - r0);
  if (rows <= 0) return;
  for (int pass = 0; pass < 2; ++pass) {
    const T* src = static_cast<const T*>(pass == 0 ? a.k : a.v) + (size_t)b * a.seq_stride +
                   (size_t)kvh * a.head_stride;
    for (int x = threadIdx.x; x < rows * kHeadDim; x += blockDim.x) {
      const int rr = x / kHeadDim, d = x - rr * kHeadDim;
      xs[rr][d] = to_f<T>(src[(size_t)(r0 + rr) * kHeadDim + d]);
    }
    __syncthreads();
    const int r = pass == 0 ? a.rk : a.rv;
    const float* P = (pass == 0 ? a.P_k : a.P_v) + (size_t)b * a.basis_bs +
                     (size_t)kvh * kHeadDim * r;
    T* dst = static_cast<T*>(a.codes);
    for (int o = threadIdx.x; o < rows * r; o += blockDim.x) {
      const int rr = o / r, jj = o - rr * r;
      float s = 0.f;
#pragma unroll 8
      for (int i = 0; i < kHeadDim; ++i) s = fmaf(P[(size_t)i * r + jj], xs[rr][i], s);
      const int j = L0 + r0 + rr - a.n_sink;  // latent index
      long long off = code_off<T>(a, b, kvh, j, jj, pass);
      if (off >= 0) dst[off] = from_f<T>(s);
    }
    __syncthreads();
  }
}

template <typename T>
static int compress_t(const AppendArgs& a, cudaStream_t st) {
  const bool small = a.n <= kSmallN;
  if (!small) {
    dim3 g((a.n + kBulkRows - 1) / kBulkRows, a.H_kv, a.B);
    bulk_compress_kernel<T><<<g, 256, 0, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  }
  append_kernel<T><<<dim3(a.H_kv, a.B), 256, 0, st>>>(a, small ? 1 : 0);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

int compress_launch(const lrkv_cache& c, const void* k, const void* v, int n, const int* n_new,
                    long long seq_stride, long long head_stride, const float* P_k,
                    const float* P_v, long long basis_bs, cudaStream_t st) {
  AppendArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.rk = c.rank_k; a.rv = c.rank_v;
  a.n_sink = c.n_sink; a.W = c.window; a.maxp = c.max_pages_per_seq; a.num_pages = c.num_pages;
  a.n = n; a.anchor_tiles = (c.n_sink + c.window + kFrTile - 1) / kFrTile;
  a.codes = c.codes; a.anchors = c.anchors;
  a.bt = c.block_table; a.seq_len = c.seq_len; a.counter = c.append_counter; a.n_new = n_new;
  a.k = k; a.v = v; a.seq_stride = seq_stride; a.head_stride = head_stride;
  a.P_k = P_k; a.P_v = P_v; a.basis_bs = basis_bs;
  return c.dtype == LRKV_BF16 ? compress_t<__nv_bfloat16>(a, st) : compress_t<float>(a, st);
}

// ------------------------------------------------------------ dense baseline
struct DenseAppendArgs {
  int B, H_kv, maxp, num_pages, n;
  void* kvp;
  const int* bt;
  int* seq_len;
  int* counter;
  const int* n_new;
  const void *k, *v;
  long long seq_stride, head_stride;
};

template <typename T>
__global__ void __launch_bounds__(256) dense_append_kernel(DenseAppendArgs a) {
  constexpr int CE = Elem<T>::CE;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int L0 = a.seq_len[b], nb = appended(a.n_new, a.n, b);
  const T* kin = static_cast<const T*>(a.k) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* vin = static_cast<const T*>(a.v) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  T* kvp = static_cast<T*>(a.kvp);
  for (int x = threadIdx.x; x < nb * kHeadDim; x += blockDim.x) {
    const int q = x / kHeadDim, d = x - q * kHeadDim;
    const int t = L0 + q, pi = t / kFrTile;
    if (pi >= a.maxp) continue;
    const int page = a.bt[(size_t)b * a.maxp + pi];
    if (page < 0 || page >= a.num_pages) continue;
    const size_t slab = ((size_t)page * a.H_kv + kvh) * (2 * kHeadDim / CE);
    const size_t row = (size_t)(t % kFrTile) * CE + d % CE;
    kvp[(slab + d / CE) * kFrTile * CE + row] = kin[(size_t)q * kHeadDim + d];
    kvp[(slab + kHeadDim / CE + d / CE) * kFrTile * CE + row] = vin[(size_t)q * kHeadDim + d];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(&a.counter[b], 1);
    if (old == a.H_kv - 1) {
      a.seq_len[b] = L0 + nb;
      a.counter[b] = 0;
      __threadfence();
    }
  }
}

int dense_append_launch(const lrkv_dense_cache& c, const void* k, const void* v, int n,
                        const int* n_new, long long seq_stride, long long head_stride, cudaStream_t st) {
  DenseAppendArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.maxp = c.max_pages_per_seq;
  a.num_pages = c.num_pages; a.n = n; a.kvp = c.kv_pages;
  a.bt = c.block_table; a.seq_len = c.seq_len; a.counter = c.append_counter; a.n_new = n_new;
  a.k = k; a.v = v; a.seq_stride = seq_stride; a.head_stride = head_stride;
  dim3 g(a.H_kv, a.B);
  if (c.dtype == LRKV_BF16)
    dense_append_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(a);
  else
    dense_append_kernel<float><<<g, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
