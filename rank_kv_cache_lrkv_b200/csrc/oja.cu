// Oja subspace update and QR re-orthonormalisation of per-stream bases
// (OjaKV article: Oja's algorithm for online PCA adapts the projection basis
// during prompt prefill and periodically during decode).
//
// One CTA of 128 threads per stream keeps its basis P [128][r] in shared
// memory (row stride r + 1, so row-wise and column-wise walks are both free
// of bank conflicts).  For each token, in order:
//   y_j = sum_i P[i][j] x_i          (thread j)
//   z_i = x_i - sum_j P[i][j] y_j    (thread i, row i)
//   P[i][j] += eta z_i y_j           (thread i updates its own row)
// and after every qr_every-th token P <- Q of QR(P) with diag(R) > 0, by
// Gram-Schmidt with a second orthogonalisation pass per column.
#include "common.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kOjaThreads = 128;

__device__ float block_sum128(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

// Q of QR(P), diag(R) > 0, in place on the padded shared basis.
__device__ void qr_shared(float* P, int r, int ld, float* col, float* h, float* red) {
  const int i = threadIdx.x;
  for (int j = 0; j < r; ++j) {
    col[i] = P[i * ld + j];
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      // h_k = P[:, k] . col for every k < j (thread k)
      for (int k = threadIdx.x; k < j; k += blockDim.x) {
        float s = 0.f;
        for (int ii = 0; ii < kHeadDim; ++ii) s = fmaf(P[ii * ld + k], col[ii], s);
        h[k] = s;
      }
      __syncthreads();
      float c = col[i];
      for (int k = 0; k < j; ++k) c = fmaf(-h[k], P[i * ld + k], c);
      __syncthreads();
      col[i] = c;
      __syncthreads();
    }
    const float nrm = sqrtf(block_sum128(col[i] * col[i], red));
    P[i * ld + j] = col[i] / nrm;
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(kOjaThreads) oja_kernel(float* P, int r, long long bstride,
                                                         const T* __restrict__ x,
                                                         long long xstride, int n, float eta,
                                                         int qr_every, long long seen) {
  extern __shared__ float sm[];
  const int ld = r + 1;
  float* Ps = sm;                        // [128][ld]
  float* xs = Ps + kHeadDim * ld;        // [2][128]
  float* ys = xs + 2 * kHeadDim;         // [128]
  float* col = ys + kHeadDim;            // [128]
  float* h = col + kHeadDim;             // [128]
  __shared__ float red[4];
  const int i = threadIdx.x;
  float* Pg = P + (size_t)blockIdx.x * bstride;
  const T* xg = x + (size_t)blockIdx.x * xstride;
  for (int e = i; e < kHeadDim * r; e += blockDim.x) Ps[(e / r) * ld + e % r] = Pg[e];
  if (n > 0) xs[i] = to_f<T>(xg[i]);
  __syncthreads();
  for (int t = 0; t < n; ++t) {
    const float* xc = xs + (t & 1) * kHeadDim;
    if (i < r) {
      float y = 0.f;
#pragma unroll 8
      for (int k = 0; k < kHeadDim; ++k) y = fmaf(Ps[k * ld + i], xc[k], y);
      ys[i] = y;
    }
    __syncthreads();
    float* row = Ps + i * ld;
    float z = xc[i];
    for (int j = 0; j < r; ++j) z = fmaf(-row[j], ys[j], z);
    const float ez = eta * z;
    for (int j = 0; j < r; ++j) row[j] = fmaf(ez, ys[j], row[j]);
    if (t + 1 < n) xs[((t + 1) & 1) * kHeadDim + i] = to_f<T>(xg[(size_t)(t + 1) * kHeadDim + i]);
    __syncthreads();
    if (qr_every > 0 && (seen + t + 1) % qr_every == 0) qr_shared(Ps, r, ld, col, h, red);
  }
  for (int e = i; e < kHeadDim * r; e += blockDim.x) Pg[e] = Ps[(e / r) * ld + e % r];
}

__global__ void __launch_bounds__(kOjaThreads) qr_kernel(float* P, int r, long long bstride) {
  extern __shared__ float sm[];
  const int ld = r + 1;
  float* Ps = sm;
  float* col = Ps + kHeadDim * ld;
  float* h = col + kHeadDim;
  __shared__ float red[4];
  float* Pg = P + (size_t)blockIdx.x * bstride;
  for (int e = threadIdx.x; e < kHeadDim * r; e += blockDim.x) Ps[(e / r) * ld + e % r] = Pg[e];
  __syncthreads();
  qr_shared(Ps, r, ld, col, h, red);
  for (int e = threadIdx.x; e < kHeadDim * r; e += blockDim.x) Pg[e] = Ps[(e / r) * ld + e % r];
}

static size_t oja_smem(int r) { return (size_t)(kHeadDim * (r + 1) + 5 * kHeadDim) * 4; }

int oja_launch(float* P, int S, int r, long long basis_stride, const void* x, int x_dtype,
               long long x_stride, int n, float eta, int qr_every, long long tokens_seen,
               cudaStream_t st) {
  const size_t sm = oja_smem(r);
  if (x_dtype == LRKV_BF16) {
    auto k = oja_kernel<__nv_bfloat16>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return LRKV_ERR_CUDA;
    k<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride, static_cast<const __nv_bfloat16*>(x),
                                   x_stride, n, eta, qr_every, tokens_seen);
  } else {
    auto k = oja_kernel<float>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
      return LRKV_ERR_CUDA;
    k<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride, static_cast<const float*>(x), x_stride, n,
                                   eta, qr_every, tokens_seen);
  }
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

int qr_launch(float* P, int S, int r, long long basis_stride, cudaStream_t st) {
  const size_t sm = oja_smem(r);
  if (cudaFuncSetAttribute(qr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
      cudaSuccess)
    return LRKV_ERR_CUDA;
  qr_kernel<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
