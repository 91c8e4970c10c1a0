// Oja subspace update and QR re-orthonormalisation of per-stream bases
// (OjaKV article: Oja's algorithm for online PCA adapts the projection basis
// during prompt prefill and periodically during decode).
//
// For r <= 64 the basis lives in registers (oja2_kernel below).  Otherwise
// one CTA of 128 threads per stream keeps its basis P [128][r] in shared
// memory (row stride r + 1, so row-wise and column-wise walks are both free
// of bank conflicts).  For each token, in order:
//   y_j = sum_i P[i][j] x_i          (thread j)
//   z_i = x_i - sum_j P[i][j] y_j    (thread i, row i)
//   P[i][j] += eta z_i y_j           (thread i updates its own row)
// and after every qr_every-th token P <- Q of QR(P) with diag(R) > 0, by
// Gram-Schmidt with a second orthogonalisation pass per column.
#include <cstdint>

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

// ---- register-resident Oja update for r <= 64
// 64 threads per stream; thread t holds rows t and t + 64 of P as float
// pairs (RM >= r columns, the padding columns are zero and stay zero).  Per
// token:
//   y = P^T x : per-thread products of its two rows, reduce-scattered across
//               each warp in blocks of 16 columns (16 shuffles per block), the
//               two warps combined through shared memory;
//   z_i = x_i - P_i . y,  P_i += eta z_i y   (registers; y read back as
//               broadcast 16-byte loads).
// Token rows arrive by cp.async in chunks of kOjaChunk tokens, double
// buffered.  The QR every qr_every tokens writes P to a padded shared tile,
// runs classical Gram-Schmidt with a second pass per column, and reads it back.
constexpr int kOja2Threads = 64;
constexpr int kOjaChunk = 8;

__device__ __forceinline__ void bar64() { named_bar(1, kOja2Threads); }

// One reduce-scatter stage over lane bit O: the lanes with the bit set keep
// the upper half of their N values, the others the lower half, each adding
// the partner's copy of the half it keeps.
template <int N, int O>
__device__ __forceinline__ void rs_stage(float (&w)[16], int lane) {
  const bool up = (lane & O) != 0;
#pragma unroll
  for (int k = 0; k < N / 2; ++k) {
    const float send = up ? w[k] : w[k + N / 2];
    const float keep = up ? w[k + N / 2] : w[k];
    w[k] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}

// Sum of w[0..15] over the 32 lanes, scattered: the lane ends with the sum of
// column (lane & 15) (lanes l and l ^ 16 hold the same column).
__device__ __forceinline__ float reduce16(float (&w)[16], int lane) {
  rs_stage<16, 8>(w, lane);
  rs_stage<8, 4>(w, lane);
  rs_stage<4, 2>(w, lane);
  rs_stage<2, 1>(w, lane);
  return w[0] + __shfl_xor_sync(0xffffffffu, w[0], 16);
}

// Q of QR(P), diag(R) > 0, on the padded shared tile [128][ld], 64 threads
// (rows t and t + 64 each).
__device__ void qr_shared64(float* PQ, int r, int ld, float* col, float* h, float* red) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  for (int j = 0; j < r; ++j) {
    col[t] = PQ[t * ld + j];
    col[t + 64] = PQ[(t + 64) * ld + j];
    bar64();
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = t; k < j; k += kOja2Threads) {
        float s0 = 0.f, s1 = 0.f;
        for (int i = 0; i < kHeadDim; i += 2) {
          s0 = fmaf(PQ[i * ld + k], col[i], s0);
          s1 = fmaf(PQ[(i + 1) * ld + k], col[i + 1], s1);
        }
        h[k] = s0 + s1;
      }
      bar64();
      float c0 = col[t], c1 = col[t + 64];
      for (int k = 0; k < j; ++k) {
        c0 = fmaf(-h[k], PQ[t * ld + k], c0);
        c1 = fmaf(-h[k], PQ[(t + 64) * ld + k], c1);
      }
      bar64();
      col[t] = c0;
      col[t + 64] = c1;
      bar64();
    }
    const float c0 = col[t], c1 = col[t + 64];
    const float ss = warp_sum(c0 * c0 + c1 * c1);
    if (lane == 0) red[w] = ss;
    bar64();
    const float nrm = sqrtf(red[0] + red[1]);
    PQ[t * ld + j] = c0 / nrm;
    PQ[(t + 64) * ld + j] = c1 / nrm;
    bar64();
  }
}

inline size_t oja2_smem_bytes(int r, int esize) {
  const int RM = (r + 15) / 16 * 16;
  return (size_t)kHeadDim * (r + 1) * 4            // PQ
         + (size_t)2 * kOjaChunk * kHeadDim * esize  // x ring
         + (size_t)2 * 2 * RM * 4                    // red [parity][warp][RM]
         + (size_t)2 * RM * 4                        // ys [parity][RM]
         + (size_t)kHeadDim * 4 + (size_t)RM * 4 + 16;  // col, h, norm
}

template <typename T, int RM>
__global__ void __launch_bounds__(kOja2Threads, 6) oja2_kernel(float* P, int r, long long bstride,
                                                            const T* __restrict__ x,
                                                            long long xstride, int n, float eta,
                                                            int qr_every, long long seen) {
  constexpr int NB = RM / 16;                // column blocks
  constexpr int NP = RM / 2;                 // float pairs per row
  constexpr int CE = 16 / sizeof(T);         // elements per 16-byte copy
  extern __shared__ __align__(16) float sm[];
  const int ld = r + 1;
  float* PQ = sm;                                                       // [128][ld]
  T* xr = reinterpret_cast<T*>(PQ + ((kHeadDim * ld + 3) & ~3));         // [2][chunk][128]
  float* red = reinterpret_cast<float*>(xr + 2 * kOjaChunk * kHeadDim);  // [2][2][RM]
  float* ys = red + 2 * 2 * RM;                                         // [2][RM]
  float* col = ys + 2 * RM;                                             // [128]
  float* h = col + kHeadDim;                                            // [RM]
  float* nred = h + RM;                                                 // [2]
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  float* Pg = P + (size_t)blockIdx.x * bstride;
  const T* xg = x + (size_t)blockIdx.x * xstride;

  auto stage = [&](int c, int buf) {  // chunk c of token rows into ring buffer buf
    const int t0 = c * kOjaChunk;
    for (int q = t; q < kOjaChunk * kHeadDim / CE; q += kOja2Threads) {
      const int row = q / (kHeadDim / CE), e = (q - row * (kHeadDim / CE)) * CE;
      const bool ok = t0 + row < n;
      cp_async16(xr + (buf * kOjaChunk + row) * kHeadDim + e,
                 xg + (size_t)(ok ? t0 + row : 0) * kHeadDim + e, ok ? 16u : 0u);
    }
    cp_async_commit();
  };
  if (n > 0) stage(0, 0);

  float2 P0[NP], P1[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = 2 * p;
    P0[p] = make_float2(j < r ? Pg[t * r + j] : 0.f, j + 1 < r ? Pg[t * r + j + 1] : 0.f);
    P1[p] = make_float2(j < r ? Pg[(t + 64) * r + j] : 0.f,
                        j + 1 < r ? Pg[(t + 64) * r + j + 1] : 0.f);
  }
  for (int q = t; q < 2 * RM; q += kOja2Threads) ys[q] = 0.f;  // padding columns stay 0

  for (int tok = 0; tok < n; ++tok) {
    const int c = tok / kOjaChunk, slot = tok - c * kOjaChunk, buf = c & 1, par = tok & 1;
    if (slot == 0) {
      if ((c + 1) * kOjaChunk < n) {
        stage(c + 1, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      bar64();  // chunk c is in place for every thread
    }
    const T* xrow = xr + (buf * kOjaChunk + slot) * kHeadDim;
    const float x0 = to_f<T>(xrow[t]), x1 = to_f<T>(xrow[t + 64]);
    const float2 x02 = make_float2(x0, x0), x12 = make_float2(x1, x1);
    // y = P^T x: this thread's two rows, then across the warp and the two warps
#pragma unroll
    for (int bk = 0; bk < NB; ++bk) {
      float wv[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float2 v = mul2(P1[bk * 8 + u], x12);
        fma2(v, P0[bk * 8 + u], x02);
        wv[2 * u] = v.x;
        wv[2 * u + 1] = v.y;
      }
      const float s = reduce16(wv, lane);
      if (lane < 16) red[(par * 2 + w) * RM + bk * 16 + lane] = s;
    }
    bar64();
    if (t < r) ys[par * RM + t] = red[(par * 2) * RM + t] + red[(par * 2 + 1) * RM + t];
    bar64();
    // z = x - P y, then P += eta z y^T
    const float4* y4 = reinterpret_cast<const float4*>(ys + par * RM);
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < RM / 4; ++q) {
      const float4 yv = y4[q];
      const float2 ylo = make_float2(yv.x, yv.y), yhi = make_float2(yv.z, yv.w);
      fma2(a0, P0[2 * q], ylo);
      fma2(a0, P0[2 * q + 1], yhi);
      fma2(a1, P1[2 * q], ylo);
      fma2(a1, P1[2 * q + 1], yhi);
    }
    const float ez0 = eta * (x0 - (a0.x + a0.y)), ez1 = eta * (x1 - (a1.x + a1.y));
    const float2 e02 = make_float2(ez0, ez0), e12 = make_float2(ez1, ez1);
#pragma unroll
    for (int q = 0; q < RM / 4; ++q) {
      const float4 yv = y4[q];
      const float2 ylo = make_float2(yv.x, yv.y), yhi = make_float2(yv.z, yv.w);
      fma2(P0[2 * q], e02, ylo);
      fma2(P0[2 * q + 1], e02, yhi);
      fma2(P1[2 * q], e12, ylo);
      fma2(P1[2 * q + 1], e12, yhi);
    }
    if (qr_every > 0 && (seen + tok + 1) % qr_every == 0) {
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int j = 2 * p;
        if (j < r) { PQ[t * ld + j] = P0[p].x; PQ[(t + 64) * ld + j] = P1[p].x; }
        if (j + 1 < r) { PQ[t * ld + j + 1] = P0[p].y; PQ[(t + 64) * ld + j + 1] = P1[p].y; }
      }
      bar64();
      qr_shared64(PQ, r, ld, col, h, nred);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int j = 2 * p;
        P0[p] = make_float2(j < r ? PQ[t * ld + j] : 0.f, j + 1 < r ? PQ[t * ld + j + 1] : 0.f);
        P1[p] = make_float2(j < r ? PQ[(t + 64) * ld + j] : 0.f,
                            j + 1 < r ? PQ[(t + 64) * ld + j + 1] : 0.f);
      }
      bar64();
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = 2 * p;
    if (j < r) { Pg[t * r + j] = P0[p].x; Pg[(t + 64) * r + j] = P1[p].x; }
    if (j + 1 < r) { Pg[t * r + j + 1] = P0[p].y; Pg[(t + 64) * r + j + 1] = P1[p].y; }
  }
}

// ---- chunked Oja (P frozen within a chunk)
// One CTA of 128 threads per stream, r <= 64.  Per chunk of nc <= 64 tokens
// (a chunk ends early at a QR point):
//   Y = X P        [nc][r]    thread -> 4 tokens x r/8 columns
//   Z = X - Y P^T  [nc][128]  in place over X; thread -> 8 tokens x 8 rows
//   P += eta Z^T Y [128][r]   thread -> 4 rows x r/4 columns
// in fp32 from shared memory, register-blocked so each loaded value feeds
// several multiply-adds.  The next chunk's rows arrive by cp.async while
// the current one is processed.  QR every qr_every tokens seen, as in the
// sequential kernel.
constexpr int kBlkRows = 64;     // tokens per chunk at most
constexpr int kBlkLdX = 132;     // fp32 row stride of X / Z

inline size_t oja_blocked_smem_bytes(int r, int esize) {
  return (size_t)(kBlkRows * kBlkLdX + kBlkRows * (r + 1) + kHeadDim * (r + 1) + 2 * kHeadDim) *
             4 +
         (size_t)2 * kBlkRows * kHeadDim * esize;
}

template <typename T>
__global__ void __launch_bounds__(kOjaThreads) oja_blocked_kernel(
    float* P, int r, long long bstride, const T* __restrict__ x, long long xstride, int n,
    float eta, int qr_every, long long seen, int chunk) {
  extern __shared__ __align__(16) float bsm[];
  const int ldp = r + 1;
  float* X = bsm;                                   // [64][132] fp32, becomes Z
  float* Y = X + kBlkRows * kBlkLdX;                // [64][r + 1]
  float* Ps = Y + kBlkRows * ldp;                   // [128][r + 1]
  float* col = Ps + kHeadDim * ldp;                 // [128] QR scratch
  float* h = col + kHeadDim;                        // [128]
  T* stg = reinterpret_cast<T*>(h + kHeadDim);      // [2][64][128] raw rows
  __shared__ float red[4];
  const int tid = threadIdx.x;
  constexpr int CE = Elem<T>::CE;
  float* Pg = P + (size_t)blockIdx.x * bstride;
  const T* xg = x + (size_t)blockIdx.x * xstride;
  for (int e = tid; e < kHeadDim * r; e += kOjaThreads) Ps[(e / r) * ldp + e % r] = Pg[e];

  // length of the chunk starting at token j
  auto chunk_len = [&](int j) {
    int nc = min(min(chunk, kBlkRows), n - j);
    if (qr_every > 0) {
      const long long to_qr = qr_every - (seen + j) % qr_every;
      if (to_qr < nc) nc = (int)to_qr;
    }
    return nc;
  };
  auto stage = [&](int j, int buf) {
    const int nc = chunk_len(j);
    T* dst = stg + (size_t)buf * kBlkRows * kHeadDim;
    for (int e = tid; e < nc * (kHeadDim / CE); e += kOjaThreads) {
      const int t = e / (kHeadDim / CE), c = e - t * (kHeadDim / CE);
      cp_async16(dst + t * kHeadDim + c * CE, xg + (size_t)(j + t) * kHeadDim + c * CE, 16u);
    }
    cp_async_commit();
  };
  if (n > 0) stage(0, 0);
  int buf = 0;
  for (int j = 0; j < n;) {
    const int nc = chunk_len(j);
    cp_async_wait<0>();
    __syncthreads();  // rows of this chunk landed; P and the buffers are free
    {
      const T* src = stg + (size_t)buf * kBlkRows * kHeadDim;
      for (int e = tid; e < kBlkRows * kHeadDim; e += kOjaThreads) {
        const int t = e >> 7, i = e & 127;
        X[t * kBlkLdX + i] = t < nc ? to_f<T>(src[e]) : 0.f;
      }
    }
    if (j + nc < n) stage(j + nc, buf ^ 1);
    __syncthreads();
    // Y = X P: thread -> tokens 4 tb .. 4 tb + 3, columns jb * (r / 8) ..
    {
      const int tb = tid >> 3, jb = tid & 7, rj = r >> 3, j0 = jb * rj;
      float acc[4][8];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
#pragma unroll 4
      for (int k = 0; k < kHeadDim; ++k) {
        float xv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) xv[a] = X[(4 * tb + a) * kBlkLdX + k];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c < rj) {
            const float pv = Ps[k * ldp + j0 + c];
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a][c] = fmaf(xv[a], pv, acc[a][c]);
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (c < rj) Y[(4 * tb + a) * ldp + j0 + c] = acc[a][c];
    }
    __syncthreads();
    // Z = X - Y P^T, in place: thread -> tokens 8 tb .. + 7, rows ib + 16 m
    {
      const int tb = tid >> 4, ib = tid & 15;
      float acc[8][8];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[a][m] = X[(8 * tb + a) * kBlkLdX + ib + 16 * m];
      for (int k = 0; k < r; ++k) {
        float yv[8], pv[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) yv[a] = Y[(8 * tb + a) * ldp + k];
#pragma unroll
        for (int m = 0; m < 8; ++m) pv[m] = Ps[(ib + 16 * m) * ldp + k];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int m = 0; m < 8; ++m) acc[a][m] = fmaf(-yv[a], pv[m], acc[a][m]);
      }
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int m = 0; m < 8; ++m) X[(8 * tb + a) * kBlkLdX + ib + 16 * m] = acc[a][m];
    }
    __syncthreads();
    // P += eta Z^T Y: thread -> rows ib + 32 m, columns jb * (r / 4) ..
    {
      const int ib = tid & 31, jb = tid >> 5, rj = r >> 2, j0 = jb * rj;
      float acc[4][16];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[m][c] = 0.f;
      for (int t = 0; t < nc; ++t) {
        float zv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) zv[m] = X[t * kBlkLdX + ib + 32 * m];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (c < rj) {
            const float yv = Y[t * ldp + j0 + c];
#pragma unroll
            for (int m = 0; m < 4; ++m) acc[m][c] = fmaf(zv[m], yv, acc[m][c]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c < rj) {
            float& pp = Ps[(ib + 32 * m) * ldp + j0 + c];
            pp = fmaf(eta, acc[m][c], pp);
          }
    }
    j += nc;
    buf ^= 1;
    __syncthreads();
    if (qr_every > 0 && (seen + j) % qr_every == 0) qr_shared(Ps, r, ldp, col, h, red);
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int e = tid; e < kHeadDim * r; e += kOjaThreads) Pg[e] = Ps[(e / r) * ldp + e % r];
}

// ---- chunked Oja on the tensor cores (bf16 token rows)
// One CTA of 256 threads (8 warps) per stream, r <= 64.  Per chunk of
// nc <= 64 tokens, three warp-level bf16 MMA products (m16n8k16, fp32
// accumulation) with every fp32 operand split into hi + lo bf16 halves (the
// lo x lo term dropped), so each product keeps about 16 mantissa bits:
//   Y = X P          warp -> m-block w % 4 (16 tokens), half the columns
//   Z = X - Y P^T    warp -> m-block w % 4, half of the 128 dims
//   P += eta Z^T Y   warp -> dims 16 w .. 16 w + 15, every column
// X is exact in bf16.  P is kept in fp32 (the master the update and the QR
// work on) and as hi/lo bf16 rows [128][ldp] that serve as the B operand of
// the first product (ldmatrix.trans) and of the second (ldmatrix); Y and Z
// are kept as hi/lo bf16 only.  Row strides are odd multiples of 16 bytes
// (ldmatrix without bank conflicts).  Rows of the next chunk arrive by
// cp.async (rows past the chunk zero-filled) while the current one runs.
constexpr int kMmaOjaThreads = 256;
constexpr int kLdX = kHeadDim + 8;  // bf16 row stride of X and Z (272 bytes)

__host__ __device__ inline int oja_ld16(int r) { return (r / 8) % 2 == 0 ? r + 8 : r + 16; }

struct OjaMmaPlan {
  int pf, ph, pl, x, yh, yl, zh, zl, col, h, red, total;
};
__host__ __device__ inline OjaMmaPlan oja_mma_plan(int r) {
  OjaMmaPlan p;
  int off = 0;
  auto take = [&](int bytes) {
    off = (off + 15) / 16 * 16;
    const int at = off;
    off += bytes;
    return at;
  };
  const int ldp = oja_ld16(r);
  p.pf = take(kHeadDim * (r + 1) * 4);          // fp32 master [128][r + 1]
  p.ph = take(kHeadDim * ldp * 2);              // [128][ldp] bf16
  p.pl = take(kHeadDim * ldp * 2);
  p.x = take(2 * kBlkRows * kLdX * 2);          // [2][64][kLdX] bf16
  p.yh = take(kBlkRows * ldp * 2);              // [64][ldp]
  p.yl = take(kBlkRows * ldp * 2);
  p.zh = take(kBlkRows * kLdX * 2);             // [64][kLdX]
  p.zl = take(kBlkRows * kLdX * 2);
  p.col = take(kHeadDim * 4);
  p.h = take(kHeadDim * 4);
  p.red = take(8 * 4);
  p.total = off;
  return p;
}

// Q of QR(P), diag(R) > 0, on the fp32 tile [128][ld] with 256 threads
// (threads < 128 own a row each; the others join the barriers).
__device__ void qr_rows256(float* P, int r, int ld, float* col, float* h, float* red) {
  const int i = threadIdx.x, lane = i & 31, w = i >> 5;
  for (int j = 0; j < r; ++j) {
    if (i < kHeadDim) col[i] = P[i * ld + j];
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = i; k < j; k += kMmaOjaThreads) {
        float s0 = 0.f, s1 = 0.f;
        for (int ii = 0; ii < kHeadDim; ii += 2) {
          s0 = fmaf(P[ii * ld + k], col[ii], s0);
          s1 = fmaf(P[(ii + 1) * ld + k], col[ii + 1], s1);
        }
        h[k] = s0 + s1;
      }
      __syncthreads();
      float c = i < kHeadDim ? col[i] : 0.f;
      if (i < kHeadDim)
        for (int k = 0; k < j; ++k) c = fmaf(-h[k], P[i * ld + k], c);
      __syncthreads();
      if (i < kHeadDim) col[i] = c;
      __syncthreads();
    }
    const float c = i < kHeadDim ? col[i] : 0.f;
    const float ss = warp_sum(c * c);
    if (lane == 0) red[w] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kMmaOjaThreads / 32; ++k) tot += red[k];
    if (i < kHeadDim) P[i * ld + j] = c / sqrtf(tot);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kMmaOjaThreads, 1) oja_chunked_mma(
    float* P, int r, long long bstride, const __nv_bfloat16* __restrict__ x, long long xstride,
    int n, float eta, int qr_every, long long seen, int chunk) {
  using bf16 = __nv_bfloat16;
  extern __shared__ __align__(16) uint8_t osm[];
  const OjaMmaPlan pl = oja_mma_plan(r);
  const int ldp = oja_ld16(r), ldf = r + 1;
  float* Pf = reinterpret_cast<float*>(osm + pl.pf);
  bf16* Ph = reinterpret_cast<bf16*>(osm + pl.ph);
  bf16* Pl = reinterpret_cast<bf16*>(osm + pl.pl);
  bf16* Xs = reinterpret_cast<bf16*>(osm + pl.x);
  bf16* Yh = reinterpret_cast<bf16*>(osm + pl.yh);
  bf16* Yl = reinterpret_cast<bf16*>(osm + pl.yl);
  bf16* Zh = reinterpret_cast<bf16*>(osm + pl.zh);
  bf16* Zl = reinterpret_cast<bf16*>(osm + pl.zl);
  float* col = reinterpret_cast<float*>(osm + pl.col);
  float* hq = reinterpret_cast<float*>(osm + pl.h);
  float* red = reinterpret_cast<float*>(osm + pl.red);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  float* Pg = P + (size_t)blockIdx.x * bstride;
  const bf16* xg = x + (size_t)blockIdx.x * xstride;
  const int NB = (r + 7) / 8, KSr = (r + 15) / 16;  // n-blocks of the columns, k-steps over r

  // the fp32 master and its hi/lo rows (padding columns zero)
  for (int e = tid; e < kHeadDim * ldp; e += kMmaOjaThreads) {
    const int i = e / ldp, j = e - i * ldp;
    const float v = j < r ? Pg[(size_t)i * r + j] : 0.f;
    if (j < r) Pf[i * ldf + j] = v;
    const bf16 hh = __float2bfloat16_rn(v);
    Ph[e] = hh;
    Pl[e] = __float2bfloat16_rn(v - __bfloat162float(hh));
  }
  for (int e = tid; e < kBlkRows * ldp; e += kMmaOjaThreads) {  // Y padding stays zero
    Yh[e] = __float2bfloat16_rn(0.f);
    Yl[e] = __float2bfloat16_rn(0.f);
  }
  auto refresh_rows = [&](int i0, int i1) {  // hi/lo rows from the master
    for (int e = i0 * r + tid; e < i1 * r; e += kMmaOjaThreads) {
      const int i = e / r, j = e - i * r;
      const float v = Pf[i * ldf + j];
      const bf16 hh = __float2bfloat16_rn(v);
      Ph[i * ldp + j] = hh;
      Pl[i * ldp + j] = __float2bfloat16_rn(v - __bfloat162float(hh));
    }
  };
  auto chunk_len = [&](int j) {
    int nc = min(min(chunk, kBlkRows), n - j);
    if (qr_every > 0) {
      const long long to_qr = qr_every - (seen + j) % qr_every;
      if (to_qr < nc) nc = (int)to_qr;
    }
    return nc;
  };
  auto stage = [&](int j, int buf) {  // rows of the chunk at j; the rest zero-filled
    const int nc = chunk_len(j);
    bf16* dst = Xs + (size_t)buf * kBlkRows * kLdX;
    for (int e = tid; e < kBlkRows * (kHeadDim / 8); e += kMmaOjaThreads) {
      const int t = e >> 4, c = e & 15;
      const bool ok = t < nc;
      cp_async16(dst + t * kLdX + c * 8, xg + (size_t)(ok ? j + t : j) * kHeadDim + c * 8,
                 ok ? 16u : 0u);
    }
    cp_async_commit();
  };
  if (n > 0) stage(0, 0);
  int buf = 0;
  const int arow = lane & 15, ahalf = lane >> 4;                     // A, ldmatrix
  const int brow = (lane & 7) + ((lane >> 4) << 3), bk = ((lane >> 3) & 1) * 8;  // B, ldmatrix
  const int trow = (lane & 7) + ((lane >> 3) & 1) * 8, tcol = (lane >> 4) * 8;   // B, .trans
  const int atrow = (lane & 7) + ((lane >> 4) << 3), atcol = ((lane >> 3) & 1) * 8;  // A, .trans
  for (int j = 0; j < n;) {
    const int nc = chunk_len(j);
    cp_async_wait<0>();
    __syncthreads();  // X of this chunk landed; the previous chunk's products are done
    if (j + nc < n) stage(j + nc, buf ^ 1);
    const bf16* X = Xs + (size_t)buf * kBlkRows * kLdX;
    const uint32_t xb = smem_u32(X);
    // ---- Y = X P : warp -> tokens 16 (w % 4) .., n-block pairs of its half
    {
      const int mb = warp & 3, half = warp >> 2, NP = (NB + 1) / 2;
      const int p0 = half ? (NP + 1) / 2 : 0, p1 = half ? NP : (NP + 1) / 2;
      float acc[4][2][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][u][e] = 0.f;
#pragma unroll 2
      for (int ks = 0; ks < kHeadDim / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(xb + (uint32_t)(((mb * 16 + arow) * kLdX + ks * 16 + ahalf * 8) * 2), a);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int pr = p0 + q;
          if (pr < p1) {
            // B[k = dim][n = column] = P[dim][column]: rows k, so .trans
            const uint32_t off =
                (uint32_t)(((ks * 16 + trow) * ldp + pr * 16 + tcol) * 2);
            uint32_t bh[4], bl[4];
            ldsm_x4_trans(smem_u32(Ph) + off, bh);
            ldsm_x4_trans(smem_u32(Pl) + off, bl);
            mma_bf16_16816(acc[q][0], a, bh[0], bh[1]);
            mma_bf16_16816(acc[q][1], a, bh[2], bh[3]);
            mma_bf16_16816(acc[q][0], a, bl[0], bl[1]);
            mma_bf16_16816(acc[q][1], a, bl[2], bl[3]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int pr = p0 + q;
        if (pr < p1) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col0 = (2 * pr + u) * 8 + 2 * t4;
            if (col0 < r) {
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int row = mb * 16 + g + 8 * h2;
                const float y0 = acc[q][u][2 * h2], y1 = acc[q][u][2 * h2 + 1];
                const uint32_t hh = pack_bf16x2(y0, y1);
                *reinterpret_cast<uint32_t*>(Yh + row * ldp + col0) = hh;
                *reinterpret_cast<uint32_t*>(Yl + row * ldp + col0) =
                    pack_bf16x2(y0 - bf_lo(hh), y1 - bf_hi(hh));
              }
            }
          }
        }
      }
    }
    __syncthreads();
    // ---- Z = X - Y P^T : warp -> tokens 16 (w % 4) .., dims 64 (w / 4) ..
    {
      const int mb = warp & 3, d0 = (warp >> 2) * 64;
      float acc[4][2][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][u][e] = 0.f;
      for (int ks = 0; ks < KSr; ++ks) {
        uint32_t ah[4], al[4];
        const uint32_t aoff = (uint32_t)(((mb * 16 + arow) * ldp + ks * 16 + ahalf * 8) * 2);
        ldsm_x4(smem_u32(Yh) + aoff, ah);
        ldsm_x4(smem_u32(Yl) + aoff, al);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // B[k = column][n = dim] = P[dim][column]: rows n
          const uint32_t off = (uint32_t)(((d0 + q * 16 + brow) * ldp + ks * 16 + bk) * 2);
          uint32_t bh[4], bl[4];
          ldsm_x4(smem_u32(Ph) + off, bh);
          ldsm_x4(smem_u32(Pl) + off, bl);
          mma_bf16_16816(acc[q][0], ah, bh[0], bh[1]);
          mma_bf16_16816(acc[q][1], ah, bh[2], bh[3]);
          mma_bf16_16816(acc[q][0], ah, bl[0], bl[1]);
          mma_bf16_16816(acc[q][1], ah, bl[2], bl[3]);
          mma_bf16_16816(acc[q][0], al, bh[0], bh[1]);
          mma_bf16_16816(acc[q][1], al, bh[2], bh[3]);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int row = mb * 16 + g + 8 * h2, d = d0 + q * 16 + u * 8 + 2 * t4;
            const uint32_t xv = *reinterpret_cast<const uint32_t*>(X + row * kLdX + d);
            const float z0 = bf_lo(xv) - acc[q][u][2 * h2], z1 = bf_hi(xv) - acc[q][u][2 * h2 + 1];
            const uint32_t hh = pack_bf16x2(z0, z1);
            *reinterpret_cast<uint32_t*>(Zh + row * kLdX + d) = hh;
            *reinterpret_cast<uint32_t*>(Zl + row * kLdX + d) =
                pack_bf16x2(z0 - bf_lo(hh), z1 - bf_hi(hh));
          }
    }
    __syncthreads();
    // ---- P += eta Z^T Y : warp -> dims 16 w .., every column
    {
      const int i0 = warp * 16;
      float acc[4][2][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][u][e] = 0.f;
      const int NP = (NB + 1) / 2;
#pragma unroll
      for (int ks = 0; ks < kBlkRows / 16; ++ks) {
        if (ks * 16 < nc) {
          // A[m = dim][k = token] = Z[token][dim]: rows k, so .trans
          const uint32_t aoff = (uint32_t)(((ks * 16 + atrow) * kLdX + i0 + atcol) * 2);
          uint32_t ah[4], al[4];
          ldsm_x4_trans(smem_u32(Zh) + aoff, ah);
          ldsm_x4_trans(smem_u32(Zl) + aoff, al);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q < NP) {
              // B[k = token][n = column] = Y[token][column]: rows k, so .trans
              const uint32_t off = (uint32_t)(((ks * 16 + trow) * ldp + q * 16 + tcol) * 2);
              uint32_t bh[4], bl[4];
              ldsm_x4_trans(smem_u32(Yh) + off, bh);
              ldsm_x4_trans(smem_u32(Yl) + off, bl);
              mma_bf16_16816(acc[q][0], ah, bh[0], bh[1]);
              mma_bf16_16816(acc[q][1], ah, bh[2], bh[3]);
              mma_bf16_16816(acc[q][0], ah, bl[0], bl[1]);
              mma_bf16_16816(acc[q][1], ah, bl[2], bl[3]);
              mma_bf16_16816(acc[q][0], al, bh[0], bh[1]);
              mma_bf16_16816(acc[q][1], al, bh[2], bh[3]);
            }
          }
        }
      }
      // the warp owns rows i0 .. i0 + 15 of P: master and hi/lo updated here
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c0 = (2 * q + u) * 8 + 2 * t4;
          if (q < NP && c0 < r) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int i = i0 + g + 8 * h2;
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (c0 + e < r) {
                  float& pp = Pf[i * ldf + c0 + e];
                  pp = fmaf(eta, acc[q][u][2 * h2 + e], pp);
                  const bf16 hh = __float2bfloat16_rn(pp);
                  Ph[i * ldp + c0 + e] = hh;
                  Pl[i * ldp + c0 + e] = __float2bfloat16_rn(pp - __bfloat162float(hh));
                }
              }
            }
          }
        }
    }
    j += nc;
    buf ^= 1;
    if (qr_every > 0 && (seen + j) % qr_every == 0) {
      __syncthreads();
      qr_rows256(Pf, r, ldf, col, hq, red);
      refresh_rows(0, kHeadDim);
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int e = tid; e < kHeadDim * r; e += kMmaOjaThreads) Pg[e] = Pf[(e / r) * ldf + e % r];
}

int oja_blocked_launch(float* P, int S, int r, long long basis_stride, const void* x,
                       int x_dtype, long long x_stride, int n, float eta, int qr_every,
                       long long tokens_seen, int chunk, cudaStream_t st) {
  const int es = x_dtype == LRKV_BF16 ? 2 : 4;
  // rows are copied in 16-byte pieces
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0 || (x_stride * es) % 16 != 0)
    return LRKV_ERR_ARG;
  if (r > 64 || r % 8 != 0) return LRKV_ERR_UNSUPPORTED;
  if (x_dtype == LRKV_BF16) {  // token rows exact in bf16: the tensor-core kernel
    const int rc = prepare_kernel((const void*)oja_chunked_mma, false);
    if (rc != LRKV_OK) return rc;
    oja_chunked_mma<<<S, kMmaOjaThreads, oja_mma_plan(r).total, st>>>(
        P, r, basis_stride, static_cast<const __nv_bfloat16*>(x), x_stride, n, eta, qr_every,
        tokens_seen, chunk);
    return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
  }
  const size_t sm = oja_blocked_smem_bytes(r, es);
  const void* fn = x_dtype == LRKV_BF16 ? (const void*)oja_blocked_kernel<__nv_bfloat16>
                                        : (const void*)oja_blocked_kernel<float>;
  const int rc = prepare_kernel(fn, false);
  if (rc != LRKV_OK) return rc;
  if (x_dtype == LRKV_BF16)
    oja_blocked_kernel<__nv_bfloat16><<<S, kOjaThreads, sm, st>>>(
        P, r, basis_stride, static_cast<const __nv_bfloat16*>(x), x_stride, n, eta, qr_every,
        tokens_seen, chunk);
  else
    oja_blocked_kernel<float><<<S, kOjaThreads, sm, st>>>(P, r, basis_stride,
                                                          static_cast<const float*>(x), x_stride,
                                                          n, eta, qr_every, tokens_seen, chunk);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

template <typename T>
static int oja2_launch_t(float* P, int S, int r, long long bs, const T* x, long long xs, int n,
                         float eta, int qr_every, long long seen, cudaStream_t st) {
  const size_t sm = oja2_smem_bytes(r, (int)sizeof(T));
  auto go = [&](auto kern) -> int {
    const int rc = prepare_kernel((const void*)kern, false);
    if (rc != LRKV_OK) return rc;
    kern<<<S, kOja2Threads, sm, st>>>(P, r, bs, x, xs, n, eta, qr_every, seen);
    return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
  };
  if (r <= 16) return go(oja2_kernel<T, 16>);
  if (r <= 32) return go(oja2_kernel<T, 32>);
  if (r <= 48) return go(oja2_kernel<T, 48>);
  return go(oja2_kernel<T, 64>);
}

static size_t oja_smem(int r) { return (size_t)(kHeadDim * (r + 1) + 5 * kHeadDim) * 4; }

int oja_launch(float* P, int S, int r, long long basis_stride, const void* x, int x_dtype,
               long long x_stride, int n, float eta, int qr_every, long long tokens_seen,
               cudaStream_t st) {
  // register-resident kernel for r <= 64 when rows can be copied in 16-byte pieces
  const int es = x_dtype == LRKV_BF16 ? 2 : 4;
  const bool aligned = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (x_stride * es) % 16 == 0;
  if (r <= 64 && aligned && n > 0) {
    if (x_dtype == LRKV_BF16)
      return oja2_launch_t(P, S, r, basis_stride, static_cast<const __nv_bfloat16*>(x), x_stride,
                           n, eta, qr_every, tokens_seen, st);
    return oja2_launch_t(P, S, r, basis_stride, static_cast<const float*>(x), x_stride, n, eta,
                         qr_every, tokens_seen, st);
  }
  const size_t sm = oja_smem(r);
  if (x_dtype == LRKV_BF16) {
    auto k = oja_kernel<__nv_bfloat16>;
    const int rc = prepare_kernel((const void*)k, false);
    if (rc != LRKV_OK) return rc;
    k<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride, static_cast<const __nv_bfloat16*>(x),
                                   x_stride, n, eta, qr_every, tokens_seen);
  } else {
    auto k = oja_kernel<float>;
    const int rc = prepare_kernel((const void*)k, false);
    if (rc != LRKV_OK) return rc;
    k<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride, static_cast<const float*>(x), x_stride, n,
                                   eta, qr_every, tokens_seen);
  }
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

int qr_launch(float* P, int S, int r, long long basis_stride, cudaStream_t st) {
  const size_t sm = oja_smem(r);
  const int rc = prepare_kernel((const void*)qr_kernel, false);
  if (rc != LRKV_OK) return rc;
  qr_kernel<<<S, kOjaThreads, sm, st>>>(P, r, basis_stride);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
