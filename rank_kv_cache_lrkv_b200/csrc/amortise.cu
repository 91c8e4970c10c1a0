// Value amortisation (LowRAM abstract: within a head values are largely
// predictable from their keys; a light per-head predictor is fitted at test
// time and residuals are stored only for the tokens it reconstructs worst).
//
// Reading taken (the pages give neither the predictor's form nor the
// selection rule): per (sequence, KV head) unit a linear map A (r_k x r_v)
// predicts the value code from the key code, c_v ~ A^T c_k, fitted by least
// squares over the unit's prompt latent tokens; each 64-token page keeps the
// residual c_v - A^T c_k of the LRKV_VA_KEEP tokens with the largest residual
// norm (ties: the earlier token).
//
// lrkv_amortise runs three launches after the prompt was compressed into a
// value-amortised cache (key codes only):
//  1. va_gram_kernel: per (unit, token split), the partial Gram matrices
//     G = C_k^T C_k and H = C_k^T C_v over the split's latent tokens, with
//     c_k read from the pages and c_v = P_v^T v computed from the prompt's
//     value rows (the value codes are never stored).
//  2. va_solve_kernel: per unit, the partials summed and G A = H solved by a
//     Cholesky factorisation in fp64 (a ridge of 1e-12 trace(G) / r_k keeps
//     a rank-deficient G solvable).
//  3. va_residual_kernel: per (page, unit), the residuals of the page's
//     tokens, the LRKV_VA_KEEP largest by norm selected, and the page's
//     residual slots written.
// Decode-time evictions keep each page's slots up to date in append_kernel.
#include "common.cuh"
#include "compress.cuh"
#include "internal.h"

namespace lrkv {

namespace {

constexpr int kVaThreads = 256;
constexpr int kVaTile = 64;      // tokens per Gram tile
constexpr int kVaSplits = 16;    // token splits per unit in the Gram pass

struct VaArgs {
  int B, H_kv, rk, rv, n_sink, W, maxp, num_pages, n;
  const uint8_t* codes;          // key codes of the amortised slabs
  uint8_t* codes_w;              // the same pool, written by the residual pass
  const int* bt;
  const int* seq_len;
  const __nv_bfloat16* v;        // prompt value rows
  long long seq_stride, head_stride;
  const float* P_v;
  long long basis_bs;
  float* A;                      // [B][H_kv][rk][rv]
  float* part;                   // [B][H_kv][kVaSplits][rk * (rk + rv)]
  int* err;
};

// Latent tokens of sequence b's prompt: the first min(seq_len, n) tokens.
__device__ inline int va_latent(const VaArgs& a, int b) {
  const int L = min(max(0, __ldcg(a.seq_len + b)), a.n);
  return split_tokens(L, a.n_sink, a.W).lat;
}

// Key code row of latent token j of unit (b, kvh) -> fp32 dst[rk]; false when
// the page is out of range.
__device__ inline bool va_key_row(const VaArgs& a, int b, int kvh, int j, float* dst, int lane,
                                  int nlanes) {
  const int pi = j / kLatPage;
  if (pi >= a.maxp) return false;
  const int page = __ldg(a.bt + (size_t)b * a.maxp + pi);
  if (page < 0 || page >= a.num_pages) return false;
  const __nv_bfloat16* slab = reinterpret_cast<const __nv_bfloat16*>(
      a.codes + ((size_t)page * a.H_kv + kvh) * va_slab_bytes(a.rk, a.rv));
  for (int c = lane; c < a.rk / 8; c += nlanes) {
    float f[8];
    unpack_chunk<__nv_bfloat16>(
        __ldg(reinterpret_cast<const uint4*>(slab) + c * kLatPage + j % kLatPage), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[8 * c + e] = f[e];
  }
  return true;
}

constexpr int kVaPerThread = 24;  // partial sums per thread
constexpr int kVaBlock = kVaPerThread * kVaThreads;

// Partial G and H of unit (blockIdx.z, blockIdx.y) over token split
// blockIdx.x % kVaSplits, outputs [blk * kVaBlock, (blk + 1) * kVaBlock) of
// the rk x (rk + rv) block [G | H] with blk = blockIdx.x / kVaSplits.
__global__ void __launch_bounds__(kVaThreads) va_gram_kernel(VaArgs a) {
  extern __shared__ __align__(16) float vsm[];
  const int split = blockIdx.x % kVaSplits, blk = blockIdx.x / kVaSplits;
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int rk = a.rk, rv = a.rv;
  float* Pv = vsm;                          // [128][rv]
  float* ck = Pv + kHeadDim * rv;           // [tile][rk]
  float* cv = ck + kVaTile * rk;            // [tile][rv]
  float* vr = cv + kVaTile * rv;            // [tile][128]
  const float* Pg = a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * rv;
  for (int x = tid; x < kHeadDim * rv; x += kVaThreads) Pv[x] = __ldg(Pg + x);
  const int lat = va_latent(a, b);
  const int per = (lat + kVaSplits - 1) / kVaSplits;
  const int j0 = split * per, j1 = min(lat, j0 + per);
  // thread -> outputs x = blk * kVaBlock + tid + 256 m of the block [G | H]
  const int NO = rk * (rk + rv), xb = blk * kVaBlock;
  float acc[kVaPerThread];
#pragma unroll
  for (int m = 0; m < kVaPerThread; ++m) acc[m] = 0.f;
  const __nv_bfloat16* vin = a.v + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  for (int t0 = j0; t0 < j1; t0 += kVaTile) {
    const int nt = min(kVaTile, j1 - t0);
    __syncthreads();  // the previous tile is consumed
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < kVaTile; t += kVaThreads / 32) {
      if (t < nt) {
        if (!va_key_row(a, b, kvh, t0 + t, ck + t * rk, lane, 32)) {
          for (int c = lane; c < rk; c += 32) ck[t * rk + c] = 0.f;
          if (lane == 0) *a.err = kErrBadPage;
        }
        const __nv_bfloat16* row = vin + (size_t)(a.n_sink + t0 + t) * kHeadDim;
        for (int d = lane; d < kHeadDim; d += 32) vr[t * kHeadDim + d] = __bfloat162float(row[d]);
      } else {
        for (int c = lane; c < rk; c += 32) ck[t * rk + c] = 0.f;
        for (int d = lane; d < kHeadDim; d += 32) vr[t * kHeadDim + d] = 0.f;
      }
    }
    __syncthreads();
    // c_v = P_v^T v for the tile's tokens
    for (int x = tid; x < kVaTile * rv; x += kVaThreads) {
      const int t = x / rv, n = x - t * rv;
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < kHeadDim; ++d) s = fmaf(vr[t * kHeadDim + d], Pv[d * rv + n], s);
      cv[x] = s;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kVaPerThread; ++m) {
      const int x = xb + tid + kVaThreads * m;
      if (x < NO) {
        const int i = x / (rk + rv), c = x - i * (rk + rv);
        const float* col = c < rk ? ck + c : cv + (c - rk);
        const int cs = c < rk ? rk : rv;
        float s = acc[m];
        for (int t = 0; t < nt; ++t) s = fmaf(ck[t * rk + i], col[t * cs], s);
        acc[m] = s;
      }
    }
  }
  float* out = a.part + (((size_t)b * a.H_kv + kvh) * kVaSplits + split) * NO;
#pragma unroll
  for (int m = 0; m < kVaPerThread; ++m) {
    const int x = xb + tid + kVaThreads * m;
    if (x < NO) out[x] = acc[m];
  }
}

// A of unit (blockIdx.y, blockIdx.x): G A = H by Cholesky in fp64.
__global__ void __launch_bounds__(kVaThreads) va_solve_kernel(VaArgs a) {
  extern __shared__ __align__(16) double dsm[];
  const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int rk = a.rk, rv = a.rv, NO = rk * (rk + rv);
  double* M = dsm;                 // [rk][rk + rv]: G | H, then L | Y
  __shared__ double ridge;
  const float* p = a.part + ((size_t)b * a.H_kv + kvh) * kVaSplits * NO;
  for (int x = tid; x < NO; x += kVaThreads) {
    double s = 0.0;
    for (int sp = 0; sp < kVaSplits; ++sp) s += (double)p[(size_t)sp * NO + x];
    M[x] = s;
  }
  __syncthreads();
  const int ld = rk + rv;
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < rk; ++i) tr += M[i * ld + i];
    ridge = 1e-12 * tr / rk + 1e-300;
  }
  __syncthreads();
  for (int i = tid; i < rk; i += kVaThreads) M[i * ld + i] += ridge;
  __syncthreads();
  // G = L L^T in place (lower triangle), column by column
  for (int j = 0; j < rk; ++j) {
    if (tid == 0) {
      double d = M[j * ld + j];
      for (int k = 0; k < j; ++k) d -= M[j * ld + k] * M[j * ld + k];
      M[j * ld + j] = sqrt(d > 0.0 ? d : 1e-300);
    }
    __syncthreads();
    for (int i = j + 1 + tid; i < rk; i += kVaThreads) {
      double s = M[i * ld + j];
      for (int k = 0; k < j; ++k) s -= M[i * ld + k] * M[j * ld + k];
      M[i * ld + j] = s / M[j * ld + j];
    }
    __syncthreads();
  }
  // forward (L Y = H) and back (L^T A = Y) substitution, one thread per column
  float* Aout = a.A + ((size_t)b * a.H_kv + kvh) * rk * rv;
  for (int n = tid; n < rv; n += kVaThreads) {
    for (int i = 0; i < rk; ++i) {
      double s = M[i * ld + rk + n];
      for (int k = 0; k < i; ++k) s -= M[i * ld + k] * M[k * ld + rk + n];
      M[i * ld + rk + n] = s / M[i * ld + i];
    }
    for (int i = rk - 1; i >= 0; --i) {
      double s = M[i * ld + rk + n];
      for (int k = i + 1; k < rk; ++k) s -= M[k * ld + i] * M[k * ld + rk + n];
      M[i * ld + rk + n] = s / M[i * ld + i];
      Aout[i * rv + n] = (float)M[i * ld + rk + n];
    }
  }
}

// Residual slots of page blockIdx.x of unit (blockIdx.z, blockIdx.y).
__global__ void __launch_bounds__(kVaThreads) va_residual_kernel(VaArgs a) {
  extern __shared__ __align__(16) float rsm_[];
  const int p = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int rk = a.rk, rv = a.rv;
  const int lat = va_latent(a, b);
  const int rows = min(kLatPage, lat - p * kLatPage);
  if (rows <= 0) return;
  const int page = __ldg(a.bt + (size_t)b * a.maxp + p);
  if (page < 0 || page >= a.num_pages) {
    if (tid == 0) *a.err = kErrBadPage;
    return;
  }
  float* Pv = rsm_;                        // [128][rv]
  float* Am = Pv + kHeadDim * rv;          // [rk][rv]
  float* ck = Am + rk * rv;                // [64][rk]
  float* vr = ck + kLatPage * rk;          // [64][128]
  float* e = vr + kLatPage * kHeadDim;     // [64][rv] residuals
  float* nrm = e + kLatPage * rv;          // [64]
  int* sel = reinterpret_cast<int*>(nrm + kLatPage);  // [16]
  const float* Pg = a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * rv;
  const float* Ag = a.A + ((size_t)b * a.H_kv + kvh) * rk * rv;
  for (int x = tid; x < kHeadDim * rv; x += kVaThreads) Pv[x] = __ldg(Pg + x);
  for (int x = tid; x < rk * rv; x += kVaThreads) Am[x] = __ldcg(Ag + x);
  const __nv_bfloat16* vin = a.v + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < kLatPage; t += kVaThreads / 32) {
    const int j = p * kLatPage + t;
    if (t < rows) {
      va_key_row(a, b, kvh, j, ck + t * rk, lane, 32);
      const __nv_bfloat16* row = vin + (size_t)(a.n_sink + j) * kHeadDim;
      for (int d = lane; d < kHeadDim; d += 32) vr[t * kHeadDim + d] = __bfloat162float(row[d]);
    }
  }
  __syncthreads();
  // e = P_v^T v - A^T c_k
  for (int x = tid; x < rows * rv; x += kVaThreads) {
    const int t = x / rv, n = x - t * rv;
    float s = 0.f;
#pragma unroll 8
    for (int d = 0; d < kHeadDim; ++d) s = fmaf(vr[t * kHeadDim + d], Pv[d * rv + n], s);
    float pr = 0.f;
    for (int k = 0; k < rk; ++k) pr = fmaf(ck[t * rk + k], Am[k * rv + n], pr);
    e[x] = s - pr;
  }
  __syncthreads();
  for (int t = tid; t < kLatPage; t += kVaThreads) {
    float s = 0.f;
    if (t < rows)
      for (int n = 0; n < rv; ++n) s = fmaf(e[t * rv + n], e[t * rv + n], s);
    nrm[t] = t < rows ? s : -1.f;
  }
  __syncthreads();
  // the LRKV_VA_KEEP largest norms (ties: the earlier row), one warp
  if (warp == 0) {
    for (int k = 0; k < kVaKeep; ++k) {
      float bv = -1.f;
      int bi = kLatPage;
      for (int t = lane; t < kLatPage; t += 32)
        if (nrm[t] > bv) { bv = nrm[t]; bi = t; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (lane == 0) {
        sel[k] = bv >= 0.f ? bi : -1;
        if (bv >= 0.f) nrm[bi] = -2.f;  // taken
      }
      __syncwarp();
    }
  }
  __syncthreads();
  uint8_t* slab = a.codes_w + ((size_t)page * a.H_kv + kvh) * va_slab_bytes(rk, rv);
  __nv_bfloat16* res = reinterpret_cast<__nv_bfloat16*>(slab + (size_t)kLatPage * rk * 2);
  int* sidx = reinterpret_cast<int*>(slab + (size_t)kLatPage * rk * 2 + kVaKeep * rv * 2);
  float* snrm = reinterpret_cast<float*>(sidx + kVaKeep);
  // residual rows of the slots: [rv / 8][16][8] bf16
  for (int x = tid; x < kVaKeep * rv; x += kVaThreads) {
    const int sl = x / rv, n = x - sl * rv, t = sel[sl];
    res[((n >> 3) * kVaKeep + sl) * 8 + (n & 7)] =
        __float2bfloat16_rn(t >= 0 ? e[t * rv + n] : 0.f);
  }
  if (tid < kVaKeep) {
    const int t = sel[tid];
    sidx[tid] = t;
    float s = -1.f;
    if (t >= 0) {
      s = 0.f;
      for (int n = 0; n < rv; ++n) s = fmaf(e[t * rv + n], e[t * rv + n], s);
    }
    snrm[tid] = s;
  }
}

inline size_t gram_smem(int rk, int rv) {
  return ((size_t)kHeadDim * rv + (size_t)kVaTile * (rk + rv) + (size_t)kVaTile * kHeadDim) * 4;
}
inline size_t residual_smem(int rk, int rv) {
  return ((size_t)kHeadDim * rv + (size_t)rk * rv + (size_t)kLatPage * rk +
          (size_t)kLatPage * kHeadDim + (size_t)kLatPage * rv + kLatPage + kVaKeep) * 4;
}

}  // namespace

size_t amortise_workspace_bytes(int B, int H_kv, int rk, int rv) {
  return 256 + (size_t)B * H_kv * kVaSplits * rk * (rk + rv) * 4;
}

int amortise_launch(const lrkv_cache& c, const void* v, int n, long long seq_stride,
                    long long head_stride, const float* P_v, long long basis_bs, float* A,
                    void* ws, cudaStream_t st) {
  VaArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.rk = c.rank_k; a.rv = c.rank_v;
  a.n_sink = c.n_sink; a.W = c.window; a.maxp = c.max_pages_per_seq; a.num_pages = c.num_pages;
  a.n = n;
  a.codes = static_cast<const uint8_t*>(c.codes);
  a.codes_w = static_cast<uint8_t*>(c.codes);
  a.bt = c.block_table; a.seq_len = c.seq_len;
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.seq_stride = seq_stride; a.head_stride = head_stride;
  a.P_v = P_v; a.basis_bs = basis_bs; a.A = A;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.err = reinterpret_cast<int*>(w);
  a.part = reinterpret_cast<float*>(w + 256);
  int rc = prepare_kernel((const void*)va_gram_kernel, false);
  if (rc == LRKV_OK) rc = prepare_kernel((const void*)va_solve_kernel, false);
  if (rc == LRKV_OK) rc = prepare_kernel((const void*)va_residual_kernel, false);
  if (rc != LRKV_OK) return rc;
  const int nblk = (a.rk * (a.rk + a.rv) + kVaBlock - 1) / kVaBlock;
  va_gram_kernel<<<dim3(kVaSplits * nblk, a.H_kv, a.B), kVaThreads, gram_smem(a.rk, a.rv),
                   st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  va_solve_kernel<<<dim3(a.H_kv, a.B), kVaThreads,
                    (size_t)a.rk * (a.rk + a.rv) * sizeof(double), st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  va_residual_kernel<<<dim3(a.maxp, a.H_kv, a.B), kVaThreads, residual_smem(a.rk, a.rv), st>>>(
      a);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
