// Re-basing of the stored latent codes after the bases changed.
//
// The pages adapt the basis online with Oja's rule (OjaKV page, online
// subspace adaptation) and leave open what becomes of codes stored under the
// old basis.  Here a stored code c stands for its rank-r reconstruction
// P_old c, and re-basing replaces it with that vector's code under the new
// basis: c' = P_new^T (P_old c) = R c with R = P_new^T P_old (r x r per
// (sequence, KV head) unit and side).
//
// Two launches:
//  1. rebase_matrix_kernel: one CTA per (unit, side) stages P_old and P_new
//     in shared memory and writes R^T (row j = column j of R) to the
//     workspace in fp32.
//  2. rebase_codes_kernel: one CTA per (page of a sequence, KV head).  It
//     reads seq_len, skips pages past the sequence's latent tokens, brings
//     the page's slab into shared memory as fp32 rows, multiplies each
//     token's code by R for each side being re-based, rounds to the cache
//     dtype once, and writes the slab back in place with 16-byte stores.
//     The work is small next to a decode step's stream (every latent byte
//     is read and written once, plus r multiply-adds per code element), so
//     it runs on the CUDA cores.
#include "common.cuh"
#include "internal.h"

namespace lrkv {

namespace {

constexpr int kRebaseThreads = 256;

struct RebaseArgs {
  int B, H_kv, rk, rv, n_sink, W, maxp, num_pages;
  void* codes;
  const int* bt;
  const int* seq_len;
  const float *Pk_old, *Pk_new, *Pv_old, *Pv_new;  // a side is skipped when its old basis is null
  long long basis_bs;
  int* err;
  float *Rk, *Rv;  // [B][H_kv][r][r], R^T per unit
};

// Shared memory of rebase_matrix_kernel for rank r: both bases [128][r] fp32.
inline size_t matrix_smem_bytes(int r) { return (size_t)2 * kHeadDim * r * 4; }

// R^T[j][i] = sum_d P_new[d][i] P_old[d][j] for unit (blockIdx.y, blockIdx.x),
// side blockIdx.z (0 keys, 1 values).
__global__ void __launch_bounds__(kRebaseThreads, 1) rebase_matrix_kernel(RebaseArgs a) {
  extern __shared__ __align__(16) float msm[];
  const int kvh = blockIdx.x, b = blockIdx.y, side = blockIdx.z, tid = threadIdx.x;
  const float* Po = side ? a.Pv_old : a.Pk_old;
  const float* Pn = side ? a.Pv_new : a.Pk_new;
  if (!Po) return;
  const int r = side ? a.rv : a.rk;
  const size_t base = (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * r;
  float* so = msm;                  // [128][r] old basis
  float* sn = msm + kHeadDim * r;   // [128][r] new basis
  const int n4 = kHeadDim * r / 4;
  for (int x = tid; x < n4; x += kRebaseThreads) {
    reinterpret_cast<float4*>(so)[x] = __ldg(reinterpret_cast<const float4*>(Po + base) + x);
    reinterpret_cast<float4*>(sn)[x] = __ldg(reinterpret_cast<const float4*>(Pn + base) + x);
  }
  __syncthreads();
  float* Rt = (side ? a.Rv : a.Rk) + ((size_t)b * a.H_kv + kvh) * r * r;
  // thread -> (row j, column i) of R^T; consecutive threads take consecutive
  // i, so the new basis is read along its rows and the old one broadcast
  for (int x = tid; x < r * r; x += kRebaseThreads) {
    const int j = x / r, i = x - j * r;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int d = 0; d < kHeadDim; d += 2) {
      s0 = fmaf(sn[d * r + i], so[d * r + j], s0);
      s1 = fmaf(sn[(d + 1) * r + i], so[(d + 1) * r + j], s1);
    }
    Rt[x] = s0 + s1;
  }
}

// Shared memory of rebase_codes_kernel: the slab as fp32 rows
// [64][r_k + r_v + 1] (the odd row length keeps the transposing writes free
// of bank conflicts), the re-based slab in the cache's chunk-major layout,
// and R^T of one side at a time.
template <typename T>
inline size_t codes_smem_bytes(int rk, int rv) {
  const int rmax = rk > rv ? rk : rv;
  return (size_t)kLatPage * (rk + rv + 1) * 4 + (size_t)kLatPage * (rk + rv) * sizeof(T) +
         (size_t)rmax * rmax * 4;
}

template <typename T>
__global__ void __launch_bounds__(kRebaseThreads, 1) rebase_codes_kernel(RebaseArgs a) {
  constexpr int CE = Elem<T>::CE;
  extern __shared__ __align__(16) float csm[];
  const int p = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int NJ = a.rk + a.rv, nch = NJ / CE, XS = NJ + 1;
  // latent tokens of this page
  const int L = __ldg(a.seq_len + b);
  const int n_lat = split_tokens(L < 0 ? 0 : L, a.n_sink, a.W).lat;
  const int rows = min(kLatPage, n_lat - p * kLatPage);
  if (rows <= 0) return;
  const int page = __ldg(a.bt + (size_t)b * a.maxp + p);
  if (page < 0 || page >= a.num_pages) {
    if (tid == 0) *a.err = kErrBadPage;
    return;
  }
  float* x = csm;                                                          // [64][XS] fp32
  T* y = reinterpret_cast<T*>(x + ((kLatPage * XS + 3) & ~3));             // [nch][64][CE]
  float* Rt = reinterpret_cast<float*>(y + (size_t)kLatPage * NJ);         // [r][r] R^T
  T* slab = static_cast<T*>(a.codes) + ((size_t)page * a.H_kv + kvh) * kLatPage * NJ;
  const uint4* src = reinterpret_cast<const uint4*>(slab);
  // the slab, chunk-major: 16-byte word w holds chunk w / 64 of token w % 64
  for (int w = tid; w < nch * kLatPage; w += kRebaseThreads) {
    const uint4 u = src[w];
    reinterpret_cast<uint4*>(y)[w] = u;  // kept: the side not re-based goes back as it was
    const int ch = w / kLatPage, t = w - ch * kLatPage;
    unpack_chunk<T>(u, x + t * XS + ch * CE);
  }
  const size_t unit = (size_t)b * a.H_kv + kvh;
  // c'[t][i] = sum_j R[i][j] c[t][j] per side; thread -> (token, column i)
#pragma unroll 1
  for (int side = 0; side < 2; ++side) {
    if (!(side ? a.Pv_old : a.Pk_old)) continue;
    const int r = side ? a.rv : a.rk, off = side ? a.rk : 0;
    __syncthreads();  // the slab is staged; R^T of the previous side is no longer read
    const float4* s4 = reinterpret_cast<const float4*>((side ? a.Rv : a.Rk) + unit * r * r);
    for (int w = tid; w < r * r / 4; w += kRebaseThreads)
      reinterpret_cast<float4*>(Rt)[w] = __ldcg(s4 + w);
    __syncthreads();
    // thread -> (group of kTok tokens, column i): one R^T load feeds kTok
    // multiply-adds, the token rows are broadcast across the warp
    constexpr int kTok = 8;
    const int ng = (rows + kTok - 1) / kTok;
    for (int q = tid; q < ng * r; q += kRebaseThreads) {
      const int tg = q / r, i = q - tg * r, t0 = tg * kTok;
      const float* c = x + t0 * XS + off;
      float acc[kTok];
#pragma unroll
      for (int k = 0; k < kTok; ++k) acc[k] = 0.f;
#pragma unroll 4
      for (int j = 0; j < r; ++j) {
        const float rj = Rt[j * r + i];
#pragma unroll
        for (int k = 0; k < kTok; ++k) acc[k] = fmaf(rj, c[k * XS + j], acc[k]);
      }
      const int col = off + i;
#pragma unroll
      for (int k = 0; k < kTok; ++k)
        if (t0 + k < rows)
          y[((size_t)(col / CE) * kLatPage + t0 + k) * CE + col % CE] = from_f<T>(acc[k]);
    }
  }
  __syncthreads();
  // write back the rows that hold latent tokens, 16 bytes at a time
  uint4* dst = reinterpret_cast<uint4*>(slab);
  for (int w = tid; w < nch * kLatPage; w += kRebaseThreads) {
    const int t = w % kLatPage;
    if (t < rows) dst[w] = reinterpret_cast<const uint4*>(y)[w];
  }
}

template <typename T>
int launch_rebase_t(const RebaseArgs& a, cudaStream_t st) {
  const int rmax = a.rk > a.rv ? a.rk : a.rv;
  const size_t ms = matrix_smem_bytes(rmax);
  if (cudaFuncSetAttribute(rebase_matrix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ms) != cudaSuccess)
    return LRKV_ERR_CUDA;
  rebase_matrix_kernel<<<dim3(a.H_kv, a.B, 2), kRebaseThreads, ms, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  const size_t cs = codes_smem_bytes<T>(a.rk, a.rv);
  if (cudaFuncSetAttribute(rebase_codes_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)cs) != cudaSuccess)
    return LRKV_ERR_CUDA;
  rebase_codes_kernel<T><<<dim3(a.maxp, a.H_kv, a.B), kRebaseThreads, cs, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace

size_t rebase_workspace_bytes(int B, int H_kv, int rk, int rv) {
  return 256 + ((size_t)B * H_kv * ((size_t)rk * rk + (size_t)rv * rv)) * 4;
}

int rebase_launch(const lrkv_cache& c, const float* Pk_old, const float* Pk_new,
                  const float* Pv_old, const float* Pv_new, long long basis_bs, void* ws,
                  cudaStream_t st) {
  RebaseArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.rk = c.rank_k; a.rv = c.rank_v;
  a.n_sink = c.n_sink; a.W = c.window; a.maxp = c.max_pages_per_seq; a.num_pages = c.num_pages;
  a.codes = c.codes; a.bt = c.block_table; a.seq_len = c.seq_len;
  a.Pk_old = Pk_old; a.Pk_new = Pk_new; a.Pv_old = Pv_old; a.Pv_new = Pv_new;
  a.basis_bs = basis_bs;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.err = reinterpret_cast<int*>(w);
  a.Rk = reinterpret_cast<float*>(w + 256);
  a.Rv = a.Rk + (size_t)a.B * a.H_kv * a.rk * a.rk;
  if (c.dtype == LRKV_BF16) return launch_rebase_t<__nv_bfloat16>(a, st);
  return launch_rebase_t<float>(a, st);
}

}  // namespace lrkv
