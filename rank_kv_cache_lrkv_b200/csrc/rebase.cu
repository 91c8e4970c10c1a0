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
//  1. rebase_matrix_kernel: eight CTAs per (unit, side), each staging P_new
//     and its eighth of P_old's columns in shared memory, write R^T (row j =
//     column j of R) to the workspace in fp32.
//  2. the codes, by the first of these that serves the cache:
//     rebase_codes_tc (bf16 codes, re-based ranks multiples of 16: the
//     fifth-generation tensor cores, two pages per MMA), rebase_codes_mma
//     (bf16 codes: warp-level MMAs), rebase_codes_kernel (fp32 codes, or
//     when neither plan fits: CUDA cores, one CTA per page).  Each reads
//     every latent byte once and writes it back once, rounding to the cache
//     dtype once.
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

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

// R^T rows are split over kRmSlices CTAs per (unit, side), so the small
// products spread over the GPU instead of running as one long loop per unit.
constexpr int kRmSlices = 8;
__host__ __device__ inline int rm_rows(int r) { return (r + kRmSlices - 1) / kRmSlices; }
// Shared memory of rebase_matrix_kernel for rank r: the new basis [128][r]
// and the slice's columns of the old one [128][rm_rows(r)], fp32.
inline size_t matrix_smem_bytes(int r) { return (size_t)kHeadDim * (r + rm_rows(r)) * 4; }

// R^T[j][i] = sum_d P_new[d][i] P_old[d][j] for unit (blockIdx.y, blockIdx.x),
// side blockIdx.z / kRmSlices (0 keys, 1 values), rows j of slice
// blockIdx.z % kRmSlices.  The re-basing pass that follows is launched as its
// programmatic dependent and waits for this grid before reading R.
__global__ void __launch_bounds__(kRebaseThreads) rebase_matrix_kernel(RebaseArgs a) {
  extern __shared__ __align__(16) float msm[];
  pdl_trigger();
  const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int side = blockIdx.z / kRmSlices, slice = blockIdx.z - side * kRmSlices;
  const float* Po = side ? a.Pv_old : a.Pk_old;
  const float* Pn = side ? a.Pv_new : a.Pk_new;
  if (!Po) return;
  const int r = side ? a.rv : a.rk, js = rm_rows(r);
  const int j0 = slice * js, nj = min(r, j0 + js) - j0;
  if (nj <= 0) return;
  const size_t base = (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * r;
  float* sn = msm;                  // [128][r] new basis
  float* so = msm + kHeadDim * r;   // [128][js] old basis, columns j0 ..
  const int n4 = kHeadDim * r / 4;
  for (int x = tid; x < n4; x += kRebaseThreads)
    reinterpret_cast<float4*>(sn)[x] = __ldg(reinterpret_cast<const float4*>(Pn + base) + x);
  for (int x = tid; x < kHeadDim * nj; x += kRebaseThreads) {
    const int d = x / nj, jj = x - d * nj;
    so[d * js + jj] = __ldg(Po + base + (size_t)d * r + j0 + jj);
  }
  __syncthreads();
  float* Rt = (side ? a.Rv : a.Rk) + ((size_t)b * a.H_kv + kvh) * r * r;
  // thread -> (row j, column i) of R^T; consecutive threads take consecutive
  // i, so the new basis is read along its rows and the old one broadcast
  for (int x = tid; x < nj * r; x += kRebaseThreads) {
    const int jj = x / r, i = x - jj * r;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int d = 0; d < kHeadDim; d += 2) {
      s0 = fmaf(sn[d * r + i], so[d * js + jj], s0);
      s1 = fmaf(sn[(d + 1) * r + i], so[(d + 1) * js + jj], s1);
    }
    Rt[(size_t)(j0 + jj) * r + i] = s0 + s1;
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

// ---- bf16 codes on the tensor cores
// rebase_codes_mma: persistent, one CTA per SM.  The latent pages of every
// (sequence, KV head) unit are laid end to end and each CTA takes an equal
// contiguous range.  A producer warp streams one slab per page into a ring
// of shared-memory stages with bulk copies (block-table entries resolved a
// batch of 32 pages ahead).  Three groups of four consumer warps take the
// pages in turn; in a group, warp w owns the 16 tokens of m-block w and
// every code column, and computes c'[t][n] = sum_k c[t][k] R[n][k] with
// warp-level bf16 MMAs (m16n8k16, fp32 accumulation), R split into hi + lo
// bf16 halves so the products keep about 16 mantissa bits.  A fragments
// come by ldmatrix straight from the chunk-major slab and the new codes are
// written in place.  A full page then goes back to its slab with one bulk
// store, and its stage is released once that store has read it (one store
// of the group kept in flight); a partial page goes back row by row.  Each
// group keeps R of its current unit in its own padded rows [n][k], rebuilt
// by its four warps when its pages enter a new unit.
constexpr int kRbGroups = 3;
constexpr int kRbGroupWarps = 4;
constexpr int kRbGroupThreads = 32 * kRbGroupWarps;
constexpr int kRbThreads = 32 * (1 + kRbGroups * kRbGroupWarps);
constexpr int kRbMaxStages = 16;

__host__ __device__ inline int rb_r16(int r) { return (r + 15) / 16 * 16; }
__host__ __device__ inline int rb_row(int r) { return rb_r16(r) + 8; }  // padded R row (bf16)

struct RbPlan {
  int ring, R[kRbGroups], full, empty, meta, start, flag, total;
  int rk_lo, rv_hi, rv_lo;  // offsets inside a group's R block (rk_hi at 0)
};
__host__ __device__ inline RbPlan rb_plan(int NS, int rk, int rv, int B) {
  RbPlan p;
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int at = off;
    off += bytes;
    return at;
  };
  const int slab = kLatPage * (rk + rv) * 2;
  p.ring = take(NS * slab, 128);
  const int kb = rb_r16(rk) * rb_row(rk) * 2, vb = rb_r16(rv) * rb_row(rv) * 2;
  p.rk_lo = kb;
  p.rv_hi = 2 * kb;
  p.rv_lo = 2 * kb + vb;
  for (int gi = 0; gi < kRbGroups; ++gi) p.R[gi] = take(2 * kb + 2 * vb, 16);
  p.full = take(NS * 8, 8);
  p.empty = take(NS * 8, 8);
  p.meta = take(NS * 2 * 4, 4);      // per stage: page (-1 bad), latent rows
  p.start = take((B + 1) * 4, 4);
  p.flag = take(8, 4);               // producer's and consumers' failure flags
  p.total = off;
  return p;
}

// Pages of sequence b's latent tokens (capped by the block-table row).
__device__ inline int rb_pages(const RebaseArgs& a, int b) {
  const int L = max(0, __ldcg(a.seq_len + b));
  const int n_lat = split_tokens(L, a.n_sink, a.W).lat;
  return min((n_lat + kLatPage - 1) / kLatPage, a.maxp);
}

// Bounded wait by lane 0 that also gives up once fail is set, its result
// given to the warp.
__device__ inline bool rb_wait_warp(uint64_t* bar, uint32_t parity, volatile int* fail,
                                    int lane) {
  int ok = 1;
  if (lane == 0) {
    ok = 0;
    if (!*fail) {
      if (mbar_try_wait(bar, parity)) {
        ok = 1;
      } else {
        const uint64_t t0 = global_ns();
        while (!*fail) {
          if (mbar_try_wait(bar, parity)) { ok = 1; break; }
          if (global_ns() - t0 > 2000000000ull) { *fail = 1; break; }
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__global__ void __launch_bounds__(kRbThreads, 1) rebase_codes_mma(RebaseArgs a, int NS) {
  using bf16 = __nv_bfloat16;
  extern __shared__ __align__(128) uint8_t rsm[];
  const RbPlan pl = rb_plan(NS, a.rk, a.rv, a.B);
  uint64_t* full = reinterpret_cast<uint64_t*>(rsm + pl.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(rsm + pl.empty);
  int* meta = reinterpret_cast<int*>(rsm + pl.meta);
  int* start = reinterpret_cast<int*>(rsm + pl.start);
  volatile int* fail = reinterpret_cast<volatile int*>(rsm + pl.flag);
  volatile int* cfail = fail + 1;  // set only by consumer waits
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NJ = a.rk + a.rv, slab_bytes = kLatPage * NJ * 2;

  // page prefix over sequences, one warp
  if (warp == 0) {
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    int own = 0;
    for (int b = b0; b < b1; ++b) own += rb_pages(a, b) * a.H_kv;
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int e = incl - own;
    for (int b = b0; b < b1; ++b) {
      start[b] = e;
      e += rb_pages(a, b) * a.H_kv;
    }
    if (lane == 31) start[a.B] = incl;
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);  // the consuming group's leader, once its store has read
    }
    *fail = 0;
    *cfail = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const int total = start[a.B];
  const int q = total / (int)gridDim.x, rem = total - q * (int)gridDim.x;
  const int lo = blockIdx.x * q + (blockIdx.x * rem) / gridDim.x;
  const int hi = (blockIdx.x + 1) * q + ((blockIdx.x + 1) * rem) / gridDim.x;
  const int N = hi - lo;
  if (N <= 0) return;
  auto locate = [&](int k, int& b, int& kvh, int& p) {
    int l = 0, h = a.B;
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (start[mid] <= k) l = mid; else h = mid;
    }
    b = l;
    const int pages = (start[b + 1] - start[b]) / a.H_kv;
    const int r = k - start[b];
    kvh = r / pages;
    p = r - kvh * pages;
  };

  if (warp == 0) {
    // ---------------- producer: lane l resolves page base + l of each batch
    int issued = 0;
    for (int base = 0; base < N; base += 32) {
      int page = -1, rows = 0, kvh = 0;
      if (base + lane < N) {
        int b, p;
        locate(lo + base + lane, b, kvh, p);
        const int L = max(0, __ldcg(a.seq_len + b));
        rows = min(kLatPage, split_tokens(L, a.n_sink, a.W).lat - p * kLatPage);
        page = __ldg(a.bt + (size_t)b * a.maxp + p);
        if (page < 0 || page >= a.num_pages) page = -1;
      }
      const int cnt = min(32, N - base);
      bool ok = true;
      for (int jj = 0; jj < cnt; ++jj) {
        int f = 0;
        if (lane == jj) {
          const int k = base + jj, s = k % NS, n = k / NS;
          if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
            f = 1;
          } else {
            meta[2 * s] = page;
            meta[2 * s + 1] = rows;
            if (page >= 0) {
              mbar_arrive_expect_tx(&full[s], slab_bytes);
              bulk_g2s(rsm + pl.ring + (size_t)s * slab_bytes,
                       static_cast<const bf16*>(a.codes) +
                           ((size_t)page * a.H_kv + kvh) * kLatPage * NJ,
                       slab_bytes, &full[s]);
            } else {
              *a.err = kErrBadPage;
              mbar_arrive(&full[s]);
            }
            issued = k + 1;
          }
        }
        if (__any_sync(0xffffffffu, f) || *fail || *cfail) {
          *fail = 1;
          ok = false;
          break;
        }
      }
      issued = __reduce_max_sync(0xffffffffu, issued);
      if (!ok) break;
    }
    // every copy issued has landed before the CTA may exit
    if (lane == 0)
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        mbar_wait_bounded(&full[s], (last / NS) & 1);
      }
    return;
  }

  // ---------------- consumers: group gi takes pages gi, gi + 3, ...; its
  // warp cw owns rows 16 cw .. 16 cw + 15
  const int gi = (warp - 1) / kRbGroupWarps, cw = (warp - 1) % kRbGroupWarps;
  const int gtid = cw * 32 + lane, gbar = 1 + gi;
  const bool leader = cw == 0 && lane == 0;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* Rb = rsm + pl.R[gi];
  auto Rh = [&](int sd) { return reinterpret_cast<bf16*>(Rb + (sd ? pl.rv_hi : 0)); };
  auto Rl = [&](int sd) { return reinterpret_cast<bf16*>(Rb + (sd ? pl.rv_lo : pl.rk_lo)); };
  auto side_on = [&](int sd) { return (sd ? a.Pv_old : a.Pk_old) != nullptr; };
  int cur_unit = -1;
  int pending = -1;  // leader: stage whose bulk store may still be reading it
  for (int k = gi; k < N; k += kRbGroups) {
    const int s = k % NS;
    int b, kvh, p;
    locate(lo + k, b, kvh, p);
    const int unit = b * a.H_kv + kvh;
    if (unit != cur_unit) {
      // R of the new unit as padded [n][k] rows, hi + lo, zero past the rank.
      // Every warp of the group takes this branch at the same page.
      named_bar(gbar, kRbGroupThreads);  // no warp still reads the old R
#pragma unroll 1
      for (int sd = 0; sd < 2; ++sd) {
        if (!side_on(sd)) continue;
        const int r = sd ? a.rv : a.rk, R16 = rb_r16(r), RS = rb_row(r);
        const float* Rt = (sd ? a.Rv : a.Rk) + (size_t)unit * r * r;  // Rt[k][n] = R[n][k]
        bf16* rh = Rh(sd);
        bf16* rl = Rl(sd);
        // thread -> (row kk of R^T, four columns n); eight float4 loads in
        // flight per thread before any is stored (r is a multiple of 8)
        const int n4 = R16 / 4;
        for (int x0 = gtid; x0 < R16 * n4; x0 += 8 * kRbGroupThreads) {
          float4 v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int x = x0 + u * kRbGroupThreads, kk = x / n4, n = 4 * (x - kk * n4);
            v[u] = (x < R16 * n4 && kk < r && n < r)
                       ? __ldcg(reinterpret_cast<const float4*>(Rt + (size_t)kk * r + n))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int x = x0 + u * kRbGroupThreads, kk = x / n4, n = 4 * (x - kk * n4);
            if (x < R16 * n4) {
              const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const bf16 h = __float2bfloat16_rn(e[i]);
                rh[(n + i) * RS + kk] = h;
                rl[(n + i) * RS + kk] = __float2bfloat16_rn(e[i] - __bfloat162float(h));
              }
            }
          }
        }
      }
      cur_unit = unit;
      named_bar(gbar, kRbGroupThreads);
    }
    const bool landed = rb_wait_warp(&full[s], (k / NS) & 1, cfail, lane);
    const int page = meta[2 * s], rows = meta[2 * s + 1];
    uint8_t* st = rsm + pl.ring + (size_t)s * slab_bytes;
    if (landed && page >= 0) {
      const uint32_t sbase = smem_u32(st);
      bf16* sb = reinterpret_cast<bf16*>(st);
#pragma unroll 1
      for (int sd = 0; sd < 2; ++sd) {
        if (!side_on(sd)) continue;
        const int r = sd ? a.rv : a.rk, nch = r / 8, cb = sd ? a.rk / 8 : 0;
        const int NP = rb_r16(r) / 16;            // n-block pairs = k-steps of 16
        const uint32_t rh = smem_u32(Rh(sd)), rl = smem_u32(Rl(sd));
        const int RS = rb_row(r);
        float acc[16][4];
#pragma unroll
        for (int nb = 0; nb < 16; ++nb)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[nb][i] = 0.f;
        for (int ks = 0; ks < NP; ++ks) {
          const int c = min(2 * ks + (lane >> 4), nch - 1);
          uint32_t af[4];
          ldsm_x4(sbase + (uint32_t)(((cb + c) * kLatPage + cw * 16 + (lane & 15)) * 16), af);
#pragma unroll
          for (int pr = 0; pr < 8; ++pr) {
            if (pr < NP) {
              const int o = 16 * pr + (lane & 7) + ((lane >> 4) << 3);
              const int koff = 16 * ks + ((lane >> 3) & 1) * 8;
              uint32_t bh[4], bl[4];
              ldsm_x4(rh + (uint32_t)((o * RS + koff) * 2), bh);
              ldsm_x4(rl + (uint32_t)((o * RS + koff) * 2), bl);
              mma_bf16_16816(acc[2 * pr], af, bh[0], bh[1]);
              mma_bf16_16816(acc[2 * pr + 1], af, bh[2], bh[3]);
              mma_bf16_16816(acc[2 * pr], af, bl[0], bl[1]);
              mma_bf16_16816(acc[2 * pr + 1], af, bl[2], bl[3]);
            }
          }
        }
        __syncwarp();  // every lane's reads of this side's old codes are done
#pragma unroll
        for (int nb = 0; nb < 16; ++nb) {
          if (nb < nch) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int row = cw * 16 + g + 8 * h2;
              *reinterpret_cast<uint32_t*>(sb + ((size_t)(cb + nb) * kLatPage + row) * 8 + 2 * t) =
                  pack_bf16x2(acc[nb][2 * h2], acc[nb][2 * h2 + 1]);
            }
          }
        }
      }
      if (rows < kLatPage) {
        // a partial page: only its latent rows go back, 16 bytes at a time
        __syncwarp();
        const uint4* src = reinterpret_cast<const uint4*>(st);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(a.codes) +
                                              ((size_t)page * a.H_kv + kvh) * kLatPage * NJ);
        const int c0 = side_on(0) ? 0 : a.rk / 8, c1 = side_on(1) ? NJ / 8 : a.rk / 8;
        for (int x = lane; x < (c1 - c0) * 16; x += 32) {
          const int c = c0 + x / 16, row = cw * 16 + (x & 15);
          if (row < rows) dst[c * kLatPage + row] = src[c * kLatPage + row];
        }
      }
    }
    // the group's new codes are in place (and a partial page's rows read);
    // each thread's shared-memory writes are ordered before the bulk store
    proxy_fence_smem();
    named_bar(gbar, kRbGroupThreads);
    if (leader) {
      if (landed && page >= 0 && rows >= kLatPage) {
        // a full page: the whole slab back with one bulk store
        bulk_s2g(static_cast<bf16*>(a.codes) + ((size_t)page * a.H_kv + kvh) * kLatPage * NJ,
                 st, slab_bytes);
        bulk_commit();
        bulk_wait_read<1>();  // the group's previous store has read its stage
        if (pending >= 0) mbar_arrive(&empty[pending]);
        pending = s;
      } else {
        mbar_arrive(&empty[s]);  // nothing reads this stage any more
      }
    }
  }
  if (leader) {
    bulk_wait_read<0>();
    if (pending >= 0) mbar_arrive(&empty[pending]);
    bulk_wait<0>();  // the stores are complete before the CTA exits
  }
}

// ---- bf16 codes on the fifth-generation tensor cores
// rebase_codes_tc: persistent, one CTA per SM.  The latent pages of every
// unit are laid end to end and each CTA takes an equal contiguous range,
// walked as jobs of one or two pages of one unit.  The chunk-major slab of a
// page ([chunk of 8 codes][64 tokens][16 bytes]) is already the K-major
// layout of 8 x 16-byte core matrices a tensor-memory MMA reads without
// swizzle; the two pages of a job are interleaved chunk by chunk
// ([chunk][page][64][16 B]) so that they form one M = 128 operand: core
// matrices 128 bytes apart along the tokens (SBO) and 2 KB apart along the
// codes (LBO).
//  * warp 0: the producer.  Per job one tensor load brings two consecutive
//    pages (a tensor map over the pool whose dimensions, innermost first,
//    are the 1 KB chunk row, the page, the chunk and the KV head lands them
//    interleaved); other jobs' lanes copy each page's chunks (1 KB each) with
//    bulk copies; both complete on the stage's mbarrier.  The
//    kernel is the programmatic dependent of the R launch: the producer
//    streams pages at once, every other warp waits for that grid first.
//  * warp 1: the MMA issuer.  Per job and re-based side, c'^T = R c^T as
//    tcgen05.mma (M 128 tokens, N = rank rounded up to 16, K 16) with R
//    split into hi + lo bf16 halves (about 16 mantissa bits), both into the
//    same fp32 accumulator in tensor memory (up to four in flight).
//  * warps 2..5: the epilogue.  One token row per thread (tensor-memory lane
//    = row), tcgen05.ld, rounded to bf16 once, 16-byte stores straight back
//    into the row's page; rows past a page's latent tokens are not written.
//  * warp 6: the R warp.  R^T of each unit of the range (fp32, from the
//    first launch) as hi/lo bf16 rows [k chunk][n][16 B] into one of two
//    buffers, once the MMAs of the unit before last are done.
// Every wait is bounded; on a timeout the CTA raises a shared flag, every
// role leaves its loop, the producer waits (bounded) for its copies in
// flight, and tensor memory is freed before the CTA exits.
constexpr int kRtThreads = 224;
constexpr int kRtMaxStages = 10;
constexpr int kRtWarp = 6;

__host__ __device__ inline int rt_r16(int r) { return (r + 15) / 16 * 16; }
// Tensor-memory columns of one accumulator (both sides), and of the allocation.
__host__ __device__ inline int rt_acc_cols(int rk, int rv) { return rt_r16(rk) + rt_r16(rv); }
// Accumulators in flight: as many as fit the 512 tensor-memory columns, at
// most four (the MMA runs that many jobs ahead of the epilogue).
__host__ __device__ inline int rt_nacc(int rk, int rv) {
  return min(4, 512 / rt_acc_cols(rk, rv));
}
__host__ __device__ inline int rt_tmem_cols(int rk, int rv) {
  int n = 32;
  while (n < rt_nacc(rk, rv) * rt_acc_cols(rk, rv)) n *= 2;
  return n;
}
// Job slots of the metadata ring: the producer runs at most NS + 4 jobs
// ahead of the epilogue (NS stages, at most four accumulators), so NS + 5
// slots are never overwritten before the epilogue has read them.
__host__ __device__ inline int rt_slots(int NS) { return NS + 5; }
struct RtPlan {
  int ring, rbuf, rsize, rk_lo, rv_hi, rv_lo, bars, meta, start, misc, total;
};
// R buffer: R_k^T hi, lo ([rk/8][rk16][16 B] each), then R_v^T hi, lo.
__host__ __device__ inline RtPlan rt_plan(int NS, int rk, int rv, int B) {
  RtPlan p;
  const int stage = 2 * kLatPage * (rk + rv) * 2;
  p.ring = 0;
  const int kb = (rk / 8) * rt_r16(rk) * 16, vb = (rv / 8) * rt_r16(rv) * 16;
  p.rk_lo = kb;
  p.rv_hi = 2 * kb;
  p.rv_lo = 2 * kb + vb;
  p.rsize = 2 * kb + 2 * vb;
  p.rbuf = NS * stage;
  p.bars = p.rbuf + 2 * p.rsize;
  // full, empty, accf[4], acce[4], rfull, rfree, mdone, then mfull per job slot
  p.meta = p.bars + (2 * NS + 8 + 4 + 1 + rt_slots(NS)) * 8;
  p.start = p.meta + rt_slots(NS) * 8 * 4;      // per job slot: pages[2], rows[2], kvh
  p.misc = p.start + ((B + 1 + 3) / 4 * 4) * 4;
  p.total = p.misc + 16;
  return p;
}

__global__ void __launch_bounds__(kRtThreads, 1)
    rebase_codes_tc(RebaseArgs a, int NS, const __grid_constant__ CUtensorMap tmC, int pair_tm) {
  using bf16 = __nv_bfloat16;
  extern __shared__ __align__(1024) uint8_t rt_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(rt_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const RtPlan pl = rt_plan(NS, a.rk, a.rv, a.B);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + pl.bars);
  uint64_t* empty = full + NS;
  uint64_t* accf = empty + NS;   // [4]
  uint64_t* acce = accf + 4;     // [4]
  uint64_t* rfull = acce + 4;    // [2]
  uint64_t* rfree = rfull + 2;   // [2]
  uint64_t* mdone = rfree + 2;
  uint64_t* mfull = mdone + 1;   // [NM] job metadata written
  int* meta = reinterpret_cast<int*>(sm + pl.meta);  // [NM][8]
  const int NM = rt_slots(NS);
  int* start = reinterpret_cast<int*>(sm + pl.start);
  uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sm + pl.misc);
  volatile int* fail = reinterpret_cast<volatile int*>(sm + pl.misc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NJ = a.rk + a.rv, nch = NJ / 8, stage_bytes = 2 * kLatPage * NJ * 2;
  const bool on_k = a.Pk_old != nullptr, on_v = a.Pv_old != nullptr;

  // page prefix over sequences, one warp
  if (warp == 0) {
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    int own = 0;
    for (int b = b0; b < b1; ++b) own += rb_pages(a, b) * a.H_kv;
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int e = incl - own;
    for (int b = b0; b < b1; ++b) {
      start[b] = e;
      e += rb_pages(a, b) * a.H_kv;
    }
    if (lane == 31) start[a.B] = incl;
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rfree[i], 1);
    }
    mbar_init(mdone, 1);
    for (int i = 0; i < NM; ++i) mbar_init(&mfull[i], 1);
    *fail = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const int total = start[a.B];
  const int q = total / (int)gridDim.x, rem = total - q * (int)gridDim.x;
  const int lo = blockIdx.x * q + (blockIdx.x * rem) / gridDim.x;
  const int hi = (blockIdx.x + 1) * q + ((blockIdx.x + 1) * rem) / gridDim.x;
  if (lo >= hi) return;  // uniform across the CTA
  auto locate = [&](int k, int& b, int& kvh, int& p, int& pages) {
    int l = 0, h = a.B;
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (start[mid] <= k) l = mid; else h = mid;
    }
    b = l;
    pages = (start[b + 1] - start[b]) / a.H_kv;
    const int r = k - start[b];
    kvh = r / pages;
    p = r - kvh * pages;
  };
  // job j starts at page k and holds two pages when the next page of the
  // range is in the same unit; every role walks the jobs the same way
  auto job_pages = [&](int k) {
    int b, kvh, p, pages;
    locate(k, b, kvh, p, pages);
    return (k + 1 < hi && p + 1 < pages) ? 2 : 1;
  };

  const int tcols = rt_tmem_cols(a.rk, a.rv), acols = rt_acc_cols(a.rk, a.rv);
  const int nacc = rt_nacc(a.rk, a.rv);
  if (warp == 1) {
    tmem_alloc(taddr_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *taddr_slot;

  // R^T of unit `unit` as hi/lo bf16 rows of the canonical layout: element
  // (n, k) of side sd at chunk k / 8, row n, half-word k % 8
  auto build_r = [&](int unit, int buf, int t, int nt) {
    for (int sd = 0; sd < 2; ++sd) {
      if (!(sd ? on_v : on_k)) continue;
      const int r = sd ? a.rv : a.rk, R16 = rt_r16(r);
      const float* Rt = (sd ? a.Rv : a.Rk) + (size_t)unit * r * r;  // Rt[k][n] = R[n][k]
      uint8_t* hb = sm + pl.rbuf + buf * pl.rsize + (sd ? pl.rv_hi : 0);
      uint8_t* lb = sm + pl.rbuf + buf * pl.rsize + (sd ? pl.rv_lo : pl.rk_lo);
      // item = (k chunk kc, row n): 8 values R[n][8 kc .. 8 kc + 7]
      for (int it = t; it < (r / 8) * R16; it += nt) {
        const int kc = it / R16, n = it - kc * R16;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = n < r ? __ldcg(Rt + (size_t)(8 * kc + e) * r + n) : 0.f;
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
          l[e] = pack_bf16x2(x[2 * e] - bf_lo(h[e]), x[2 * e + 1] - bf_hi(h[e]));
        }
        const size_t off = ((size_t)kc * R16 + n) * 16;
        *reinterpret_cast<uint4*>(hb + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lb + off) = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
    fence_proxy_async_smem();
  };
  auto unit_of = [&](int k) {
    int b, kvh, p, pages;
    locate(k, b, kvh, p, pages);
    return b * a.H_kv + kvh;
  };
  // The R of the range's first two units, built before the stream by every
  // warp but the producer: R comes from the grid this one depends on, the
  // codes do not, so the producer starts copying pages at once.
  int nfirst = 0;
  if (warp != 0) {
    pdl_wait();
    int cur = -1;
    for (int k = lo; k < hi && nfirst < 2; ++k) {
      int b, kvh, p, pages;
      locate(k, b, kvh, p, pages);
      const int unit = b * a.H_kv + kvh;
      if (unit == cur) continue;
      cur = unit;
      build_r(unit, nfirst, tid - 32, kRtThreads - 32);
      ++nfirst;
      k += pages - p - 1;  // to the unit's last page
    }
    named_bar(1, kRtThreads - 32);
    if (tid == 32)
      for (int m = 0; m < nfirst; ++m) mbar_arrive(&rfull[m]);
  }

  const bf16* codes_in = static_cast<const bf16*>(a.codes);
  if (warp == 0) {
    // ---------------- producer: the warp resolves pages 32 at a time (lane l
    // holds the block-table entry, latent rows and KV head of page base + l;
    // the next batch's loads are in flight while this one is issued); lane 0
    // issues the copies and publishes each job's pages for the epilogue
    const uint64_t pol = l2_evict_first_policy();
    auto resolve = [&](int kk, int& pg, int& rw, int& kv) {
      pg = -1;
      rw = 0;
      kv = 0;
      if (kk >= hi) return;
      int b, p, pages;
      locate(kk, b, kv, p, pages);
      const int L = max(0, __ldcg(a.seq_len + b));
      rw = min(kLatPage, split_tokens(L, a.n_sink, a.W).lat - p * kLatPage);
      const int page = __ldg(a.bt + (size_t)b * a.maxp + p);
      pg = (page >= 0 && page < a.num_pages) ? page : -1;
    };
    int base = lo, cpg, crw, ckv, npg, nrw, nkv;
    resolve(base + lane, cpg, crw, ckv);
    resolve(base + 32 + lane, npg, nrw, nkv);
    int issued = 0, j = 0;
    for (int k = lo; k < hi; ++j) {
      const int np = job_pages(k);
      int pg[2] = {-1, -1}, rw[2] = {0, 0}, kvh = 0;
      for (int i = 0; i < 2; ++i) {
        const int o = k + i - base;  // < 64: k < base + 32
        const int x = __shfl_sync(0xffffffffu, o < 32 ? cpg : npg, o & 31);
        const int y = __shfl_sync(0xffffffffu, o < 32 ? crw : nrw, o & 31);
        const int z = __shfl_sync(0xffffffffu, o < 32 ? ckv : nkv, o & 31);
        if (i < np) {
          pg[i] = x;
          rw[i] = y;
          kvh = i == 0 ? z : kvh;
        }
      }
      const int s = j % NS, n = j / NS;
      int ok = 1;
      if (lane == 0) {
        if (n > 0 && !tc_wait(&empty[s], (n - 1) & 1, fail)) {
          ok = 0;
        } else {
          if (pg[0] < 0 || (np > 1 && pg[1] < 0)) *a.err = kErrBadPage;
          const uint32_t bytes = (uint32_t)(((pg[0] >= 0) + (pg[1] >= 0)) * nch * 1024);
          mbar_arrive_expect_tx(&full[s], bytes);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      uint8_t* dst = sm + pl.ring + (size_t)s * stage_bytes;
      if (pair_tm && np == 2 && pg[0] >= 0 && pg[1] == pg[0] + 1) {
        // consecutive pages: one tensor load of the box (1 KB chunk, page
        // pair, every chunk) lands them already interleaved
        if (lane == 0) tma_load_4d(dst, &tmC, 0, pg[0], 0, kvh, &full[s], pol);
      } else {
        // the job's 1 KB chunk copies, spread over the lanes
        for (int x = lane; x < np * nch; x += 32) {
          const int i = x / nch, c = x - i * nch;
          if (pg[i] >= 0)
            bulk_g2s_hint(dst + (size_t)c * 2048 + i * 1024,
                          codes_in + ((size_t)pg[i] * a.H_kv + kvh) * kLatPage * NJ +
                              (size_t)c * kLatPage * 8,
                          1024, &full[s], pol);
        }
      }
      if (lane == 0) {
        int* m = meta + (j % NM) * 8;
        m[0] = pg[0];
        m[1] = pg[1];
        m[2] = rw[0];
        m[3] = rw[1];
        m[4] = kvh;
        mbar_arrive(&mfull[j % NM]);
      }
      issued = j + 1;
      k += np;
      if (k >= base + 32) {
        base += 32;
        cpg = npg; crw = nrw; ckv = nkv;
        resolve(base + 32 + lane, npg, nrw, nkv);
      }
    }
    // no copy may still be landing when the CTA exits
    if (lane == 0)
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(&full[s], (last / NS) & 1) && global_ns() - t0 < kTcTimeoutNs) {
        }
      }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    const uint32_t ring0 = smem_u32(sm + pl.ring);
    const uint32_t rb0 = smem_u32(sm + pl.rbuf);
    int cur_unit = -1, m = -1, j = 0;
    for (int k = lo; k < hi; ++j) {
      if (__shfl_sync(0xffffffffu, *fail, 0)) break;
      const int np = job_pages(k);
      const int unit = unit_of(k);
      if (unit != cur_unit) {
        if (m >= 0 && lane == 0) tc_commit(&rfree[m & 1]);
        ++m;
        cur_unit = unit;
        if (!tc_wait_warp(&rfull[m & 1], (m >> 1) & 1, fail, lane)) break;
      }
      const int s = j % NS, n = j / NS, buf = j % nacc, u = j / nacc;
      if (!tc_wait_warp(&full[s], n & 1, fail, lane)) break;
      if (u > 0 && !tc_wait_warp(&acce[buf], (u - 1) & 1, fail, lane)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sa = ring0 + s * stage_bytes;
        const uint32_t rb = rb0 + (m & 1) * pl.rsize;
        for (int sd = 0; sd < 2; ++sd) {
          if (!(sd ? on_v : on_k)) continue;
          const int r = sd ? a.rv : a.rk, R16 = rt_r16(r), cb = sd ? a.rk / 8 : 0;
          const uint32_t d = tmem + buf * acols + (sd ? rt_r16(a.rk) : 0);
          const uint32_t idesc = tc_idesc(R16);
          const uint32_t hb = rb + (sd ? pl.rv_hi : 0), lb = rb + (sd ? pl.rv_lo : pl.rk_lo);
          for (int ks = 0; ks < r / 16; ++ks) {
            // A: codes chunks cb + 2 ks, + 1; B: R^T chunks 2 ks, + 1
            const uint64_t ad = interleave_desc(sa + (cb + 2 * ks) * 2048, 2048, 128);
            const uint32_t bo = (2 * ks) * R16 * 16;
            tc_mma(d, ad, interleave_desc(hb + bo, R16 * 16, 128), idesc, ks > 0 ? 1u : 0u);
            tc_mma(d, ad, interleave_desc(lb + bo, R16 * 16, 128), idesc, 1u);
          }
        }
        tc_commit(&empty[s]);
        tc_commit(&accf[buf]);
      }
      __syncwarp();
      k += np;
    }
    // every MMA issued has completed before tensor memory is freed
    if (lane == 0) {
      tc_commit(mdone);
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(mdone, 0) && global_ns() - t0 < kTcTimeoutNs) {
      }
    }
    __syncwarp();
  } else if (warp == kRtWarp) {
    // ---------------- R warp: units 2, 3, ... of the range, in order
    int cur_unit = -1, m = -1;
    for (int k = lo; k < hi; ++k) {
      int b, kvh, p, pages;
      locate(k, b, kvh, p, pages);
      const int unit = b * a.H_kv + kvh;
      k += pages - p - 1;  // to the unit's last page
      if (unit == cur_unit) continue;
      cur_unit = unit;
      if (++m < nfirst) continue;  // built by the whole CTA
      if (!tc_wait_warp(&rfree[m & 1], ((m - 2) >> 1) & 1, fail, lane)) break;
      build_r(unit, m & 1, lane, 32);
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[m & 1]);
    }
  } else {
    // ---------------- epilogue: tensor-memory lanes 32 qd .. 32 qd + 31 = token rows
    const int qd = warp & 3, row = 32 * qd + lane, pi = row >> 6, t = row & 63;
    bf16* codes = static_cast<bf16*>(a.codes);
    int j = 0;
    for (int k = lo; k < hi; ++j) {
      const int np = job_pages(k);
      const int buf = j % nacc, u = j / nacc;
      // the job's pages, as the producer resolved them
      if (!tc_wait_warp(&mfull[j % NM], (j / NM) & 1, fail, lane)) break;
      __syncwarp();  // lane 0's acquire orders the other lanes' reads too
      const int* m = meta + (j % NM) * 8;
      const int page = pi < np ? m[pi] : -1, rows = m[2 + pi], kvh = m[4];
      if (!tc_wait_warp(&accf[buf], u & 1, fail, lane)) break;
      tc_fence_after();
      const bool write = page >= 0 && t < rows;
      bf16* dst = codes + ((size_t)(page >= 0 ? page : 0) * a.H_kv + kvh) * kLatPage * NJ;
      for (int sd = 0; sd < 2; ++sd) {
        if (!(sd ? on_v : on_k)) continue;
        const int r = sd ? a.rv : a.rk, cb = sd ? a.rk / 8 : 0;
        const uint32_t tb = tmem + ((uint32_t)(32 * qd) << 16) + buf * acols +
                            (sd ? rt_r16(a.rk) : 0);
        uint32_t v[8][16];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (16 * c < r) tmem_ld16_async(tb + 16 * c, v[c]);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (16 * c < r) tmem_wait_tie(v[c]);
        if (write) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c8 = 16 * c + 8 * h;  // r is a multiple of 8
              if (c8 < r) {
                const uint4 w = make_uint4(
                    pack_bf16x2(__uint_as_float(v[c][8 * h + 0]), __uint_as_float(v[c][8 * h + 1])),
                    pack_bf16x2(__uint_as_float(v[c][8 * h + 2]), __uint_as_float(v[c][8 * h + 3])),
                    pack_bf16x2(__uint_as_float(v[c][8 * h + 4]), __uint_as_float(v[c][8 * h + 5])),
                    pack_bf16x2(__uint_as_float(v[c][8 * h + 6]), __uint_as_float(v[c][8 * h + 7])));
                *reinterpret_cast<uint4*>(dst + ((size_t)(cb + c8 / 8) * kLatPage + t) * 8) = w;
              }
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      k += np;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

template <typename T>
int launch_rebase_t(const RebaseArgs& a, cudaStream_t st) {
  const int rmax = a.rk > a.rv ? a.rk : a.rv;
  const size_t ms = matrix_smem_bytes(rmax);
  int rc = prepare_kernel((const void*)rebase_matrix_kernel, false);
  if (rc == LRKV_OK) rc = prepare_kernel((const void*)rebase_codes_kernel<T>, false);
  if (rc != LRKV_OK) return rc;
  rebase_matrix_kernel<<<dim3(a.H_kv, a.B, 2 * kRmSlices), kRebaseThreads, ms, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // tensor-core pass: as many ring stages as fit beside R and the prefix
    int dev = 0;
    DevInfo info;
    rc = current_device_info(dev, info);
    if (rc != LRKV_OK) return rc;
    // tensor-memory kernel when both re-based ranks are multiples of 16 and
    // its plan fits: one CTA per SM, as many stages as fit
    const bool k16 = !a.Pk_old || a.rk % 16 == 0, v16 = !a.Pv_old || a.rv % 16 == 0;
    if (k16 && v16) {
      int NT = kRtMaxStages;
      while (NT >= 2 && (size_t)rt_plan(NT, a.rk, a.rv, a.B).total + 1024 > (size_t)info.optin)
        --NT;
      if (NT >= 2) {
        rc = prepare_kernel((const void*)rebase_codes_tc, false);
        if (rc != LRKV_OK) return rc;
        const size_t smem = (size_t)rt_plan(NT, a.rk, a.rv, a.B).total + 1024;
        // the code pool as [H_kv][chunk][page][1 KB chunk row] (dimensions
        // innermost first: chunk row as 256 words, page, chunk, KV head), so
        // a box of two pages lands as [chunk][page][1 KB]
        CUtensorMap tmC;
        memset(&tmC, 0, sizeof(tmC));
        int pair_tm = 0;
        if (a.num_pages >= 2) {
          const int nch = (a.rk + a.rv) / 8;
          const cuuint64_t slab = (cuuint64_t)kLatPage * (a.rk + a.rv) * 2;
          const cuuint64_t dims[4] = {(cuuint64_t)kLatPage * 4, (cuuint64_t)a.num_pages,
                                      (cuuint64_t)nch, (cuuint64_t)a.H_kv};
          const cuuint64_t strides[3] = {slab * a.H_kv, (cuuint64_t)kLatPage * 16, slab};
          const cuuint32_t box[4] = {(cuuint32_t)kLatPage * 4, 2, (cuuint32_t)nch, 1};
          pair_tm = encode_tiled(&tmC, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.codes, dims,
                                 strides, box)
                        ? 1
                        : 0;
        }
        void* args[] = {const_cast<RebaseArgs*>(&a), &NT, &tmC, &pair_tm};
        return launch_pdl((const void*)rebase_codes_tc, dim3(info.sms), dim3(kRtThreads), smem,
                          st, args) == cudaSuccess
                   ? LRKV_OK
                   : LRKV_ERR_CUDA;
      }
    }
    // otherwise warp-level MMAs: one CTA per SM; each consumer group keeps
    // one stage back for its store, so at least two stages per group
    int NS = kRbMaxStages;
    while (NS >= 2 * kRbGroups && rb_plan(NS, a.rk, a.rv, a.B).total > info.optin) --NS;
    if (NS >= 2 * kRbGroups) {
      rc = prepare_kernel((const void*)rebase_codes_mma, false);
      if (rc != LRKV_OK) return rc;
      const int smem = rb_plan(NS, a.rk, a.rv, a.B).total;
      rebase_codes_mma<<<info.sms, kRbThreads, smem, st>>>(a, NS);
      return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
    }
  }
  const size_t cs = codes_smem_bytes<T>(a.rk, a.rv);
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
