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
#include <type_traits>

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

template <typename T>
int launch_rebase_t(const RebaseArgs& a, cudaStream_t st) {
  const int rmax = a.rk > a.rv ? a.rk : a.rv;
  const size_t ms = matrix_smem_bytes(rmax);
  int rc = prepare_kernel((const void*)rebase_matrix_kernel, false);
  if (rc == LRKV_OK) rc = prepare_kernel((const void*)rebase_codes_kernel<T>, false);
  if (rc != LRKV_OK) return rc;
  rebase_matrix_kernel<<<dim3(a.H_kv, a.B, 2), kRebaseThreads, ms, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // tensor-core pass: as many ring stages as fit beside R and the prefix
    int dev = 0;
    DevInfo info;
    rc = current_device_info(dev, info);
    if (rc != LRKV_OK) return rc;
    // one CTA per SM; each consumer group keeps one stage back for its
    // store, so at least two stages per group
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
