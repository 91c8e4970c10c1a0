// bf16 prefill compress on the fifth-generation tensor cores.
//
// c = x P for every input token that goes straight to a latent page (Half
// the Memory, section 04: each 128-dim key and value is projected to an
// r-dim code and only the code is stored).  Per 128-token tile of a
// (sequence, KV head) unit this is two dense contractions,
// [128 x 128] K rows x P_k and [128 x 128] V rows x P_v, bf16 operands and
// fp32 accumulation.  The basis is rounded to bf16 once: on the workloads'
// inputs the stored codes then differ from the exact ones by at most
// 6.1e-3 of each row's largest code, against 3.9e-3 with P split into
// hi + lo halves (the code's own bf16 rounding dominates both; the bar is
// 1e-2).  The single half keeps the basis buffers small, so the ring holds
// one more 32 KB stage: with a tile taking about 5 us to land under a full
// stream, the bytes in flight set this kernel's pace.
//
// Persistent: one CTA per SM.  The tiles of every unit are laid end to end
// and each CTA takes an equal contiguous range (ragged prompts balance).  A
// CTA walks its range as a sequence of jobs, job = (tile, side K|V):
//  * warp 0, one lane: the tensor-memory-access producer.  Per job it loads
//    the tile's 128 rows of one side as two boxes of 64 dims (128-byte
//    swizzle) through a tensor map over this GPU's own input (no cluster,
//    no multicast) into a ring of 32 KB stages, completing on mbarriers,
//    and prefetches the rows of the jobs up to eight ahead into L2.
//  * warp 6: the basis warp.  For each unit of the CTA's range, in order, it
//    writes P^T of the unit (bf16) into one of two shared-memory buffers in
//    the 128-byte-swizzled K-major layout, fences it for the async proxy
//    and marks the buffer full; it refills a buffer once the MMAs of the
//    unit before last have completed.  The basis loads stay off the MMA
//    warp's path.
//  * warp 1: the MMA issuer.  Per job one lane issues 8 tcgen05.mma
//    (M 128, N = rank rounded up to 16, K 16 each) into one of two TMEM
//    accumulators, then commits to the stage's "empty" barrier and the
//    accumulator's "full" barrier; after a unit's last job it commits to
//    that unit's basis buffer's "free" barrier.
//  * warps 2..5: the epilogue.  Warp w reads TMEM lanes 32 (w % 4) ..
//    +31, i.e. one token row per thread, with tcgen05.ld, rounds to bf16 and
//    stores 16-byte chunks straight into the chunk-major code pages (a warp
//    writes 32 consecutive rows of one chunk: 512 contiguous bytes), then
//    releases the accumulator.
// Every wait is bounded; on a timeout the CTA raises a shared flag, every
// role leaves its loop, the producer waits (bounded) for its copies in
// flight, and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "compress.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace lrkv {

namespace {

constexpr int kTcRows = 128;                       // tokens per tile (MMA M)
constexpr int kTcThreads = 224;                    // 7 warps
constexpr int kTcHalfBytes = kTcRows * 128;        // one 64-dim box: 128 rows x 128 B
constexpr int kTcStageBytes = 2 * kTcHalfBytes;    // one side of one tile
constexpr int kTcMaxStages = 6;
constexpr int kTcPrefetch = 8;                     // jobs whose rows are prefetched to L2
constexpr int kBasisWarp = 6;
constexpr int kTcAccCols = 128;                    // TMEM columns per accumulator
constexpr int kTcAcc = 4;                          // accumulators in flight
constexpr int kTcTmemCols = kTcAcc * kTcAccCols;

struct TcPlan {
  int stages, basis, bsize, bars, prefix, misc, total;
};
// Byte offsets of the kernel's shared memory from a 1024-aligned base.  A
// basis buffer holds P_k^T ([2 halves][NK][128 B]), then P_v^T; there are
// NB (two when they fit, else one).
__host__ __device__ inline TcPlan tc_plan(int NS, int NK, int NV, int B, int NB) {
  TcPlan p;
  p.stages = 0;
  p.basis = NS * kTcStageBytes;
  p.bsize = 2 * (NK + NV) * 128;
  p.bars = p.basis + NB * p.bsize;      // mbarriers
  p.prefix = p.bars + (2 * NS + 2 * kTcAcc + 5) * 8;  // start, L0, row lo, row hi: 4 x (B + 1)
  p.misc = p.prefix + 4 * (B + 1) * 4;  // TMEM address, fail flag
  p.total = p.misc + 16;
  return p;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    bulk_compress_tc(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, AppendArgs a, int NS, int NK,
                     int NV, int NB) {
  using bf16 = __nv_bfloat16;
  extern __shared__ __align__(1024) uint8_t tsm_raw[];
  // dynamic shared memory is only 16-byte aligned by contract: align to 1024
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const TcPlan pl = tc_plan(NS, NK, NV, a.B, NB);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + pl.bars);
  uint64_t* empty = full + NS;
  uint64_t* accf = empty + NS;   // [kTcAcc]
  uint64_t* acce = accf + kTcAcc; // [kTcAcc]
  uint64_t* mdone = acce + kTcAcc;  // MMA drain
  uint64_t* bfull = mdone + 1;   // [2] basis buffer written
  uint64_t* bfree = bfull + 2;   // [2] basis buffer no longer read
  int* start = reinterpret_cast<int*>(sm + pl.prefix);
  int* sL0 = start + (a.B + 1);
  int* srlo = sL0 + (a.B + 1);
  int* srhi = srlo + (a.B + 1);
  uint32_t* taddr_slot = reinterpret_cast<uint32_t*>(sm + pl.misc);
  volatile int* fail = reinterpret_cast<volatile int*>(sm + pl.misc + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // tile prefix over sequences (tiles per unit = ceil(rows / 128)), one warp
  if (warp == 0) {
    const int per = (a.B + 31) / 32;
    const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
    int own = 0;
    for (int b = b0; b < b1; ++b) {
      int L0, rl, rh;
      bulk_rows(a, b, L0, rl, rh);
      sL0[b] = L0;
      srlo[b] = rl;
      srhi[b] = rh;
      own += (rh - rl + kTcRows - 1) / kTcRows * a.H_kv;
    }
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int e = incl - own;
    for (int b = b0; b < b1; ++b) {
      start[b] = e;
      e += (srhi[b] - srlo[b] + kTcRows - 1) / kTcRows * a.H_kv;
    }
    if (lane == 31) start[a.B] = incl;
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kTcAcc; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], 4);
    }
    mbar_init(mdone, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bfree[i], 1);
    }
    *fail = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const int total = start[a.B];
  const int lo = bulk_range_lo(blockIdx.x, total, gridDim.x);
  const int hi = bulk_range_lo(blockIdx.x + 1, total, gridDim.x);
  if (lo >= hi) return;  // uniform across the CTA
  // jobs: (tile, side) pairs; value-amortised caches store key codes only
  const int sides = a.va ? 1 : 2;
  const int njobs = sides * (hi - lo);

  if (warp == 1) {
    tmem_alloc(taddr_slot, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *taddr_slot;

  // P^T of unit (b, kvh) into basis buffer `buf` (bf16), rows past the rank
  // zero; item = (16-byte chunk kc of 8 dims, code column n), consecutive
  // threads on consecutive n (coalesced reads of P's rows)
  auto build_basis = [&](int b, int kvh, int buf, int t, int nt) {
    for (int sd = 0; sd < 2; ++sd) {
      const int r = sd ? a.rv : a.rk, N = sd ? NV : NK;
      const float* P = (sd ? a.P_v : a.P_k) + (size_t)b * a.basis_bs +
                       (size_t)kvh * kHeadDim * r;
      uint8_t* base = sm + pl.basis + buf * pl.bsize + (sd ? 2 * NK * 128 : 0);
#pragma unroll 4
      for (int it = t; it < 16 * N; it += nt) {
        const int n = it % N, kc = it / N;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = n < r ? __ldg(P + (size_t)(8 * kc + e) * r + n) : 0.f;
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
        const int half = kc >> 3, c = kc & 7;
        const size_t off = (size_t)half * N * 128 + (size_t)(n >> 3) * 1024 + (n & 7) * 128 +
                           ((c ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(base + off) = make_uint4(h[0], h[1], h[2], h[3]);
      }
    }
    fence_proxy_async_smem();
  };

  // tile index -> (sequence, KV head, tile within the unit)
  auto locate = [&](int k, int& b, int& kvh, int& i) {
    int l = 0, h = a.B;
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (start[mid] <= k) l = mid; else h = mid;
    }
    b = l;
    const int tiles = (start[b + 1] - start[b]) / a.H_kv;
    const int r = k - start[b];
    kvh = r / tiles;
    i = r - kvh * tiles;
  };

  // The bases of the range's first NB units, built by every thread of the
  // CTA before the stream of tiles starts (the basis warp alone, under the
  // stream, would take many dependent round trips); later units by the
  // basis warp in the background.
  int nfirst = 0;
  {
    int cur = -1;
    for (int k = lo; k < hi && nfirst < NB; ++k) {
      int b, kvh, i;
      locate(k, b, kvh, i);
      const int unit = b * a.H_kv + kvh;
      if (unit == cur) continue;
      cur = unit;
      build_basis(b, kvh, nfirst, tid, kTcThreads);
      ++nfirst;
      k += (start[b + 1] - start[b]) / a.H_kv - i - 1;  // to the unit's last tile
    }
  }
  __syncthreads();
  if (tid == 0)
    for (int m = 0; m < nfirst; ++m) mbar_arrive(&bfull[m]);

  if (warp == 0) {
    // ---------------- producer
    int issued = 0, pf = 0;
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      for (int j = 0; j < njobs; ++j) {
        const int s = j % NS, n = j / NS;
        if (n > 0 && !tc_wait(&empty[s], (n - 1) & 1, fail)) break;
        int b, kvh, i;
        locate(lo + j / sides, b, kvh, i);
        const int t0 = srlo[b] + i * kTcRows;
        uint8_t* dst = sm + pl.stages + (size_t)s * kTcStageBytes;
        const CUtensorMap* tm = (j % sides) ? &tmV : &tmK;
        mbar_arrive_expect_tx(&full[s], kTcStageBytes);
        tma_load_4d(dst, tm, 0, t0, kvh, b, &full[s], pol);
        tma_load_4d(dst + kTcHalfBytes, tm, 64, t0, kvh, b, &full[s], pol);
        issued = j + 1;
        // the rows of the jobs up to kTcPrefetch ahead go to L2 now, so
        // their loads land from L2 when a stage frees
        for (; pf <= j + kTcPrefetch && pf < njobs; ++pf) {
          if (pf < NS) continue;  // loaded right away
          int pb, pk, pi;
          locate(lo + pf / sides, pb, pk, pi);
          const CUtensorMap* ptm = (pf % sides) ? &tmV : &tmK;
          tma_prefetch_4d(ptm, 0, srlo[pb] + pi * kTcRows, pk, pb);
          tma_prefetch_4d(ptm, 64, srlo[pb] + pi * kTcRows, pk, pb);
        }
      }
      // no copy may still be landing when the CTA exits (immediate when the
      // MMA warp consumed them all)
      for (int s = 0; s < NS && s < issued; ++s) {
          const int last = s + ((issued - 1 - s) / NS) * NS;
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(&full[s], (last / NS) & 1) && global_ns() - t0 < kTcTimeoutNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    const uint32_t stage0 = smem_u32(sm + pl.stages);
    const uint32_t basis0 = smem_u32(sm + pl.basis);
    int cur_unit = -1, m = -1;
    for (int j = 0; j < njobs; ++j) {
      if (__shfl_sync(0xffffffffu, *fail, 0)) break;
      const int side = j % sides;
      if (side == 0) {
        int b, kvh, i;
        locate(lo + j / sides, b, kvh, i);
        const int unit = b * a.H_kv + kvh;
        if (unit != cur_unit) {
          // the unit before is done once its MMAs complete: its buffer may refill
          if (m >= 0 && lane == 0) tc_commit(&bfree[m % NB]);
          ++m;
          cur_unit = unit;
          if (!tc_wait_warp(&bfull[m % NB], (m / NB) & 1, fail, lane)) break;
        }
      }
      const int s = j % NS, n = j / NS, buf = j % kTcAcc, u = j / kTcAcc;
      if (!tc_wait_warp(&full[s], n & 1, fail, lane)) break;
      if (u > 0 && !tc_wait_warp(&acce[buf], (u - 1) & 1, fail, lane)) break;
      tc_fence_after();
      if (lane == 0) {
        const int N = side ? NV : NK;
        const uint32_t bb = basis0 + (m % NB) * pl.bsize + (side ? 2 * NK * 128 : 0);
        const uint32_t idesc = tc_idesc(N);
        const uint32_t d = tmem + buf * kTcAccCols;
        const uint32_t sa = stage0 + s * kTcStageBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * kTcHalfBytes + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * N * 128 + (kk & 3) * 32;
          tc_mma(d, sw128_desc(sa + koff), sw128_desc(bb + boff), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        tc_commit(&accf[buf]);
      }
      __syncwarp();
    }
    // every MMA issued has completed before TMEM is freed
    if (lane == 0) {
      tc_commit(mdone);
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(mdone, 0) && global_ns() - t0 < kTcTimeoutNs) {
      }
    }
    __syncwarp();
  } else if (warp == kBasisWarp) {
    // ---------------- basis warp: the bases of units 1, 2, ... of the range,
    // in order, into buffer m % NB once the MMAs of unit m - NB are done
    int cur_unit = -1, m = -1;
    for (int k = lo; k < hi; ++k) {
      int b, kvh, i;
      locate(k, b, kvh, i);
      const int unit = b * a.H_kv + kvh;
      if (unit == cur_unit) continue;
      cur_unit = unit;
      if (++m < nfirst) continue;  // built by the whole CTA
      if (m >= NB && !tc_wait_warp(&bfree[m % NB], ((m - NB) / NB) & 1, fail, lane)) break;
      build_basis(b, kvh, m % NB, lane, 32);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bfull[m % NB]);
    }
  } else {
    // ---------------- epilogue: TMEM lanes 32 q .. 32 q + 31 = token rows
    const int q = warp & 3, row = 32 * q + lane;
    bf16* codes = static_cast<bf16*>(a.codes);
    // this thread's row of tile k -> (KV head, latent index, page); the page
    // of the next tile is looked up while the current one is stored
    auto row_of = [&](int k, int& kvh_, int& jlat_, int& page_) {
      int b, i;
      locate(k, b, kvh_, i);
      const int rin = srlo[b] + i * kTcRows + row;
      jlat_ = sL0[b] + rin - a.n_sink;
      page_ = rin < srhi[b] ? latent_page(a, b, jlat_) : -1;
    };
    int page = -1, jlat = 0, kvh = 0, npage = -1, njlat = 0, nkvh = 0;
    row_of(lo, nkvh, njlat, npage);
    for (int j = 0; j < njobs; ++j) {
      const int side = j % sides, buf = j % kTcAcc, u = j / kTcAcc;
      if (side == 0) {
        page = npage;
        jlat = njlat;
        kvh = nkvh;
        if (lo + j / sides + 1 < hi) row_of(lo + j / sides + 1, nkvh, njlat, npage);
      }
      if (!tc_wait_warp(&accf[buf], u & 1, fail, lane)) break;
      tc_fence_after();
      const int r = side ? a.rv : a.rk;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * kTcAccCols;
      // every column group of the row in flight at once, then one wait
      uint32_t v[8][16];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (16 * c < r) tmem_ld16_async(tbase + 16 * c, v[c]);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (16 * c < r) tmem_wait_tie(v[c]);
      if (a.q8) {
        // per-token int8 (r is a multiple of 16): the row's max |c| sets the
        // scale, the codes follow under it
        float mx = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (16 * c < r)
#pragma unroll
            for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(__uint_as_float(v[c][e])));
        const float sc = __fdiv_rn(mx, 127.f);
        uint8_t* cb = static_cast<uint8_t*>(a.codes);
        if (page >= 0) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (16 * c < r) {
              uint32_t w[4];
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                uint32_t x = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  x |= (static_cast<uint32_t>(q8_code(__uint_as_float(v[c][4 * e4 + e]), sc)) &
                        0xffu)
                       << (8 * e);
                w[e4] = x;
              }
              *reinterpret_cast<uint4*>(cb + q8_code_off(a, page, kvh, jlat, 16 * c, side)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          *reinterpret_cast<float*>(cb + q8_scale_off(a, page, kvh, jlat, side)) = sc;
        }
      } else if (page >= 0) {
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
              *reinterpret_cast<uint4*>(codes + code_off_in<bf16>(a, page, kvh, jlat, c8, side)) =
                  w;
            }
          }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over rows [B][H_kv][n][128] bf16 with element strides
// (seq_stride, head_stride); boxes of 64 dims x 128 rows, 128-byte swizzle.
bool encode_rows(CUtensorMap* tm, const void* base, int n, int H_kv, int B,
                 long long seq_stride, long long head_stride) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)n, (cuuint64_t)H_kv, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)head_stride * 2,
                           (cuuint64_t)seq_stride * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)kTcRows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

bool encode_tiled(CUtensorMap* tm, CUtensorMapDataType dt, int rank, const void* base,
                  const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(tm, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

size_t bulk_tc_smem_bytes(int rk, int rv, int NS, int B, int NB) {
  return (size_t)tc_plan(NS, round16(rk), round16(rv), B, NB).total + 1024;
}

int bulk_compress_tc_launch(const AppendArgs& a, int sms, int optin, cudaStream_t st) {
  const int NK = round16(a.rk), NV = round16(a.rv);
  // two basis buffers and at least four stages when they fit, else one
  // basis buffer and as many stages as fit (at least two)
  int NB = 2, NS = kTcMaxStages;
  while (NS >= 4 && bulk_tc_smem_bytes(a.rk, a.rv, NS, a.B, NB) > (size_t)optin) --NS;
  if (NS < 4) {
    NB = 1;
    NS = kTcMaxStages;
    while (NS >= 2 && bulk_tc_smem_bytes(a.rk, a.rv, NS, a.B, NB) > (size_t)optin) --NS;
  }
  if (NS < 2) return LRKV_ERR_UNSUPPORTED;
  // the tensor maps need 16-byte aligned rows and strides (checked by the API)
  if (a.head_stride < 0 || a.seq_stride < 0 || a.n < 1) return LRKV_ERR_ARG;
  CUtensorMap tmK, tmV;
  if (!encode_rows(&tmK, a.k, a.n, a.H_kv, a.B, a.seq_stride, a.head_stride) ||
      !encode_rows(&tmV, a.v, a.n, a.H_kv, a.B, a.seq_stride, a.head_stride))
    return LRKV_ERR_UNSUPPORTED;
  const int rc = prepare_kernel((const void*)bulk_compress_tc, false);
  if (rc != LRKV_OK) return rc;
  const size_t smem = bulk_tc_smem_bytes(a.rk, a.rv, NS, a.B, NB);
  bulk_compress_tc<<<sms, kTcThreads, smem, st>>>(tmK, tmV, a, NS, NK, NV, NB);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
