// Decode attention over the latent code cache plus full-rank anchors.
//
// Three launches per call, all stream-ordered:
//  1. qfold : q~ = P_k^T q per q head (Half the Memory, section 08: attend
//             directly against the codes), pre-scaled by scale * log2(e) so
//             the softmax runs on exp2; full-rank q is scaled the same way.
//  2. split : persistent grid.  The tiles of all (sequence, KV head) units
//             are laid end to end (latent pages first space, full-rank
//             anchor tiles second space) and each CTA takes an equal,
//             contiguous range of each space.  One producer lane streams the
//             tiles into a shared-memory ring with bulk copies completing on
//             mbarriers; eight consumer warps each take every eighth tile.
//             A consumer computes, for its tile, the G grouped heads' scores
//             (lane = token, q chunks broadcast from shared memory), an
//             online softmax on exp2 with one max per tile, and accumulates
//             p * c_v with lanes split over value chunks.  At each unit
//             boundary it writes a partial (m, l, acc) record.
//  3. merge : per (sequence, q head) combines the partials of every warp
//             that touched its unit, up-projects the latent accumulator with
//             P_v (o = P_v sum p c_v), adds the full-rank accumulator and
//             divides by the softmax denominator.
// The dense full-rank baseline runs the same kernels with an empty latent
// space and every token in the full-rank space.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kConsumers = 8;                   // consumer warps per CTA
constexpr int kThreads = 32 * (1 + kConsumers); // + one producer warp
constexpr int kMaxStages = 16;

struct DecodeArgs {
  int B, H_kv, G, H_q;
  const int* seq_len;
  int n_sink, W;  // dense mode: n_sink = 0, W = INT_MAX
  // latent space (kc == nullptr: empty)
  const void* kc;
  const void* vc;
  const int* bt_lat;
  int maxp_lat, rk, rv;
  // full-rank space (fk == nullptr: empty)
  const void* fk;
  const void* fv;
  const int* bt_fr;       // nullptr: tiles of a unit are contiguous
  int maxp_fr;            // block-table row length, or tiles per unit
  int num_pages_lat, num_pages_fr;
  // workspace
  int* err;
  float* qlat;  // [B][H_q][rk]
  float* qfr;   // [B][H_q][128]
  float* part_lat;
  float* part_fr;
  int C;        // CTAs of the split grid
  int NS;       // ring stages
  int stage_bytes;
};

__host__ __device__ inline int hdr_floats(int G) { return ((2 * G + 3) / 4) * 4; }

__device__ inline int tiles_lat(int n) { return (n + kLatPage - 1) / kLatPage; }
__device__ inline int tiles_fr(int n) { return (n + kFrTile - 1) / kFrTile; }

__device__ inline int range_lo(int c, int total, int C) {
  return (int)(((long long)c * total) / C);
}
// CTA whose range holds tile t (0 <= t < total).
__device__ inline int cta_of(int t, int total, int C) {
  int c = (int)(((long long)t * C) / total);
  if (c > C - 1) c = C - 1;
  while (c + 1 < C && range_lo(c + 1, total, C) <= t) ++c;
  while (c > 0 && range_lo(c, total, C) > t) --c;
  return c;
}

// Exclusive prefix over sequences of (tiles per unit * H_kv) for both
// spaces, built by one warp into shared arrays of B + 1 entries.
__device__ void build_prefix(const DecodeArgs& a, int* start_lat, int* start_fr) {
  const int lane = threadIdx.x & 31;
  const int per = (a.B + 31) / 32;
  const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
  int sl = 0, sf = 0;
  for (int b = b0; b < b1; ++b) {
    Split s = split_tokens(max(0, a.seq_len[b]), a.n_sink, a.W);
    int nl = a.kc ? min(tiles_lat(s.lat), a.maxp_lat) : 0;
    int nf = a.fk ? tiles_fr(s.sink + s.win) : 0;
    if (a.fk && a.bt_fr) nf = min(nf, a.maxp_fr);
    sl += nl * a.H_kv;
    sf += nf * a.H_kv;
  }
  int il = sl, jf = sf;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int x = __shfl_up_sync(0xffffffffu, il, o);
    int y = __shfl_up_sync(0xffffffffu, jf, o);
    if (lane >= o) { il += x; jf += y; }
  }
  int el = il - sl, ef = jf - sf;
  for (int b = b0; b < b1; ++b) {
    start_lat[b] = el;
    start_fr[b] = ef;
    Split s = split_tokens(max(0, a.seq_len[b]), a.n_sink, a.W);
    int nl = a.kc ? min(tiles_lat(s.lat), a.maxp_lat) : 0;
    int nf = a.fk ? tiles_fr(s.sink + s.win) : 0;
    if (a.fk && a.bt_fr) nf = min(nf, a.maxp_fr);
    el += nl * a.H_kv;
    ef += nf * a.H_kv;
  }
  if (lane == 31) { start_lat[a.B] = il; start_fr[a.B] = jf; }
}

// Locate global tile t of a space: sequence b, kv head, tile index in unit.
__device__ inline void locate(const int* start, int B, int H_kv, int t, int& b, int& kvh,
                              int& i, int& tiles) {
  int lo = 0, hi = B;  // largest b with start[b] <= t
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (start[mid] <= t) lo = mid; else hi = mid;
  }
  b = lo;
  tiles = (start[b + 1] - start[b]) / H_kv;
  int r = t - start[b];
  kvh = r / tiles;
  i = r - kvh * tiles;
}

// Tokens of sequence b in a space (latent or full-rank).
__device__ inline int space_tokens(const DecodeArgs& a, int sp, int b) {
  Split s = split_tokens(max(0, a.seq_len[b]), a.n_sink, a.W);
  return sp == 0 ? s.lat : s.sink + s.win;
}

// ------------------------------------------------------------ tile math
template <typename T, int G, int TT>
__device__ __forceinline__ void process_tile(const uint8_t* stage, int n_valid, int nck, int ncv,
                                             int TS, const float* qv, int qdim, float* pbuf,
                                             float (&m)[G], float (&l)[G],
                                             float (&acc)[G][Elem<T>::CE], int lane) {
  constexpr int CE = Elem<T>::CE;
  constexpr int TPL = TT / 32;
  const uint4* kch = reinterpret_cast<const uint4*>(stage);
  const uint4* vch = kch + nck * TT;

  // Phase A: scores, lane = token.
  float s[TPL][G];
#pragma unroll
  for (int i = 0; i < TPL; ++i)
#pragma unroll
    for (int h = 0; h < G; ++h) s[i][h] = 0.f;
#pragma unroll 2
  for (int j = 0; j < nck; ++j) {
    float qf[G][CE];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4* qp = reinterpret_cast<const float4*>(qv + h * qdim + j * CE);
#pragma unroll
      for (int e4 = 0; e4 < CE / 4; ++e4) {
        float4 x = qp[e4];
        qf[h][4 * e4 + 0] = x.x; qf[h][4 * e4 + 1] = x.y;
        qf[h][4 * e4 + 2] = x.z; qf[h][4 * e4 + 3] = x.w;
      }
    }
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      uint4 c = kch[j * TT + lane + 32 * i];
      float f[CE];
      unpack_chunk<T>(c, f);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < CE; ++e) s[i][h] = fmaf(qf[h][e], f[e], s[i][h]);
    }
  }
  // Online softmax with one running max per head, updated once per tile.
  float alpha[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float mt = -INFINITY;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      if (lane + 32 * i >= n_valid) s[i][h] = -INFINITY;
      mt = fmaxf(mt, s[i][h]);
    }
    mt = warp_max(mt);
    float mn = fmaxf(m[h], mt);
    alpha[h] = exp2f(m[h] - mn);
    m[h] = mn;
    float ps = 0.f;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      s[i][h] = exp2f(s[i][h] - mn);
      ps += s[i][h];
    }
    l[h] = l[h] * alpha[h] + ps;
  }
#pragma unroll
  for (int i = 0; i < TPL; ++i)
#pragma unroll
    for (int h = 0; h < G; ++h) pbuf[(lane + 32 * i) * G + h] = s[i][h];
  __syncwarp();

  // Phase B: acc[h][chunk jc] += p[t][h] * c_v[t][chunk jc].
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < CE; ++e) acc[h][e] *= alpha[h];
  const int jc = lane / TS, tsub = lane - jc * TS;
  if (jc < ncv) {
    const uint4* vrow = vch + jc * TT;
#pragma unroll 4
    for (int t0 = 0; t0 < n_valid; t0 += TS) {
      int t = t0 + tsub;
      if (t < n_valid) {
        float p[G];
#pragma unroll
        for (int h = 0; h < G; ++h) p[h] = pbuf[t * G + h];
        float f[CE];
        unpack_chunk<T>(vrow[t], f);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < CE; ++e) acc[h][e] = fmaf(p[h], f[e], acc[h][e]);
      }
    }
  }
  __syncwarp();
}

template <typename T, int G>
__device__ __forceinline__ void flush(float* rec, int rv, int TS, int ncv, const float (&m)[G],
                                      const float (&l)[G], float (&acc)[G][Elem<T>::CE],
                                      int lane) {
  constexpr int CE = Elem<T>::CE;
  const int H = hdr_floats(G);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float lt = warp_sum(l[h]);
    if (lane == 0) { rec[h] = m[h]; rec[G + h] = lt; }
  }
  for (int o = TS >> 1; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < CE; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], o);
  const int jc = lane / TS, tsub = lane - jc * TS;
  if (tsub == 0 && jc < ncv) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float4* dst = reinterpret_cast<float4*>(rec + H + h * rv + jc * CE);
#pragma unroll
      for (int e4 = 0; e4 < CE / 4; ++e4)
        dst[e4] = make_float4(acc[h][4 * e4], acc[h][4 * e4 + 1], acc[h][4 * e4 + 2],
                              acc[h][4 * e4 + 3]);
    }
  }
}

// ------------------------------------------------------------ kernels
template <typename T>
__global__ void __launch_bounds__(128) qfold_kernel(DecodeArgs a, const T* __restrict__ q,
                                                    const float* __restrict__ P_k,
                                                    long long basis_bs, float qscale) {
  __shared__ float qs[kHeadDim];
  const int bh = blockIdx.x, b = bh / a.H_q, h = bh - b * a.H_q, kvh = h / a.G;
  const int d = threadIdx.x;
  if (bh == 0 && d == 0) *a.err = kErrNone;
  qs[d] = to_f<T>(q[(size_t)bh * kHeadDim + d]);
  __syncthreads();
  if (a.fk) a.qfr[(size_t)bh * kHeadDim + d] = qs[d] * qscale;
  if (a.kc) {
    const float* P = P_k + (size_t)b * basis_bs + (size_t)kvh * kHeadDim * a.rk;
    for (int j = d; j < a.rk; j += blockDim.x) {
      float s = 0.f;
#pragma unroll 8
      for (int i = 0; i < kHeadDim; ++i) s = fmaf(P[(size_t)i * a.rk + j], qs[i], s);
      a.qlat[(size_t)bh * a.rk + j] = s * qscale;
    }
  }
}

template <typename T, int G>
__global__ void __launch_bounds__(kThreads, 1) split_kernel(DecodeArgs a) {
  constexpr int CE = Elem<T>::CE;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)a.NS * a.stage_bytes);
  uint64_t* empty = full + a.NS;
  int* start_lat = reinterpret_cast<int*>(empty + a.NS);
  int* start_fr = start_lat + (a.B + 1);
  float* pbuf_all = reinterpret_cast<float*>(start_fr + (a.B + 1));
  pbuf_all = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(pbuf_all) + 15) & ~uintptr_t(15));
  float* qbuf_all = pbuf_all + kConsumers * kLatPage * G;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  if (warp == 0) build_prefix(a, start_lat, start_fr);
  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int s = 0; s < a.NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_fence_init();
  }
  __syncthreads();

  const int tot[2] = {start_lat[a.B], start_fr[a.B]};
  const int* starts[2] = {start_lat, start_fr};

  if (warp == 0) {
    // ---------------- producer: one lane issues bulk copies in tile order.
    if (lane == 0) {
      int k = 0;
      int last_k[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last_k[s] = -1;
      bool ok = true;
      for (int sp = 0; sp < 2 && ok; ++sp) {
        if (tot[sp] == 0) continue;
        const int lo = range_lo(c, tot[sp], a.C), hi = range_lo(c + 1, tot[sp], a.C);
        for (int t = lo; t < hi; ++t, ++k) {
          const int s = k % a.NS, n = k / a.NS;
          if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
            *a.err = kErrTimeout; s_fail = 1; ok = false; break;
          }
          if (*(volatile int*)&s_fail) { ok = false; break; }
          int b, kvh, i, tiles;
          locate(starts[sp], a.B, a.H_kv, t, b, kvh, i, tiles);
          const T *srck, *srcv;
          uint32_t kb, vb;
          bool good = true;
          if (sp == 0) {
            int page = a.bt_lat[(size_t)b * a.maxp_lat + i];
            good = page >= 0 && page < a.num_pages_lat;
            size_t base = ((size_t)(good ? page : 0) * a.H_kv + kvh) * kLatPage;
            srck = static_cast<const T*>(a.kc) + base * a.rk;
            srcv = static_cast<const T*>(a.vc) + base * a.rv;
            kb = kLatPage * a.rk * sizeof(T);
            vb = kLatPage * a.rv * sizeof(T);
          } else {
            size_t base;
            if (a.bt_fr) {
              int page = a.bt_fr[(size_t)b * a.maxp_fr + i];
              good = page >= 0 && page < a.num_pages_fr;
              base = ((size_t)(good ? page : 0) * a.H_kv + kvh);
            } else {
              base = ((size_t)b * a.H_kv + kvh) * a.maxp_fr + i;
            }
            srck = static_cast<const T*>(a.fk) + base * kFrTile * kHeadDim;
            srcv = static_cast<const T*>(a.fv) + base * kFrTile * kHeadDim;
            kb = vb = kFrTile * kHeadDim * sizeof(T);
          }
          uint8_t* dst = ring + (size_t)s * a.stage_bytes;
          if (good) {
            mbar_arrive_expect_tx(&full[s], kb + vb);
            bulk_g2s(dst, srck, kb, &full[s]);
            bulk_g2s(dst + kb, srcv, vb, &full[s]);
          } else {
            *a.err = kErrBadPage;
            mbar_arrive(&full[s]);
          }
          last_k[s] = k;
        }
      }
      // Drain: wait (bounded) for every copy this CTA issued.
      for (int s = 0; s < a.NS && s < kMaxStages; ++s)
        if (last_k[s] >= 0 && !mbar_wait_bounded(&full[s], (last_k[s] / a.NS) & 1))
          *a.err = kErrTimeout;
    }
  } else {
    // ---------------- consumers
    const int w = warp - 1;
    float* pbuf = pbuf_all + w * kLatPage * G;
    float* qbuf = qbuf_all + w * G * kHeadDim;
    int kbase = 0;
    for (int sp = 0; sp < 2; ++sp) {
      if (tot[sp] == 0) continue;
      const int lo = range_lo(c, tot[sp], a.C), hi = range_lo(c + 1, tot[sp], a.C);
      const int nck = sp == 0 ? a.rk / CE : kHeadDim / CE;
      const int ncv = sp == 0 ? a.rv / CE : kHeadDim / CE;
      const int rvd = sp == 0 ? a.rv : kHeadDim;
      int TS = 1;
      while (TS * 2 * ncv <= 32) TS *= 2;
      const int qdim = sp == 0 ? a.rk : kHeadDim;
      float* part = sp == 0 ? a.part_lat : a.part_fr;
      const int rec_stride = hdr_floats(G) + G * rvd;
      int t = lo;
      while (t < hi) {
        int b, kvh, i0, tiles;
        locate(starts[sp], a.B, a.H_kv, t, b, kvh, i0, tiles);
        const int unit = b * a.H_kv + kvh;
        const int ustart = t - i0;
        const int ce = min(hi, ustart + tiles);
        const int ntok = space_tokens(a, sp, b);
        // this unit's folded queries -> per-warp shared buffer
        const float* qsrc = (sp == 0 ? a.qlat : a.qfr) + ((size_t)b * a.H_q + kvh * G) * qdim;
        for (int x = lane; x < G * qdim; x += 32) qbuf[x] = qsrc[x];
        __syncwarp();
        float m[G], l[G], acc[G][CE];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
          for (int e = 0; e < CE; ++e) acc[h][e] = 0.f;
        }
        const int k0 = kbase + (t - lo);
        int tt = t + ((w - k0 % kConsumers) + kConsumers) % kConsumers;
        for (; tt < ce; tt += kConsumers) {
          const int k = kbase + (tt - lo);
          const int s = k % a.NS, n = k / a.NS;
          if (!mbar_wait_bounded(&full[s], n & 1)) { *a.err = kErrTimeout; s_fail = 1; break; }
          const int it = tt - ustart;
          const int tt_tok = sp == 0 ? kLatPage : kFrTile;
          const int nv = min(tt_tok, ntok - it * tt_tok);
          const uint8_t* st = ring + (size_t)s * a.stage_bytes;
          if (sp == 0)
            process_tile<T, G, kLatPage>(st, nv, nck, ncv, TS, qbuf, qdim, pbuf, m, l, acc, lane);
          else
            process_tile<T, G, kFrTile>(st, nv, nck, ncv, TS, qbuf, qdim, pbuf, m, l, acc, lane);
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        const size_t slot = ((size_t)(unit + c)) * kConsumers + w;
        flush<T, G>(part + slot * rec_stride, rvd, TS, ncv, m, l, acc, lane);
        __syncwarp();
        t = ce;
        if (*(volatile int*)&s_fail) break;
      }
      kbase += hi - lo;
      if (*(volatile int*)&s_fail) break;
    }
  }
  __syncthreads();
}

// Slot x of a unit's span [c0, c1] x kConsumers; false if CTA c0 + x / 8 has
// an empty range (it wrote nothing).
__device__ inline bool span_slot(int x, int c0, int unit, int total, int C, size_t& slot) {
  const int cc = c0 + x / kConsumers;
  if (range_lo(cc, total, C) == range_lo(cc + 1, total, C)) return false;
  slot = (size_t)(unit + cc) * kConsumers + (x % kConsumers);
  return true;
}

template <typename T>
__global__ void __launch_bounds__(128) merge_kernel(DecodeArgs a, const float* __restrict__ P_v,
                                                    long long basis_bs, T* __restrict__ o) {
  extern __shared__ __align__(16) uint8_t smem[];
  int* start_lat = reinterpret_cast<int*>(smem);
  int* start_fr = start_lat + (a.B + 1);
  float* acc_lat = reinterpret_cast<float*>(start_fr + (a.B + 1));  // [r_v]
  __shared__ float red[4];
  __shared__ float s_M, s_L;

  const int bh = blockIdx.x, b = bh / a.H_q, h = bh - b * a.H_q, kvh = h / a.G, g = h % a.G;
  const int d = threadIdx.x, lane = d & 31, wid = d >> 5;
  const int unit = b * a.H_kv + kvh;
  if (wid == 0) build_prefix(a, start_lat, start_fr);
  __syncthreads();

  int c0[2] = {0, 0}, nslot[2] = {0, 0}, total[2];
  const int* starts[2] = {start_lat, start_fr};
  for (int sp = 0; sp < 2; ++sp) {
    total[sp] = starts[sp][a.B];
    const int tiles = (starts[sp][b + 1] - starts[sp][b]) / a.H_kv;
    if (total[sp] == 0 || tiles == 0) continue;
    const int us = starts[sp][b] + kvh * tiles;
    c0[sp] = cta_of(us, total[sp], a.C);
    nslot[sp] = (cta_of(us + tiles - 1, total[sp], a.C) - c0[sp] + 1) * kConsumers;
  }
  const int H = hdr_floats(a.G);
  const int strides[2] = {H + a.G * a.rv, H + a.G * kHeadDim};
  const float* parts[2] = {a.part_lat, a.part_fr};

  // Max of the running maxima.
  float M = -INFINITY;
  for (int sp = 0; sp < 2; ++sp)
    for (int x = d; x < nslot[sp]; x += blockDim.x) {
      size_t slot;
      if (span_slot(x, c0[sp], unit, total[sp], a.C, slot))
        M = fmaxf(M, parts[sp][slot * strides[sp] + g]);
    }
  M = warp_max(M);
  if (lane == 0) red[wid] = M;
  __syncthreads();
  if (d == 0) s_M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  M = s_M;
  const bool empty_seq = !(M > -INFINITY);

  float L = 0.f;
  for (int sp = 0; sp < 2 && !empty_seq; ++sp)
    for (int x = d; x < nslot[sp]; x += blockDim.x) {
      size_t slot;
      if (span_slot(x, c0[sp], unit, total[sp], a.C, slot)) {
        const float* rec = parts[sp] + slot * strides[sp];
        L += exp2f(rec[g] - M) * rec[a.G + g];
      }
    }
  L = warp_sum(L);
  __syncthreads();
  if (lane == 0) red[wid] = L;
  __syncthreads();
  if (d == 0) s_L = red[0] + red[1] + red[2] + red[3];

  // Latent accumulator (r_v entries), then the full-rank one (128 entries).
  if (a.kc) {
    for (int j = d; j < a.rv; j += blockDim.x) {
      float s = 0.f;
      for (int x = 0; x < nslot[0] && !empty_seq; ++x) {
        size_t slot;
        if (!span_slot(x, c0[0], unit, total[0], a.C, slot)) continue;
        const float* rec = a.part_lat + slot * strides[0];
        s += exp2f(rec[g] - M) * rec[H + g * a.rv + j];
      }
      acc_lat[j] = s;
    }
  }
  float afr = 0.f;
  if (a.fk && !empty_seq) {
    for (int x = 0; x < nslot[1]; ++x) {
      size_t slot;
      if (!span_slot(x, c0[1], unit, total[1], a.C, slot)) continue;
      const float* rec = a.part_fr + slot * strides[1];
      afr += exp2f(rec[g] - M) * rec[H + g * kHeadDim + d];
    }
  }
  __syncthreads();
  float out = afr;
  if (a.kc) {
    const float* P = P_v + (size_t)b * basis_bs + (size_t)kvh * kHeadDim * a.rv + (size_t)d * a.rv;
    for (int j = 0; j < a.rv; ++j) out = fmaf(P[j], acc_lat[j], out);
  }
  out = empty_seq ? 0.f : out / s_L;
  o[(size_t)bh * kHeadDim + d] = from_f<T>(out);
}

// ------------------------------------------------------------ host side
struct Plan {
  int C, NS, stage_bytes, smem;
  size_t off_qlat, off_qfr, off_lat, off_fr, total;
};

static int smem_fixed(int G, int B) {
  return 2 * kMaxStages * 8 + 2 * (B + 1) * 4 + 16 + kConsumers * kLatPage * G * 4 +
         kConsumers * G * kHeadDim * 4 + 64;
}

static int plan_decode(int B, int H_kv, int H_q, int rk, int rv, bool has_lat, bool has_fr,
                       int esize, Plan& p) {
  int dev = 0, sms = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LRKV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LRKV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return LRKV_ERR_CUDA;
  const int G = H_q / H_kv;
  int lat_b = has_lat ? kLatPage * (rk + rv) * esize : 0;
  int fr_b = has_fr ? 2 * kFrTile * kHeadDim * esize : 0;
  p.stage_bytes = std::max(lat_b, fr_b);
  int room = optin - smem_fixed(G, B) - 1024;
  p.NS = std::min(kMaxStages, room / p.stage_bytes);
  if (p.NS < 2) return LRKV_ERR_UNSUPPORTED;
  p.smem = p.NS * p.stage_bytes + smem_fixed(G, B);
  p.C = sms;
  const int U = B * H_kv;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 256;
  p.off_qlat = off; off = al(off + (size_t)B * H_q * (has_lat ? rk : 0) * 4);
  p.off_qfr = off;  off = al(off + (size_t)B * H_q * (has_fr ? kHeadDim : 0) * 4);
  const size_t slots = (size_t)(U + p.C - 1) * kConsumers;
  p.off_lat = off;  off = al(off + (has_lat ? slots * (hdr_floats(G) + G * rv) * 4 : 0));
  p.off_fr = off;   off = al(off + (has_fr ? slots * (hdr_floats(G) + G * kHeadDim) * 4 : 0));
  p.total = off;
  return LRKV_OK;
}

size_t decode_workspace_bytes(int B, int H_kv, int H_q, int rk, int rv, bool has_lat,
                              bool has_fr, int dtype) {
  Plan p;
  if (plan_decode(B, H_kv, H_q, rk, rv, has_lat, has_fr, dtype == LRKV_BF16 ? 2 : 4, p) !=
      LRKV_OK)
    return 0;
  return p.total;
}

template <typename T, int G>
static int launch_decode_t(DecodeArgs a, const Plan& p, const void* q, const float* P_k,
                           const float* P_v, long long bs, float scale, void* o,
                           cudaStream_t st) {
  const float qscale = scale * kLog2e;
  qfold_kernel<T><<<a.B * a.H_q, 128, 0, st>>>(a, static_cast<const T*>(q), P_k, bs, qscale);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  if (cudaFuncSetAttribute(split_kernel<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           p.smem) != cudaSuccess)
    return LRKV_ERR_CUDA;
  split_kernel<T, G><<<p.C, kThreads, p.smem, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  const int msmem = 2 * (a.B + 1) * 4 + kHeadDim * 4 + 16;  // prefix + acc_lat
  merge_kernel<T><<<a.B * a.H_q, 128, msmem, st>>>(a, P_v, bs, static_cast<T*>(o));
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

template <typename T>
static int launch_decode_g(DecodeArgs a, const Plan& p, const void* q, const float* P_k,
                           const float* P_v, long long bs, float scale, void* o,
                           cudaStream_t st) {
  switch (a.G) {
    case 1: return launch_decode_t<T, 1>(a, p, q, P_k, P_v, bs, scale, o, st);
    case 2: return launch_decode_t<T, 2>(a, p, q, P_k, P_v, bs, scale, o, st);
    case 4: return launch_decode_t<T, 4>(a, p, q, P_k, P_v, bs, scale, o, st);
    case 8: return launch_decode_t<T, 8>(a, p, q, P_k, P_v, bs, scale, o, st);
    default: return LRKV_ERR_UNSUPPORTED;
  }
}

int decode_launch(const DecodeLaunch& L, cudaStream_t st) {
  const bool has_lat = L.kc != nullptr, has_fr = L.fk != nullptr;
  const int es = L.dtype == LRKV_BF16 ? 2 : 4;
  Plan p;
  int rc = plan_decode(L.B, L.H_kv, L.H_q, L.rk, L.rv, has_lat, has_fr, es, p);
  if (rc != LRKV_OK) return rc;
  if (L.ws_bytes < p.total) return LRKV_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(L.ws);
  DecodeArgs a;
  a.B = L.B; a.H_kv = L.H_kv; a.G = L.H_q / L.H_kv; a.H_q = L.H_q;
  a.seq_len = L.seq_len; a.n_sink = L.n_sink; a.W = L.W;
  a.kc = L.kc; a.vc = L.vc; a.bt_lat = L.bt_lat; a.maxp_lat = L.maxp_lat;
  a.rk = L.rk; a.rv = L.rv;
  a.fk = L.fk; a.fv = L.fv; a.bt_fr = L.bt_fr; a.maxp_fr = L.maxp_fr;
  a.num_pages_lat = L.num_pages_lat; a.num_pages_fr = L.num_pages_fr;
  a.err = reinterpret_cast<int*>(ws);
  a.qlat = reinterpret_cast<float*>(ws + p.off_qlat);
  a.qfr = reinterpret_cast<float*>(ws + p.off_qfr);
  a.part_lat = reinterpret_cast<float*>(ws + p.off_lat);
  a.part_fr = reinterpret_cast<float*>(ws + p.off_fr);
  a.C = p.C; a.NS = p.NS; a.stage_bytes = p.stage_bytes;
  if (L.dtype == LRKV_BF16)
    return launch_decode_g<__nv_bfloat16>(a, p, L.q, L.P_k, L.P_v, L.basis_bs, L.scale, L.o, st);
  return launch_decode_g<float>(a, p, L.q, L.P_k, L.P_v, L.basis_bs, L.scale, L.o, st);
}

}  // namespace lrkv
