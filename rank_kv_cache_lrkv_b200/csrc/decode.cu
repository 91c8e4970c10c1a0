// Decode attention over the latent code cache plus full-rank anchors.
//
// One persistent launch per call, one CTA per SM.  The tiles of all
// (sequence, KV head) units are laid end to end -- latent pages (64 tokens)
// in one space, full-rank anchor tiles (32 tokens) in another -- and each CTA
// takes an equal contiguous range of each space, so any mix of sequence
// lengths is balanced across SMs.
//  * Two producer warps (odd and even tiles, each owning half the stages)
//    compute tile addresses a batch ahead (block-table reads in parallel)
//    and stream one slab per tile into a shared-memory ring with bulk
//    copies that complete on mbarriers.
//  * Eight consumer warps take every eighth tile.  At the start of each unit
//    in the CTA's range they fold that unit's queries together:
//    q~ = P_k^T q for its G query heads (Half the Memory, section 08: attend
//    directly against the codes), pre-scaled by scale * log2(e) so the
//    softmax runs on exp2.  Per tile: scores with lane = token (q chunks
//    broadcast from shared memory, packed fp32 FMA), an exp2 online softmax
//    with one max per tile, then p * c_v with lanes split over value chunks.
//  * At a unit boundary the warps' partial (m, l, acc) are combined in
//    shared memory into one record per (unit, CTA); the CTA whose record
//    completes the unit's tile count combines all records of the unit and
//    writes o = (P_v acc_lat + acc_fr) / l, then resets the unit's counter.
// The dense full-rank baseline runs the same kernel with no latent space.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kConsumers = 8;                    // consumer warps per CTA
constexpr int kProducers = 2;                    // producer warps per CTA
constexpr int kCThreads = 32 * kConsumers;       // consumer threads
constexpr int kThreads = 32 * (kProducers + kConsumers);
constexpr int kMaxStages = 16;
constexpr int kBarConsumers = 1;                 // named barrier id
constexpr int kIssue = 4;                        // producer lanes issuing at once
constexpr int kMaxPre = 4;                       // chunks whose queries are fetched at start
constexpr int kMaxRec = 160;                     // records (CTAs) per unit and space

struct DecodeArgs {
  int B, H_kv, G, H_q;
  const int* seq_len;
  int n_sink, W;  // dense mode: n_sink = 0, W = INT_MAX
  // latent space (codes == nullptr: empty); one slab per (page, kv head)
  const void* codes;
  const int* bt_lat;
  int maxp_lat, rk, rv;
  // full-rank space (fr == nullptr: empty); one slab per tile
  const void* fr;
  const int* bt_fr;  // nullptr: tiles of a unit are contiguous
  int maxp_fr;       // block-table row length, or tiles per unit
  int num_pages_lat, num_pages_fr;
  const float* P_v;
  long long basis_bs;
  void* o;
  const void* q;       // [B][H_q][128] in the cache dtype
  const float* P_k;
  float qscale;        // scale * log2(e)
  // workspace
  int* err;            // sticky error word
  int* unit_cnt;       // [B * H_kv] tile counters, zero between calls
  float* qlat;         // [B][H_q][rk] folded queries (scaled)
  float* qfr;          // [B][H_q][128] scaled queries
  float* part_lat;
  float* part_fr;
  int C;   // CTAs of the split grid
  int NS;  // ring stages
  int stage_bytes;
};

__host__ __device__ inline int hdr_floats(int G) { return ((2 * G + 3) / 4) * 4; }

__device__ inline int tiles_lat(int n) { return (n + kLatPage - 1) / kLatPage; }
__device__ inline int tiles_fr(int n) { return (n + kFrTile - 1) / kFrTile; }

// First tile of CTA c when `total` tiles are split evenly over C CTAs:
// floor(c * total / C), in 32-bit arithmetic (c * (total % C) < C * C).
__device__ inline int range_lo(int c, int total, int C) {
  const int q = total / C, r = total - q * C;
  return c * q + (c * r) / C;
}
// CTA whose range holds tile t (0 <= t < total).
__device__ inline int cta_of(int t, int total, int C) {
  int c = (int)((float)t * (float)C / (float)total);
  if (c < 0) c = 0;
  if (c > C - 1) c = C - 1;
  while (c + 1 < C && range_lo(c + 1, total, C) <= t) ++c;
  while (c > 0 && range_lo(c, total, C) > t) --c;
  return c;
}

__device__ inline int unit_lat_tiles(const DecodeArgs& a, int L) {
  if (!a.codes) return 0;
  return min(tiles_lat(split_tokens(L, a.n_sink, a.W).lat), a.maxp_lat);
}
__device__ inline int unit_fr_tiles(const DecodeArgs& a, int L) {
  if (!a.fr) return 0;
  const Split s = split_tokens(L, a.n_sink, a.W);
  const int n = tiles_fr(s.sink + s.win);
  return a.bt_fr ? min(n, a.maxp_fr) : n;
}

// Exclusive prefix over sequences of (tiles per unit * H_kv) for both
// spaces, built by one warp into shared arrays of B + 1 entries.
__device__ void build_prefix(const DecodeArgs& a, int* start_lat, int* start_fr) {
  const int lane = threadIdx.x & 31;
  const int per = (a.B + 31) / 32;
  const int b0 = min(a.B, lane * per), b1 = min(a.B, b0 + per);
  int sl = 0, sf = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = max(0, a.seq_len[b]);
    sl += unit_lat_tiles(a, L) * a.H_kv;
    sf += unit_fr_tiles(a, L) * a.H_kv;
  }
  int il = sl, jf = sf;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, il, o);
    const int y = __shfl_up_sync(0xffffffffu, jf, o);
    if (lane >= o) { il += x; jf += y; }
  }
  int el = il - sl, ef = jf - sf;
  for (int b = b0; b < b1; ++b) {
    start_lat[b] = el;
    start_fr[b] = ef;
    const int L = max(0, a.seq_len[b]);
    el += unit_lat_tiles(a, L) * a.H_kv;
    ef += unit_fr_tiles(a, L) * a.H_kv;
  }
  if (lane == 31) { start_lat[a.B] = il; start_fr[a.B] = jf; }
}

// Locate global tile t of a space: sequence b, kv head, tile index in unit.
__device__ inline void locate(const int* start, int B, int H_kv, int t, int& b, int& kvh,
                              int& i, int& tiles) {
  int lo = 0, hi = B;  // largest b with start[b] <= t (never an empty b)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (start[mid] <= t) lo = mid; else hi = mid;
  }
  b = lo;
  tiles = (start[b + 1] - start[b]) / H_kv;
  const int r = t - start[b];
  kvh = r / tiles;
  i = r - kvh * tiles;
}

// Tokens of sequence b in a space (latent or full-rank).
__device__ inline int space_tokens(const DecodeArgs& a, int sp, int b) {
  const Split s = split_tokens(max(0, a.seq_len[b]), a.n_sink, a.W);
  return sp == 0 ? s.lat : s.sink + s.win;
}

// One 16-byte chunk as CE/2 packed pairs.
template <typename T>
__device__ __forceinline__ void chunk_pairs(const uint4& c, float2* f);
template <>
__device__ __forceinline__ void chunk_pairs<__nv_bfloat16>(const uint4& c, float2* f) {
  f[0] = bf2(c.x); f[1] = bf2(c.y); f[2] = bf2(c.z); f[3] = bf2(c.w);
}
template <>
__device__ __forceinline__ void chunk_pairs<float>(const uint4& c, float2* f) {
  f[0] = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
  f[1] = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
}

// ------------------------------------------------------------ tile math
// One tile of TT tokens in a ring stage: K chunks [nck][TT], V chunks [ncv][TT].
// pbuf holds the tile's probabilities as duplicated pairs, [G][TT].
template <typename T, int G, int TT>
__device__ __forceinline__ void process_tile(const uint4* kch, int n_valid, int nck, int ncv,
                                             int TS, const float* qv, int qdim, float2* pbuf,
                                             float (&m)[G], float (&l)[G],
                                             float2 (&acc)[G][Elem<T>::CE / 2], int lane) {
  constexpr int CE = Elem<T>::CE;
  constexpr int NP = CE / 2;
  constexpr int TPL = TT / 32;
  const uint4* vch = kch + nck * TT;

  // Phase A: scores, lane = token; packed pairs over the chunk elements.
  float2 s2[TPL][G];
#pragma unroll
  for (int i = 0; i < TPL; ++i)
#pragma unroll
    for (int h = 0; h < G; ++h) s2[i][h] = make_float2(0.f, 0.f);
#pragma unroll 2
  for (int j = 0; j < nck; ++j) {
    float2 qp[G][NP];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4* src = reinterpret_cast<const float4*>(qv + h * qdim + j * CE);
#pragma unroll
      for (int e4 = 0; e4 < NP / 2; ++e4) {
        const float4 x = src[e4];
        qp[h][2 * e4] = make_float2(x.x, x.y);
        qp[h][2 * e4 + 1] = make_float2(x.z, x.w);
      }
    }
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      float2 f[NP];
      chunk_pairs<T>(kch[j * TT + lane + 32 * i], f);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < NP; ++e) fma2(s2[i][h], qp[h][e], f[e]);
    }
  }
  // Online softmax: one running max per head, updated once per tile.
  float alpha[G];
  bool rescale = false;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float s[TPL];
    float mt = -INFINITY;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      s[i] = (lane + 32 * i < n_valid) ? s2[i][h].x + s2[i][h].y : -INFINITY;
      mt = fmaxf(mt, s[i]);
    }
    mt = warp_max(mt);
    const float mn = fmaxf(m[h], mt);
    alpha[h] = exp2f(m[h] - mn);
    rescale |= (mn != m[h]);
    m[h] = mn;
    float ps = 0.f;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const float p = exp2f(s[i] - mn);
      ps += p;
      pbuf[h * TT + lane + 32 * i] = make_float2(p, p);
    }
    l[h] = l[h] * alpha[h] + ps;
  }
  __syncwarp();

  // Phase B: acc[h][chunk jc] += p[t][h] * c_v[t][chunk jc].
  if (rescale) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float2 a2 = make_float2(alpha[h], alpha[h]);
#pragma unroll
      for (int e = 0; e < NP; ++e) acc[h][e] = mul2(acc[h][e], a2);
    }
  }
  const int jc = lane / TS, tsub = lane - jc * TS;
  if (jc < ncv) {
    const uint4* vrow = vch + jc * TT;
#pragma unroll 4
    for (int t0 = 0; t0 < n_valid; t0 += TS) {
      const int t = t0 + tsub;
      if (t < n_valid) {
        float2 p[G];
#pragma unroll
        for (int h = 0; h < G; ++h) p[h] = pbuf[h * TT + t];
        float2 f[NP];
        chunk_pairs<T>(vrow[t], f);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < NP; ++e) fma2(acc[h][e], p[h], f[e]);
      }
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------ kernel pieces
// Bounded spin until the producer has issued tile k into this stage.
__device__ inline bool tag_wait_bounded(volatile int* tag, int k,
                                        uint64_t timeout_ns = 2000000000ull) {
  if (*tag == k) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (*tag == k) return true;
    if (global_ns() - t0 > timeout_ns) return false;
  }
}

// Shared-memory plan of the split kernel (byte offsets from the base).
struct SmemPlan {
  int ring, full, empty, tag, start_lat, start_fr, pbuf, qv, cml, cacc, fin_lat, recs, flags,
      total;
};
__host__ __device__ inline SmemPlan smem_plan(int NS, int stage_bytes, int B, int G) {
  SmemPlan p;
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int at = off;
    off += bytes;
    return at;
  };
  p.ring = take(NS * stage_bytes, 1024);
  p.full = take(NS * 8, 8);
  p.empty = take(NS * 8, 8);
  p.tag = take(kMaxStages * 4, 4);
  p.start_lat = take((B + 1) * 4, 4);
  p.start_fr = take((B + 1) * 4, 4);
  p.pbuf = take(kConsumers * kLatPage * G * 8, 16);
  p.qv = take((kMaxPre + 1) * G * kHeadDim * 4, 16);  // folded queries per chunk
  p.cml = take(kConsumers * 2 * G * 4, 16);
  p.cacc = take(G * kHeadDim * 4, 16);
  p.fin_lat = take(G * kHeadDim * 4, 16);
  p.recs = take(2 * kMaxRec * 4, 16);
  p.flags = take(16, 16);
  p.total = off;
  return p;
}

// Folded queries of every (sequence, KV head) unit, computed before the
// split kernel streams anything (the memory system is still quiet):
// q~ = P_k^T q for the latent space (Half the Memory, section 08: attend
// directly against the codes) and q for the full-rank space, both times
// scale * log2(e) so the softmax runs on exp2.  Also writes o = 0 for
// sequences with no tokens.  One CTA of 256 threads per unit.
template <typename T, int G>
__global__ void __launch_bounds__(256) qfold_kernel(DecodeArgs a) {
  __shared__ float qs[G * kHeadDim];
  __shared__ float red[G * 256];
  pdl_trigger();
  const int unit = blockIdx.x, b = unit / a.H_kv, kvh = unit - b * a.H_kv, tid = threadIdx.x;
  const size_t h0 = (size_t)b * a.H_q + (size_t)kvh * G;
  const T* q = static_cast<const T*>(a.q) + h0 * kHeadDim;
  for (int x = tid; x < G * kHeadDim; x += 256) qs[x] = to_f<T>(q[x]);
  __syncthreads();
  if (a.seq_len[b] <= 0) {
    T* o = static_cast<T*>(a.o) + h0 * kHeadDim;
    for (int x = tid; x < G * kHeadDim; x += 256) o[x] = from_f<T>(0.f);
  }
  if (a.fr)
    for (int x = tid; x < G * kHeadDim; x += 256) a.qfr[h0 * kHeadDim + x] = qs[x] * a.qscale;
  if (!a.codes) return;
  // thread -> (column j, row segment); all of a thread's loads in flight.
  const int rk = a.rk, nseg = 256 / rk, rows = (kHeadDim + nseg - 1) / nseg;
  const int j = tid % rk, seg = tid / rk;
  const float* P = a.P_k + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * rk;
  float acc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g] = 0.f;
  if (seg < nseg) {
    const int i0 = seg * rows, i1 = min(kHeadDim, i0 + rows);
    for (int ib = i0; ib < i1; ib += 32) {
      float pij[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) pij[u] = ib + u < i1 ? __ldg(P + (size_t)(ib + u) * rk + j) : 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u)
        if (ib + u < i1)
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] = fmaf(pij[u], qs[g * kHeadDim + ib + u], acc[g]);
    }
    for (int g = 0; g < G; ++g) red[(seg * G + g) * rk + j] = acc[g];
  }
  __syncthreads();
  for (int x = tid; x < G * rk; x += 256) {
    const int g = x / rk, jj = x - g * rk;
    float sum = 0.f;
    for (int sg = 0; sg < nseg; ++sg) sum += red[(sg * G + g) * rk + jj];
    a.qlat[h0 * rk + x] = sum * a.qscale;
  }
}

// Copy the folded queries of unit (b, kvh) for space sp into dst.
template <int G>
__device__ inline void fetch_queries(const DecodeArgs& a, int sp, int b, int kvh, float* dst,
                                     int ctid) {
  const int dim = sp == 0 ? a.rk : kHeadDim;
  const float* src = (sp == 0 ? a.qlat : a.qfr) + ((size_t)b * a.H_q + (size_t)kvh * G) * dim;
  for (int x = ctid; x < G * dim; x += kCThreads) dst[x] = __ldcg(src + x);
}

// Online merge of one more (max m, weight-sum) pair into (M, S1, S2).
__device__ __forceinline__ void merge_rec(float m, float l, float v, float& M, float& L, float& S) {
  if (!(m > -INFINITY)) return;
  if (m > M) {
    const float r = exp2f(M - m);
    L *= r;
    S *= r;
    M = m;
  }
  const float w = exp2f(m - M);
  L = fmaf(w, l, L);
  S = fmaf(w, v, S);
}

// Combine every record of `unit` and write its G output rows.  Run by all
// consumer threads of the CTA that completed the unit.  The records' offsets
// (or -1 where a CTA's range is empty) are listed first; then one load phase:
// each thread loads, for the accumulator elements it owns, every record's
// (m, l, value) eight at a time and merges them online (running max,
// rescaled sums).  One barrier publishes the latent accumulator, then
// o = (P_v acc_lat + acc_fr) / l.
template <typename T, int G>
__device__ void finalize_unit(const DecodeArgs& a, int unit, const int* start_lat,
                              const int* start_fr, float* fin_lat, int* recs, int ctid) {
  const int b = unit / a.H_kv, kvh = unit - b * a.H_kv;
  const int H = hdr_floats(G);
  int nr[2];
  const int* starts[2] = {start_lat, start_fr};
  const int rvs[2] = {a.rv, kHeadDim};
  const float* parts[2] = {a.part_lat, a.part_fr};
  // record list: recs[sp * kMaxRec + r] = record index (unit + c) or -1
#pragma unroll
  for (int sp = 0; sp < 2; ++sp) {
    const int total = starts[sp][a.B];
    const int tiles = (starts[sp][b + 1] - starts[sp][b]) / a.H_kv;
    nr[sp] = 0;
    if (total == 0 || tiles == 0) continue;
    const int us = starts[sp][b] + kvh * tiles;
    const int c0 = cta_of(us, total, a.C);
    nr[sp] = min(kMaxRec, cta_of(us + tiles - 1, total, a.C) - c0 + 1);
    for (int r = ctid; r < nr[sp]; r += kCThreads) {
      const int c = c0 + r;
      recs[sp * kMaxRec + r] =
          range_lo(c, total, a.C) == range_lo(c + 1, total, a.C) ? -1 : unit + c;
    }
  }
  named_bar(kBarConsumers, kCThreads);
  auto combine = [&](int g, int vsp, int vx, float& M, float& L, float& S) {
    M = -INFINITY; L = 0.f; S = 0.f;
    for (int sp = 0; sp < 2; ++sp) {
      const int stride = H + G * rvs[sp];
      for (int r0 = 0; r0 < nr[sp]; r0 += 8) {
        float mm[8], ll[8], vv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          mm[u] = -INFINITY; ll[u] = 0.f; vv[u] = 0.f;
          const int ri = r0 + u < nr[sp] ? recs[sp * kMaxRec + r0 + u] : -1;
          if (ri >= 0) {
            const float* rec = parts[sp] + (size_t)ri * stride;
            mm[u] = __ldcg(rec + g);
            ll[u] = __ldcg(rec + G + g);
            if (sp == vsp) vv[u] = __ldcg(rec + H + vx);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) merge_rec(mm[u], ll[u], vv[u], M, L, S);
      }
    }
  };
  if (a.codes)
    for (int x = ctid; x < G * a.rv; x += kCThreads) {
      float M, L, S;
      combine(x / a.rv, 0, x, M, L, S);
      fin_lat[x] = S;
    }
  constexpr int kPer = (G * kHeadDim + kCThreads - 1) / kCThreads;
  float accf[kPer], den[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int x = ctid + i * kCThreads;
    accf[i] = 0.f; den[i] = 0.f;
    if (x < G * kHeadDim) {
      float M, L, S;
      combine(x / kHeadDim, a.fr ? 1 : -1, x, M, L, S);
      accf[i] = S;
      den[i] = L;
    }
  }
  named_bar(kBarConsumers, kCThreads);
  T* o = static_cast<T*>(a.o) + ((size_t)b * a.H_q + (size_t)kvh * G) * kHeadDim;
  const float* P = a.codes ? a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rv : nullptr;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int x = ctid + i * kCThreads;
    if (x >= G * kHeadDim) break;
    const int g = x / kHeadDim, d = x - g * kHeadDim;
    float out = accf[i];
    if (P) {
      const float4* Pd = reinterpret_cast<const float4*>(P + (size_t)d * a.rv);
      const float4* al = reinterpret_cast<const float4*>(fin_lat + g * a.rv);
#pragma unroll 8
      for (int j4 = 0; j4 < a.rv / 4; ++j4) {
        const float4 pv = __ldg(Pd + j4), av = al[j4];
        out = fmaf(pv.x, av.x, fmaf(pv.y, av.y, fmaf(pv.z, av.z, fmaf(pv.w, av.w, out))));
      }
    }
    o[x] = from_f<T>(den[i] > 0.f ? out / den[i] : 0.f);
  }
  if (ctid == 0) a.unit_cnt[unit] = 0;  // ready for the next call
  named_bar(kBarConsumers, kCThreads);
}

// ------------------------------------------------------------ the kernel
template <typename T, int G>
__global__ void __launch_bounds__(kThreads, 1) split_kernel(DecodeArgs a) {
  constexpr int CE = Elem<T>::CE;
  constexpr int NP = CE / 2;
  extern __shared__ __align__(1024) uint8_t smem[];
  const SmemPlan sp_ = smem_plan(a.NS, a.stage_bytes, a.B, G);
  uint8_t* ring = smem + sp_.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sp_.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + sp_.empty);
  // tag[s]: index of the last tile issued into stage s.  Consumers share the
  // ring with a stride of kConsumers tiles, so a consumer may reach stage s
  // while its barrier is still two phases behind (same parity).  Waiting
  // for tag[s] == k first makes the parity test unambiguous: tile k is only
  // issued after tile k - NS was released, i.e. after phase n - 1 completed.
  volatile int* tag = reinterpret_cast<volatile int*>(smem + sp_.tag);
  int* start_lat = reinterpret_cast<int*>(smem + sp_.start_lat);
  int* start_fr = reinterpret_cast<int*>(smem + sp_.start_fr);
  // flags: [0] failure (any warp, any time), [1] finalize this unit,
  // [2] consumers' snapshot of [0] taken between their named barriers.
  int* flags = reinterpret_cast<int*>(smem + sp_.flags);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  if (warp == 0) build_prefix(a, start_lat, start_fr);
  if (threadIdx.x == 32) {
    flags[0] = flags[1] = flags[2] = 0;
    for (int s = 0; s < a.NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      tag[s] = -1;
    }
    mbar_fence_init();
  }
  __syncthreads();

  const int tot0 = start_lat[a.B], tot1 = start_fr[a.B];
  const int lo0 = range_lo(c, tot0, a.C), hi0 = range_lo(c + 1, tot0, a.C);
  const int lo1 = range_lo(c, tot1, a.C), hi1 = range_lo(c + 1, tot1, a.C);
  const int n0 = hi0 - lo0, N = n0 + (hi1 - lo1);

  if (warp < kProducers) {
    // ---------------- producer warp p: tiles k = p, p + 2, p + 4, ...
    // Lane l holds the slab address of tile base + kProducers * l; the next
    // batch's block-table reads are in flight while this batch is issued,
    // kIssue lanes at a time.
    const int p = warp;
    auto addr = [&](int kk, const void*& src, uint32_t& bytes, int& good) {
      src = nullptr; bytes = 0; good = 0;
      if (kk >= N) return;
      const int sp = kk < n0 ? 0 : 1;
      const int t = sp == 0 ? lo0 + kk : lo1 + (kk - n0);
      int b, kvh, i, tiles;
      locate(sp == 0 ? start_lat : start_fr, a.B, a.H_kv, t, b, kvh, i, tiles);
      size_t slab;
      if (sp == 0) {
        const int page = a.bt_lat[(size_t)b * a.maxp_lat + i];
        good = page >= 0 && page < a.num_pages_lat;
        slab = (size_t)(good ? page : 0) * a.H_kv + kvh;
        bytes = kLatPage * (a.rk + a.rv) * sizeof(T);
        src = static_cast<const T*>(a.codes) + slab * kLatPage * (a.rk + a.rv);
      } else {
        if (a.bt_fr) {
          const int page = a.bt_fr[(size_t)b * a.maxp_fr + i];
          good = page >= 0 && page < a.num_pages_fr;
          slab = (size_t)(good ? page : 0) * a.H_kv + kvh;
        } else {
          good = 1;
          slab = ((size_t)b * a.H_kv + kvh) * a.maxp_fr + i;
        }
        bytes = 2 * kFrTile * kHeadDim * sizeof(T);
        src = static_cast<const T*>(a.fr) + slab * 2 * kFrTile * kHeadDim;
      }
    };
    constexpr int kBatch = 32 * kProducers;
    const void *csrc, *nsrc;
    uint32_t cbytes, nbytes;
    int cgood, ngood;
    const uint64_t pol = l2_evict_first_policy();
    addr(p + kProducers * lane, csrc, cbytes, cgood);
    int issued_last = -1;  // last tile this warp issued
    bool ok = true;
    for (int base = 0; base < N && ok; base += kBatch) {
      addr(base + kBatch + p + kProducers * lane, nsrc, nbytes, ngood);
      const int cnt = min(32, (N - base - p + kProducers - 1) / kProducers);
      for (int j0 = 0; j0 < cnt; j0 += kIssue) {
        int fail = 0;
        if (lane >= j0 && lane < min(j0 + kIssue, cnt)) {
          const int k = base + p + kProducers * lane, s = k % a.NS, n = k / a.NS;
          if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
            *a.err = kErrTimeout;
            fail = 1;
          } else {
            uint8_t* dst = ring + (size_t)s * a.stage_bytes;
            if (cgood) {
              mbar_arrive_expect_tx(&full[s], cbytes);
              bulk_g2s_hint(dst, csrc, cbytes, &full[s], pol);
            } else {
              *a.err = kErrBadPage;
              mbar_arrive(&full[s]);
            }
            tag[s] = k;
          }
        }
        if (__any_sync(0xffffffffu, fail) || *(volatile int*)&flags[0]) {
          ok = false;
          flags[0] = 1;
          break;
        }
        issued_last = base + p + kProducers * (min(j0 + kIssue, cnt) - 1);
      }
      csrc = nsrc; cbytes = nbytes; cgood = ngood;
    }
    // Drain: wait (bounded) for every copy this warp issued (its stages are
    // those with s % kProducers == p, since NS is a multiple of kProducers).
    if (lane == 0 && issued_last >= 0)
      for (int s = p; s < a.NS; s += kProducers) {
        if (s > issued_last) break;
        const int last = s + ((issued_last - s) / a.NS) * a.NS;
        if (!mbar_wait_bounded(&full[s], (last / a.NS) & 1)) *a.err = kErrTimeout;
      }
  } else {
    // ---------------- consumers
    const int w = warp - kProducers, ctid = threadIdx.x - 32 * kProducers;
    float2* pbuf = reinterpret_cast<float2*>(smem + sp_.pbuf) + w * kLatPage * G;
    float* qv = reinterpret_cast<float*>(smem + sp_.qv);
    float* cml = reinterpret_cast<float*>(smem + sp_.cml);
    float* cacc = reinterpret_cast<float*>(smem + sp_.cacc);
    for (int x = ctid; x < G * kHeadDim; x += kCThreads) cacc[x] = 0.f;
    named_bar(kBarConsumers, kCThreads);
    // Fetch the folded queries of the first kMaxPre chunks now, while the
    // first tiles are in flight (later these loads would queue behind the
    // streaming copies).
    pdl_wait();  // the q-fold kernel's results (and counters) are visible
    {
      int npre = 0;
      for (int sp = 0; sp < 2 && npre < kMaxPre; ++sp) {
        const int lo = sp == 0 ? lo0 : lo1, hi = sp == 0 ? hi0 : hi1;
        for (int t = lo; t < hi && npre < kMaxPre; ++npre) {
          int b, kvh, i0, tiles;
          locate(sp == 0 ? start_lat : start_fr, a.B, a.H_kv, t, b, kvh, i0, tiles);
          fetch_queries<G>(a, sp, b, kvh, qv + npre * G * kHeadDim, ctid);
          t = min(hi, t - i0 + tiles);
        }
      }
      named_bar(kBarConsumers, kCThreads);
    }
    int chunk = 0;
    for (int sp = 0; sp < 2; ++sp) {
      const int lo = sp == 0 ? lo0 : lo1, hi = sp == 0 ? hi0 : hi1;
      const int kbase = sp == 0 ? 0 : n0;
      if (lo >= hi) continue;
      const int* start = sp == 0 ? start_lat : start_fr;
      const int nck = sp == 0 ? a.rk / CE : kHeadDim / CE;
      const int ncv = sp == 0 ? a.rv / CE : kHeadDim / CE;
      const int rvd = sp == 0 ? a.rv : kHeadDim;
      int TS = 1;
      while (TS * 2 * ncv <= 32) TS *= 2;
      const int jc = lane / TS, tsub = lane - jc * TS;
      const int qdim = sp == 0 ? a.rk : kHeadDim;
      float* part = sp == 0 ? a.part_lat : a.part_fr;
      const int rec_stride = hdr_floats(G) + G * rvd;
      int t = lo;
      while (t < hi) {
        int b, kvh, i0, tiles;
        locate(start, a.B, a.H_kv, t, b, kvh, i0, tiles);
        const int unit = b * a.H_kv + kvh;
        const int ustart = t - i0;
        const int ce = min(hi, ustart + tiles);
        const int ntok = space_tokens(a, sp, b);
        float* qc = qv + min(chunk, kMaxPre) * G * kHeadDim;
        if (chunk >= kMaxPre) {
          fetch_queries<G>(a, sp, b, kvh, qc, ctid);
          named_bar(kBarConsumers, kCThreads);
        }
        ++chunk;
        float m[G], l[G];
        float2 acc[G][NP];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
          for (int e = 0; e < NP; ++e) acc[h][e] = make_float2(0.f, 0.f);
        }
        const int k0 = kbase + (t - lo);
        for (int tt = t + ((w - k0 % kConsumers) + kConsumers) % kConsumers; tt < ce;
             tt += kConsumers) {
          const int k = kbase + (tt - lo), s = k % a.NS, n = k / a.NS;
          if (!tag_wait_bounded(tag + s, k) || !mbar_wait_bounded(&full[s], n & 1)) {
            *a.err = kErrTimeout;
            flags[0] = 1;
            break;
          }
          const int it = tt - ustart;
          const uint4* st = reinterpret_cast<const uint4*>(ring + (size_t)s * a.stage_bytes);
          if (sp == 0)
            process_tile<T, G, kLatPage>(st, min(kLatPage, ntok - it * kLatPage), nck, ncv, TS,
                                         qc, qdim, pbuf, m, l, acc, lane);
          else
            process_tile<T, G, kFrTile>(st, min(kFrTile, ntok - it * kFrTile), nck, ncv, TS,
                                        qc, qdim, pbuf, m, l, acc, lane);
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        // ---- combine the warps' partials into one record for (unit, CTA)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float lt = warp_sum(l[h]);
          if (lane == 0) { cml[w * 2 * G + h] = m[h]; cml[w * 2 * G + G + h] = lt; }
        }
        for (int o = TS >> 1; o > 0; o >>= 1)
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < NP; ++e) {
              acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
              acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
            }
        named_bar(kBarConsumers, kCThreads);
        if (tsub == 0 && jc < ncv) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float M = -INFINITY;
            for (int ww = 0; ww < kConsumers; ++ww) M = fmaxf(M, cml[ww * 2 * G + h]);
            const float sc = m[h] > -INFINITY ? exp2f(m[h] - M) : 0.f;
            if (sc != 0.f)
#pragma unroll
              for (int e = 0; e < NP; ++e) {
                atomicAdd(&cacc[h * rvd + jc * CE + 2 * e], acc[h][e].x * sc);
                atomicAdd(&cacc[h * rvd + jc * CE + 2 * e + 1], acc[h][e].y * sc);
              }
          }
        }
        named_bar(kBarConsumers, kCThreads);
        if (w == 0) {
          float* rec = part + (size_t)(unit + c) * rec_stride;
          if (lane < G) {
            float M = -INFINITY;
            for (int ww = 0; ww < kConsumers; ++ww) M = fmaxf(M, cml[ww * 2 * G + lane]);
            float L = 0.f;
            for (int ww = 0; ww < kConsumers; ++ww) {
              const float mw = cml[ww * 2 * G + lane];
              if (mw > -INFINITY) L += exp2f(mw - M) * cml[ww * 2 * G + G + lane];
            }
            rec[lane] = M;
            rec[G + lane] = L;
          }
          const int H = hdr_floats(G);
          for (int x = lane; x < G * rvd; x += 32) {
            rec[H + x] = cacc[x];
            cacc[x] = 0.f;
          }
          __syncwarp();
          if (lane == 0) {
            __threadfence();
            const int need = (start_lat[b + 1] - start_lat[b]) / a.H_kv +
                             (start_fr[b + 1] - start_fr[b]) / a.H_kv;
            const int got = atomicAdd(&a.unit_cnt[unit], ce - t) + (ce - t);
            flags[1] = (got == need);
            flags[2] = *(volatile int*)&flags[0];
            if (got == need) __threadfence();
          }
        }
        named_bar(kBarConsumers, kCThreads);
        if (flags[1])
          finalize_unit<T, G>(a, unit, start_lat, start_fr,
                              reinterpret_cast<float*>(smem + sp_.fin_lat),
                              reinterpret_cast<int*>(smem + sp_.recs), ctid);
        t = ce;
        if (flags[2]) break;  // uniform: written before the last named barrier
      }
      if (flags[2]) break;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------ host side
struct Plan {
  int C, NS, stage_bytes, smem;
  size_t off_cnt, off_qlat, off_qfr, off_lat, off_fr, total;
};

static int plan_decode(int B, int H_kv, int H_q, int rk, int rv, bool has_lat, bool has_fr,
                       int esize, Plan& p) {
  int dev = 0, sms = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LRKV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LRKV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return LRKV_ERR_CUDA;
  const int G = H_q / H_kv;
  const int lat_b = has_lat ? kLatPage * (rk + rv) * esize : 0;
  const int fr_b = has_fr ? 2 * kFrTile * kHeadDim * esize : 0;  // key + value
  p.stage_bytes = std::max(lat_b, fr_b);
  const int fixed = smem_plan(0, p.stage_bytes, B, G).total + 1024;
  p.NS = std::min(kMaxStages, (optin - fixed) / p.stage_bytes);
  p.NS -= p.NS % kProducers;
  if (p.NS < kProducers) return LRKV_ERR_UNSUPPORTED;
  p.smem = smem_plan(p.NS, p.stage_bytes, B, G).total;
  p.C = sms;
  const int U = B * H_kv;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 256;
  p.off_cnt = off;  off = al(off + (size_t)U * 4);
  p.off_qlat = off; off = al(off + (size_t)B * H_q * (has_lat ? rk : 0) * 4);
  p.off_qfr = off;  off = al(off + (size_t)B * H_q * (has_fr ? kHeadDim : 0) * 4);
  const size_t slots = (size_t)(U + p.C - 1);
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
static int launch_decode_t(const DecodeArgs& a, const Plan& p, cudaStream_t st) {
  qfold_kernel<T, G><<<a.B * a.H_kv, 256, 0, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  if (cudaFuncSetAttribute(split_kernel<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           p.smem) != cudaSuccess)
    return LRKV_ERR_CUDA;
  // Programmatic dependent launch: the split kernel's producers start
  // streaming while the q-fold finishes; its consumers wait for it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, split_kernel<T, G>, a) != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

template <typename T>
static int launch_decode_g(const DecodeArgs& a, const Plan& p, cudaStream_t st) {
  switch (a.G) {
    case 1: return launch_decode_t<T, 1>(a, p, st);
    case 2: return launch_decode_t<T, 2>(a, p, st);
    case 4: return launch_decode_t<T, 4>(a, p, st);
    case 8: return launch_decode_t<T, 8>(a, p, st);
    default: return LRKV_ERR_UNSUPPORTED;
  }
}

int decode_launch(const DecodeLaunch& L, cudaStream_t st) {
  const bool has_lat = L.codes != nullptr, has_fr = L.fr != nullptr;
  const int es = L.dtype == LRKV_BF16 ? 2 : 4;
  Plan p;
  int rc = plan_decode(L.B, L.H_kv, L.H_q, L.rk, L.rv, has_lat, has_fr, es, p);
  if (rc != LRKV_OK) return rc;
  if (L.ws_bytes < p.total) return LRKV_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(L.ws);
  DecodeArgs a;
  a.B = L.B; a.H_kv = L.H_kv; a.G = L.H_q / L.H_kv; a.H_q = L.H_q;
  a.seq_len = L.seq_len; a.n_sink = L.n_sink; a.W = L.W;
  a.codes = L.codes; a.bt_lat = L.bt_lat; a.maxp_lat = L.maxp_lat;
  a.rk = L.rk; a.rv = L.rv;
  a.fr = L.fr; a.bt_fr = L.bt_fr; a.maxp_fr = L.maxp_fr;
  a.num_pages_lat = L.num_pages_lat; a.num_pages_fr = L.num_pages_fr;
  a.P_v = L.P_v; a.basis_bs = L.basis_bs; a.o = L.o;
  a.q = L.q; a.P_k = L.P_k; a.qscale = L.scale * kLog2e;
  a.err = reinterpret_cast<int*>(ws);
  a.unit_cnt = reinterpret_cast<int*>(ws + p.off_cnt);
  a.qlat = reinterpret_cast<float*>(ws + p.off_qlat);
  a.qfr = reinterpret_cast<float*>(ws + p.off_qfr);
  a.part_lat = reinterpret_cast<float*>(ws + p.off_lat);
  a.part_fr = reinterpret_cast<float*>(ws + p.off_fr);
  a.C = p.C; a.NS = p.NS; a.stage_bytes = p.stage_bytes;
  if (L.dtype == LRKV_BF16) return launch_decode_g<__nv_bfloat16>(a, p, st);
  return launch_decode_g<float>(a, p, st);
}

}  // namespace lrkv
