// Decode attention over the latent code cache plus full-rank anchors.
//
// Three launches per call, stream-ordered; the second and third use
// programmatic dependent launch so they start while their predecessor ends.
//  1. qfold : per (sequence, KV head) unit, q~ = P_k^T q for its G query
//             heads (Half the Memory, section 08: attend directly against the
//             codes) and the full-rank q, both pre-scaled by scale * log2(e)
//             so the softmax runs on exp2.
//  2. split : persistent, one CTA per SM.  The latent pages of all units are
//             laid end to end and each CTA takes an equal contiguous range,
//             so any mix of sequence lengths is balanced.  A producer warp
//             streams one slab per page into a shared-memory ring with bulk
//             copies completing on mbarriers (addresses computed a batch
//             ahead).  Eight consumer warps take every eighth page: scores
//             with lane = token (q chunks broadcast from shared memory,
//             packed fp32 FMA), an exp2 online softmax with one max per page,
//             then p * c_v with lanes split over value chunks.  Each warp
//             writes its own partial (m, l, acc) record per unit it touched;
//             warps never wait for one another.  An anchor warp processes
//             this CTA's share of the full-rank anchor tiles straight from
//             global memory while the pages stream, and writes one record per
//             unit.  (The dense baseline streams its full-rank pages through
//             the ring instead and has no anchor warp.)
//  3. merge : per unit, combines every record (running max, rescaled sums),
//             up-projects the latent accumulator, o = (P_v acc_lat + acc_fr)
//             / l, and writes zeros for sequences with no tokens.
#include <limits.h>
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kConsumers = 8;                  // consumer warps per CTA
constexpr int kProducerWarp = 0;
constexpr int kAnchorWarp = 1;
constexpr int kFirstConsumer = 2;
constexpr int kThreads = 32 * (kFirstConsumer + kConsumers);
constexpr int kMaxStages = 24;
constexpr int kIssue = 4;                      // producer lanes issuing at once
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergeBuf = 64 * 1024;           // merge: bytes of records per chunk
constexpr int kMergeMaxRec = 256;              // merge: records per chunk at most
constexpr int kBarRecords = 1;                 // consumers: a unit's warp records are written

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
  const int* bt_fr;  // nullptr: anchors (tiles of a unit contiguous), else dense pages
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
  float* qlat;         // [B][H_q][rk] folded queries (scaled)
  float* qfr;          // [B][H_q][128] scaled queries
  float* part_lat;     // [U + C - 1] latent records, one per (CTA, unit)
  float* part_fr;      // [U + C - 1] full-rank records, one per (CTA, unit)
  int C;               // CTAs of the split grid
  int NS;              // ring stages
  int stage_bytes;
  int dq_bytes;        // int8 codes: per-consumer dequantised half page (bytes);
                       // value-amortised slabs: per-consumer page weights
  const float* A;      // value-amortised slabs: predictors [B][H_kv][rk][rv]
  int rw;              // latent record width per head: rv, or rk + rv (amortised)
  int wait_first;      // 1: the previous grid (a step's append) writes the cache
  int fold_split;      // q-fold CTAs per unit (each folds at most 32 columns)
  int combine;         // 1: one ring-space record per (CTA, unit), the consumer
                       // warps' records combined in shared memory; 0: one per warp
};

constexpr int kModePlain = 0;  // bf16 / fp32 latent codes
constexpr int kModeQ8 = 1;     // per-token int8 codes + scales
constexpr int kModeVA = 2;     // key codes + value residual slots

__host__ __device__ inline int hdr_floats(int G) { return ((2 * G + 3) / 4) * 4; }

__device__ inline int tiles_lat(int n) { return (n + kLatPage - 1) / kLatPage; }
__device__ inline int tiles_fr(int n) { return (n + kFrTile - 1) / kFrTile; }

// First tile of CTA c when `total` tiles are split evenly over C CTAs:
// floor(c * total / C), in 32-bit arithmetic (c * (total % C) < C * C).
__device__ inline int range_lo(int c, int total, int C) {
  const int q = total / C, r = total - q * C;
  return c * q + (c * r) / C;
}
// CTAs a space of `total` tiles is spread over: at most one tile per CTA
// short of the grid, so a small space keeps its records in few CTAs' slots
// (the merge folds fewer records).  CTAs c >= ctas_for(...) own no tile.
__device__ inline int ctas_for(int total, int C) { return total < C ? total : C; }
// Tiles [lo, hi) of CTA c in a space of `total` tiles over a grid of C CTAs.
__device__ inline void cta_range(int c, int total, int C, int& lo, int& hi) {
  const int Ce = ctas_for(total, C);
  if (c >= Ce) {
    lo = hi = total;
    return;
  }
  lo = range_lo(c, total, Ce);
  hi = range_lo(c + 1, total, Ce);
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

// ------------------------------------------------------------ tensor-core tile math (bf16)
// The same page computation on the tensor cores, one warp per page.
//  scores:  S^T (m = token, n = head) = C_k (token x dim) . q~^T, q~ split
//           as hi + lo bf16 so the product keeps about 16 mantissa bits;
//  softmax: per head over the page's tokens (shuffles across the lanes of
//           one column pair), p split as hi + lo bf16 like q~;
//  values:  acc^T (m = value dim, n = head) += C_v^T (dim x token) . P^T.
// The chunk-major page layout (16-byte rows = 8 elements of one token) is
// what ldmatrix reads: plain for C_k rows, transposed for C_v^T.  P moves
// from the score accumulator into the value step's B operand by movmatrix.
// Heads G..7 of the n = 8 tile are padding (zero queries, never stored).
// KS / VB: 16-wide steps of the score / value rows the code is built for
// (a rank class: r_k <= 16 KS, r_v <= 16 VB); the actual counts may be lower.
template <int KS>
struct QFrag {
  uint32_t hi[KS][2], lo[KS][2];  // B operands (k = dim, n = head)
};

// q~ rows of the unit's G heads (qv: row of head 0, rows qdim apart, in the
// workspace) -> B fragments.
template <int G, int KS>
__device__ inline void load_qfrag(const float* qv, int qdim, int lane, QFrag<KS>& f) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int s = 0; s < KS; ++s)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int d = 16 * s + 8 * r + 2 * t;
      float x0 = 0.f, x1 = 0.f;
      if (g < G && d < qdim) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(qv + g * qdim + d));
        x0 = x.x;
        x1 = x.y;
      }
      const uint32_t h = pack_bf16x2(x0, x1);
      f.hi[s][r] = h;
      f.lo[s][r] = pack_bf16x2(x0 - bf_lo(h), x1 - bf_hi(h));
    }
}

// Zero the bf16 halves of a (token k, token k + 1) pair that lie at or past n.
__device__ __forceinline__ uint32_t mask_tokens(uint32_t x, int k, int n) {
  return (k < n ? x & 0xffffu : 0u) | (k + 1 < n ? x & 0xffff0000u : 0u);
}

// One page (TT tokens) of a ring stage; running state per lane: m, l for
// heads 2t and 2t + 1 (l is this lane's partial), acc fragments per 16 value
// dims, kept apart for the hi and lo halves of p (shorter MMA chains; the
// record sums them).
template <int TT, int KS, int VB>
__device__ __forceinline__ void process_tile_mma(const uint4* kch, int n_valid, int nck, int ncv,
                                                 const QFrag<KS>& qf, float (&m)[2],
                                                 float (&l)[2], float (&acc)[2][VB][4],
                                                 int lane) {
  constexpr int MB = TT / 16;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t kbase = smem_u32(kch), vbase = smem_u32(kch + nck * TT);
  const int nks = (nck + 1) >> 1, nvb = (ncv + 1) >> 1;
  const bool partial = n_valid < TT;

  // Phase A (an odd last chunk is read twice; its q~ half is zero)
  float sc[MB][4], sl[MB][4];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[mb][i] = sl[mb][i] = 0.f;
  // (rows of tokens past n_valid are read but masked below)
  const int arow = lane & 15, ahalf = lane >> 4;
#pragma unroll
  for (int s = 0; s < KS; ++s) {
    if (s < nks) {
      const int c = min(2 * s + ahalf, nck - 1);
      uint32_t a[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
        ldsm_x4(kbase + (uint32_t)((c * TT + mb * 16 + arow) * 16), a[mb]);
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) mma_bf16_16816(sc[mb], a[mb], qf.hi[s][0], qf.hi[s][1]);
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) mma_bf16_16816(sl[mb], a[mb], qf.lo[s][0], qf.lo[s][1]);
    }
  }
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[mb][i] += sl[mb][i];

  // Online softmax, one running max per head updated once per page
  float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    if (partial) {
      if (mb * 16 + g >= n_valid) sc[mb][0] = sc[mb][1] = -INFINITY;
      if (mb * 16 + g + 8 >= n_valid) sc[mb][2] = sc[mb][3] = -INFINITY;
    }
    mt0 = fmaxf(mt0, fmaxf(sc[mb][0], sc[mb][2]));
    mt1 = fmaxf(mt1, fmaxf(sc[mb][1], sc[mb][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, o));
    mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, o));
  }
  const float mn0 = fmaxf(m[0], mt0), mn1 = fmaxf(m[1], mt1);
  const float al0 = ex2_approx(m[0] - mn0), al1 = ex2_approx(m[1] - mn1);
  m[0] = mn0;
  m[1] = mn1;
  // p as hi + lo bf16 B operands (k = token, n = head)
  float ps0 = 0.f, ps1 = 0.f;
  uint32_t ph[MB][2], pl[MB][2];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    const float p0 = ex2_approx(sc[mb][0] - mn0), p1 = ex2_approx(sc[mb][1] - mn1);
    const float p2 = ex2_approx(sc[mb][2] - mn0), p3 = ex2_approx(sc[mb][3] - mn1);
    ps0 += p0 + p2;
    ps1 += p1 + p3;
    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
    ph[mb][0] = movmatrix_trans(h01);
    ph[mb][1] = movmatrix_trans(h23);
    pl[mb][0] = movmatrix_trans(pack_bf16x2(p0 - bf_lo(h01), p1 - bf_hi(h01)));
    pl[mb][1] = movmatrix_trans(pack_bf16x2(p2 - bf_lo(h23), p3 - bf_hi(h23)));
  }
  l[0] = fmaf(l[0], al0, ps0);
  l[1] = fmaf(l[1], al1, ps1);

  // Phase B
#pragma unroll
  for (int hl = 0; hl < 2; ++hl)
#pragma unroll
    for (int vb = 0; vb < VB; ++vb) {
      acc[hl][vb][0] *= al0;
      acc[hl][vb][1] *= al1;
      acc[hl][vb][2] *= al0;
      acc[hl][vb][3] *= al1;
    }
  const int vrow = ((lane >> 4) << 3) + (lane & 7), vhalf = (lane >> 3) & 1;
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    if (mb * 16 < n_valid) {
#pragma unroll
      for (int vb = 0; vb < VB; ++vb) {
        if (vb < nvb) {
          const int c = min(2 * vb + vhalf, ncv - 1);
          uint32_t a[4];
          ldsm_x4_trans(vbase + (uint32_t)((c * TT + mb * 16 + vrow) * 16), a);
          if (partial) {
            const int k0 = mb * 16 + 2 * t;
            a[0] = mask_tokens(a[0], k0, n_valid);
            a[1] = mask_tokens(a[1], k0, n_valid);
            a[2] = mask_tokens(a[2], k0 + 8, n_valid);
            a[3] = mask_tokens(a[3], k0 + 8, n_valid);
          }
          mma_bf16_16816(acc[0][vb], a, ph[mb][0], ph[mb][1]);
          mma_bf16_16816(acc[1][vb], a, pl[mb][0], pl[mb][1]);
        }
      }
    }
  }
}

// The warp's (m, l, acc) of the tensor-core path -> record (m[G], l[G], acc [G][rvd]).
template <int G, int VB>
__device__ inline void write_record_mma(float* rec, int rvd, const float (&m)[2],
                                        const float (&l)[2], const float (&acc)[2][VB][4],
                                        int lane) {
  const int g = lane >> 2, t = lane & 3, H = hdr_floats(G);
  float l0 = l[0], l1 = l[1];
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int h0 = 2 * t, h1 = 2 * t + 1;
  if (g == 0) {
    if (h0 < G) { rec[h0] = m[0]; rec[G + h0] = l0; }
    if (h1 < G) { rec[h1] = m[1]; rec[G + h1] = l1; }
  }
#pragma unroll
  for (int vb = 0; vb < VB; ++vb)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int d = vb * 16 + g + 8 * r;
      if (d < rvd) {
        if (h0 < G) rec[H + h0 * rvd + d] = acc[0][vb][2 * r] + acc[1][vb][2 * r];
        if (h1 < G) rec[H + h1 * rvd + d] = acc[0][vb][2 * r + 1] + acc[1][vb][2 * r + 1];
      }
    }
}

// One value-amortised page (64 tokens): the scores and the online softmax as
// in process_tile_mma; then acck += p c_k over the key codes (the value
// prediction A^T c_k is linear, so the merge applies A to the sum once), and
// acce += p e over the page's residual slots, whose token rows come from the
// slab (a slot with row -1, or at or past n_valid, weighs 0).  pw: this
// warp's [64][8] fp32 page weights, so a slot can find its token's weight.
template <int KS, int VB>
__device__ __forceinline__ void process_tile_va(const uint4* kch, int n_valid, int nck, int ncv,
                                                const QFrag<KS>& qf, float (&m)[2], float (&l)[2],
                                                float (&acck)[2][KS][4], float (&acce)[VB][4],
                                                float* pw, int lane) {
  constexpr int TT = kLatPage, MB = TT / 16;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t kbase = smem_u32(kch);
  const uint32_t rbase = kbase + (uint32_t)(TT * nck * 16);  // residual rows [ncv][16][8]
  const int* sidx = reinterpret_cast<const int*>(reinterpret_cast<const uint8_t*>(kch) +
                                                 TT * nck * 16 + kVaKeep * ncv * 16);
  const int nks = (nck + 1) >> 1, nvb = (ncv + 1) >> 1;
  const bool partial = n_valid < TT;

  float sc[MB][4], sl[MB][4];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[mb][i] = sl[mb][i] = 0.f;
  const int arow = lane & 15, ahalf = lane >> 4;
#pragma unroll
  for (int s = 0; s < KS; ++s) {
    if (s < nks) {
      const int c = min(2 * s + ahalf, nck - 1);
      uint32_t a[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
        ldsm_x4(kbase + (uint32_t)((c * TT + mb * 16 + arow) * 16), a[mb]);
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) mma_bf16_16816(sc[mb], a[mb], qf.hi[s][0], qf.hi[s][1]);
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) mma_bf16_16816(sl[mb], a[mb], qf.lo[s][0], qf.lo[s][1]);
    }
  }
  float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[mb][i] += sl[mb][i];
    if (partial) {
      if (mb * 16 + g >= n_valid) sc[mb][0] = sc[mb][1] = -INFINITY;
      if (mb * 16 + g + 8 >= n_valid) sc[mb][2] = sc[mb][3] = -INFINITY;
    }
    mt0 = fmaxf(mt0, fmaxf(sc[mb][0], sc[mb][2]));
    mt1 = fmaxf(mt1, fmaxf(sc[mb][1], sc[mb][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, o));
    mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, o));
  }
  const float mn0 = fmaxf(m[0], mt0), mn1 = fmaxf(m[1], mt1);
  const float al0 = ex2_approx(m[0] - mn0), al1 = ex2_approx(m[1] - mn1);
  m[0] = mn0;
  m[1] = mn1;
  float ps0 = 0.f, ps1 = 0.f;
  uint32_t ph[MB][2], pl[MB][2];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    const float p0 = ex2_approx(sc[mb][0] - mn0), p1 = ex2_approx(sc[mb][1] - mn1);
    const float p2 = ex2_approx(sc[mb][2] - mn0), p3 = ex2_approx(sc[mb][3] - mn1);
    ps0 += p0 + p2;
    ps1 += p1 + p3;
    // weights by (token row, head) for the residual slots
    pw[(mb * 16 + g) * 8 + 2 * t] = p0;
    pw[(mb * 16 + g) * 8 + 2 * t + 1] = p1;
    pw[(mb * 16 + g + 8) * 8 + 2 * t] = p2;
    pw[(mb * 16 + g + 8) * 8 + 2 * t + 1] = p3;
    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
    ph[mb][0] = movmatrix_trans(h01);
    ph[mb][1] = movmatrix_trans(h23);
    pl[mb][0] = movmatrix_trans(pack_bf16x2(p0 - bf_lo(h01), p1 - bf_hi(h01)));
    pl[mb][1] = movmatrix_trans(pack_bf16x2(p2 - bf_lo(h23), p3 - bf_hi(h23)));
  }
  l[0] = fmaf(l[0], al0, ps0);
  l[1] = fmaf(l[1], al1, ps1);
#pragma unroll
  for (int kb = 0; kb < KS; ++kb)
#pragma unroll
    for (int hl = 0; hl < 2; ++hl) {
      acck[hl][kb][0] *= al0;
      acck[hl][kb][1] *= al1;
      acck[hl][kb][2] *= al0;
      acck[hl][kb][3] *= al1;
    }
#pragma unroll
  for (int vb = 0; vb < VB; ++vb) {
    acce[vb][0] *= al0;
    acce[vb][1] *= al1;
    acce[vb][2] *= al0;
    acce[vb][3] *= al1;
  }
  // acck^T (key dim x head) += C_k^T . P^T over the page's tokens
  const int vrow = ((lane >> 4) << 3) + (lane & 7), vhalf = (lane >> 3) & 1;
#pragma unroll
  for (int mb = 0; mb < MB; ++mb) {
    if (mb * 16 < n_valid) {
#pragma unroll
      for (int kb = 0; kb < KS; ++kb) {
        if (kb < nks) {
          const int c = min(2 * kb + vhalf, nck - 1);
          uint32_t a[4];
          ldsm_x4_trans(kbase + (uint32_t)((c * TT + mb * 16 + vrow) * 16), a);
          if (partial) {
            const int k0 = mb * 16 + 2 * t;
            a[0] = mask_tokens(a[0], k0, n_valid);
            a[1] = mask_tokens(a[1], k0, n_valid);
            a[2] = mask_tokens(a[2], k0 + 8, n_valid);
            a[3] = mask_tokens(a[3], k0 + 8, n_valid);
          }
          mma_bf16_16816(acck[0][kb], a, ph[mb][0], ph[mb][1]);
          mma_bf16_16816(acck[1][kb], a, pl[mb][0], pl[mb][1]);
        }
      }
    }
  }
  __syncwarp();  // pw is complete
  // acce^T (value dim x head) += E^T . P_slots^T over the 16 residual slots
  auto slot_p = [&](int sl) {
    const int r = sidx[sl];
    return (r >= 0 && r < n_valid) ? pw[r * 8 + g] : 0.f;
  };
  const uint32_t b0 = pack_bf16x2(slot_p(2 * t), slot_p(2 * t + 1));
  const uint32_t b1 = pack_bf16x2(slot_p(2 * t + 8), slot_p(2 * t + 9));
#pragma unroll
  for (int vb = 0; vb < VB; ++vb) {
    if (vb < nvb) {
      const int c = min(2 * vb + vhalf, ncv - 1);
      uint32_t a[4];
      ldsm_x4_trans(rbase + (uint32_t)((c * kVaKeep + vrow) * 16), a);
      mma_bf16_16816(acce[vb], a, b0, b1);
    }
  }
  __syncwarp();  // pw may be rewritten by the next page
}

// The warp's (m, l, acck, acce) of the value-amortised path -> record
// (m[G], l[G], then per head [rk] key-code sums and [rv] residual sums).
template <int G, int KS, int VB>
__device__ inline void write_record_va(float* rec, int rk, int rv, const float (&m)[2],
                                       const float (&l)[2], const float (&acck)[2][KS][4],
                                       const float (&acce)[VB][4], int lane) {
  const int g = lane >> 2, t = lane & 3, H = hdr_floats(G), rw = rk + rv;
  float l0 = l[0], l1 = l[1];
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int h0 = 2 * t, h1 = 2 * t + 1;
  if (g == 0) {
    if (h0 < G) { rec[h0] = m[0]; rec[G + h0] = l0; }
    if (h1 < G) { rec[h1] = m[1]; rec[G + h1] = l1; }
  }
#pragma unroll
  for (int kb = 0; kb < KS; ++kb)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int d = kb * 16 + g + 8 * r;
      if (d < rk) {
        if (h0 < G) rec[H + h0 * rw + d] = acck[0][kb][2 * r] + acck[1][kb][2 * r];
        if (h1 < G) rec[H + h1 * rw + d] = acck[0][kb][2 * r + 1] + acck[1][kb][2 * r + 1];
      }
    }
#pragma unroll
  for (int vb = 0; vb < VB; ++vb)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int d = vb * 16 + g + 8 * r;
      if (d < rv) {
        if (h0 < G) rec[H + h0 * rw + rk + d] = acce[vb][2 * r];
        if (h1 < G) rec[H + h1 * rw + rk + d] = acce[vb][2 * r + 1];
      }
    }
}

// ------------------------------------------------------------ q-fold kernel
constexpr int kFoldThreads = 128;  // small, so q-fold CTAs fit beside split CTAs
constexpr int kFoldSplit = 2;      // CTAs per unit at least, each folding a share of the columns

template <typename T, int G>
__global__ void __launch_bounds__(kFoldThreads) qfold_kernel(DecodeArgs a) {
  __shared__ float qs[G * kHeadDim];
  __shared__ float red[G * kFoldThreads];
  pdl_trigger();
  const int unit = blockIdx.x / a.fold_split, part = blockIdx.x % a.fold_split;
  const int b = unit / a.H_kv, kvh = unit - b * a.H_kv, tid = threadIdx.x;
  const size_t h0 = (size_t)b * a.H_q + (size_t)kvh * G;
  const T* q = static_cast<const T*>(a.q) + h0 * kHeadDim;
  // This CTA folds columns [c0, c1) (at most 32); thread -> (column j,
  // segment of at most 32 rows).  Its P_k loads do not depend on q, so they
  // are issued first and land together with the query rows (the split
  // kernel's stream is already running, so every round trip here is long).
  const int rk = a.codes ? a.rk : 0, cper = (rk + a.fold_split - 1) / a.fold_split;
  const int c0 = part * cper, c1 = min(rk, c0 + cper), nc = max(0, c1 - c0);
  const int nseg = nc > 0 ? max(1, kFoldThreads / nc) : 1, rows = (kHeadDim + nseg - 1) / nseg;
  int j = 0, seg = 0, nrow = 0;
  if (nc > 0 && tid < nseg * nc) {
    j = c0 + tid % nc;
    seg = tid / nc;
    nrow = min(rows, kHeadDim - seg * rows);
  }
  float pij[32];  // rows <= 32 (at most 32 columns per CTA)
  {
    const float* P = a.P_k + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * rk + j;
    const uint64_t pol = l2_evict_last_policy();
#pragma unroll
    for (int u = 0; u < 32; ++u)
      pij[u] = u < nrow ? ldg_f_hint(P + (size_t)(seg * rows + u) * rk, pol) : 0.f;
  }
  for (int x = tid; x < G * kHeadDim; x += kFoldThreads) qs[x] = to_f<T>(q[x]);
  __syncthreads();
  if (part == 0) {
    if (a.fr)
      for (int x = tid; x < G * kHeadDim; x += kFoldThreads)
        a.qfr[h0 * kHeadDim + x] = qs[x] * a.qscale;
  }
  if (nc <= 0) return;  // no latent space, or no columns for this CTA (uniform)
  if (nrow > 0) {
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    const int i0 = seg * rows;
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if (u < nrow)
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = fmaf(pij[u], qs[g * kHeadDim + i0 + u], acc[g]);
#pragma unroll
    for (int g = 0; g < G; ++g) red[(seg * G + g) * nc + (j - c0)] = acc[g];
  }
  __syncthreads();
  for (int x = tid; x < G * nc; x += kFoldThreads) {
    const int g = x / nc, jj = x - g * nc;
    float sum = 0.f;
    for (int sg = 0; sg < nseg; ++sg) sum += red[(sg * G + g) * nc + jj];
    a.qlat[h0 * rk + g * rk + c0 + jj] = sum * a.qscale;
  }
}


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

// True when the anchor warp (not the ring) handles the full-rank space.
__host__ __device__ inline bool anchor_mode(const void* fr, const int* bt_fr) {
  return fr != nullptr && bt_fr == nullptr;
}

// Shared-memory plan of the split kernel (byte offsets from the base).
struct SmemPlan {
  int ring, full, empty, tag, start_lat, start_fr, pbuf, qown, wrec, flags, dq, total;
};
// tc: the consumers run on the tensor cores and keep their query fragments in
// registers, so only the anchor warp needs probability and query slices.
// dq_bytes: per consumer warp, the bf16 form of half an int8 page.
// rvd: record width per head of the ring space (r_v, r_k + r_v, or 128).
__host__ __device__ inline SmemPlan smem_plan(int NS, int stage_bytes, int B, int G, bool tc,
                                              int dq_bytes, int rvd) {
  const int slots = tc ? 1 : kConsumers + 1;
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
  // per consumer warp and the anchor warp: probabilities [G][64] as pairs and
  // the unit's folded queries [G][128]
  p.pbuf = take(slots * kLatPage * G * 8, 16);
  p.qown = take(slots * G * kHeadDim * 4, 16);
  // the consumer warps' records of one unit, combined into the CTA's record
  p.wrec = take(kConsumers * (hdr_floats(G) + G * rvd) * 4, 16);
  p.flags = take(16, 16);
  p.dq = take(kConsumers * dq_bytes, 128);
  p.total = off;
  return p;
}

// The folded queries of unit (b, kvh) for space sp -> dst (one warp).
template <int G>
__device__ inline void fetch_queries_warp(const DecodeArgs& a, int sp, int b, int kvh,
                                          float* dst, int lane) {
  const int dim = sp == 0 ? a.rk : kHeadDim;
  const float4* src = reinterpret_cast<const float4*>(
      (sp == 0 ? a.qlat : a.qfr) + ((size_t)b * a.H_q + (size_t)kvh * G) * dim);
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int x = lane; x < G * dim / 4; x += 32) d4[x] = __ldcg(src + x);
  __syncwarp();
}

// A warp's partial (m, l, acc) -> record rec: m[G], l[G] then acc [G][rvd].
// The lanes hold acc for value chunk jc of tokens tsub (TS lanes per chunk).
template <typename T, int G>
__device__ inline void write_record(float* rec, int rvd, int TS, int ncv, const float (&m)[G],
                                    const float (&l)[G], float2 (&acc)[G][Elem<T>::CE / 2],
                                    int lane) {
  constexpr int CE = Elem<T>::CE, NP = CE / 2;
  const int H = hdr_floats(G);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float lt = warp_sum(l[h]);
    if (lane == 0) { rec[h] = m[h]; rec[G + h] = lt; }
  }
  for (int o = TS >> 1; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
        acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
      }
  const int jc = lane / TS, tsub = lane - jc * TS;
  if (tsub == 0 && jc < ncv)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float4* dst = reinterpret_cast<float4*>(rec + H + h * rvd + jc * CE);
#pragma unroll
      for (int e4 = 0; e4 < NP / 2; ++e4)
        dst[e4] = make_float4(acc[h][2 * e4].x, acc[h][2 * e4].y, acc[h][2 * e4 + 1].x,
                              acc[h][2 * e4 + 1].y);
    }
}

// One full-rank anchor tile of 32 tokens read straight from global memory by
// one warp (no ring stage): lane = token for the scores, lanes split over
// value chunks for the accumulation.  Same math as process_tile.
template <typename T, int G>
__device__ void anchor_tile(const uint4* kch, int n_valid, const float* qv, float2* pbuf,
                            float (&m)[G], float (&l)[G], float2 (&acc)[G][Elem<T>::CE / 2],
                            int lane) {
  constexpr int CE = Elem<T>::CE, NP = CE / 2, TT = kFrTile, NC = kHeadDim / CE;
  const uint4* vch = kch + NC * TT;
  // Phase A: the lane's key chunks, eight loads in flight at a time.
  float2 s2[G];
#pragma unroll
  for (int h = 0; h < G; ++h) s2[h] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j0 = 0; j0 < NC; j0 += 8) {
    uint4 kc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      kc[u] = lane < n_valid ? __ldcs(kch + (j0 + u) * TT + lane) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u;
      float2 f[NP];
      chunk_pairs<T>(kc[u], f);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4* src = reinterpret_cast<const float4*>(qv + h * kHeadDim + j * CE);
#pragma unroll
        for (int e4 = 0; e4 < NP / 2; ++e4) {
          const float4 x = src[e4];
          fma2(s2[h], make_float2(x.x, x.y), f[2 * e4]);
          fma2(s2[h], make_float2(x.z, x.w), f[2 * e4 + 1]);
        }
      }
    }
  }
  float alpha[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float sc = lane < n_valid ? s2[h].x + s2[h].y : -INFINITY;
    const float mn = fmaxf(m[h], warp_max(sc));
    alpha[h] = exp2f(m[h] - mn);
    m[h] = mn;
    const float pr = exp2f(sc - mn);
    l[h] = l[h] * alpha[h] + pr;
    pbuf[h * TT + lane] = make_float2(pr, pr);
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float2 a2 = make_float2(alpha[h], alpha[h]);
#pragma unroll
    for (int e = 0; e < NP; ++e) acc[h][e] = mul2(acc[h][e], a2);
  }
  // Phase B: lane -> (value chunk jc, token parity tsub); loads first.
  constexpr int TS = 32 / NC;  // 2 (bf16) or 1 (fp32)
  const int jc = lane / TS, tsub = lane - jc * TS;
  constexpr int STEPS = TT / TS;
#pragma unroll
  for (int i0 = 0; i0 < STEPS; i0 += 8) {  // eight loads in flight at a time
    uint4 vc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = (i0 + u) * TS + tsub;
      vc[u] = t < n_valid ? __ldcs(vch + jc * TT + t) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = (i0 + u) * TS + tsub;
      if (t < n_valid) {
        float2 f[NP];
        chunk_pairs<T>(vc[u], f);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float2 pp = pbuf[h * TT + t];
#pragma unroll
          for (int e = 0; e < NP; ++e) fma2(acc[h][e], pp, f[e]);
        }
      }
    }
  }
  __syncwarp();
}

// Half `half` (32 tokens) of an int8 latent slab -> bf16 chunk-major tile
// [rk / 8 + rv / 8][32][8] in dst (the layout process_tile_mma reads), each
// code multiplied by its token's scale and rounded to bf16 once.  Lane =
// token; tokens at or past n are written as zeros.
__device__ __forceinline__ void dequant_half(const uint4* slab, int half, int rk, int rv, int n,
                                             uint4* dst, int lane) {
  const int t = half * kFrTile + lane;
  const float* scales = reinterpret_cast<const float*>(slab + (rk + rv) / 16 * kLatPage);
  const bool ok = lane < n;
  const float sk = ok ? scales[2 * t] : 0.f, sv = ok ? scales[2 * t + 1] : 0.f;
  const int nk16 = rk / 16, n16 = (rk + rv) / 16;
  for (int c = 0; c < n16; ++c) {
    const float s = c < nk16 ? sk : sv;
    const uint4 w = ok ? slab[c * kLatPage + t] : make_uint4(0, 0, 0, 0);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      // the four int8 codes of word e4, sign-extended, times the scale
      const int x0 = (int)(ws[e4] << 24) >> 24, x1 = (int)(ws[e4] << 16) >> 24;
      const int x2 = (int)(ws[e4] << 8) >> 24, x3 = (int)ws[e4] >> 24;
      o[2 * e4] = pack_bf16x2((float)x0 * s, (float)x1 * s);
      o[2 * e4 + 1] = pack_bf16x2((float)x2 * s, (float)x3 * s);
    }
    dst[(2 * c) * kFrTile + lane] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[(2 * c + 1) * kFrTile + lane] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  __syncwarp();
}

// The consumer warps' records of one unit (shared memory wrec, kConsumers
// rows of S floats: m[G], l[G], acc [G][rvd]) -> the CTA's record for the
// unit (rec, global memory): M = max m, w = exp2(m - M), l = sum w l,
// acc = sum w acc.  Run by the 32 * kConsumers consumer threads (ltid);
// a warp without a tile of the unit holds m = -inf and weighs 0.
template <int G>
__device__ inline void combine_warp_records(const float* wrec, int S, int rvd, float* rec,
                                            int ltid) {
  const int H = hdr_floats(G);
  for (int x = ltid; x < G * rvd + G; x += 32 * kConsumers) {
    const bool hdr = x >= G * rvd;
    const int g = hdr ? x - G * rvd : x / rvd, j = hdr ? 0 : x - g * rvd;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, wrec[w * S + g]);
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float m = wrec[w * S + g];
      const float wt = m > -INFINITY ? exp2f(m - M) : 0.f;
      const float v = hdr ? wrec[w * S + G + g] : wrec[w * S + H + g * rvd + j];
      sum = fmaf(wt, wt > 0.f ? v : 0.f, sum);
    }
    if (hdr) {
      rec[g] = M;
      rec[G + g] = sum;
    } else {
      rec[H + g * rvd + j] = sum;
    }
  }
}

// ------------------------------------------------------------ split kernel
// kDense: the ring carries full-rank pages (dense baseline) instead of latent
// pages; KS / VB: rank class of the tensor-core tiles (bf16 only).
// 168 registers: ten warps, three on two of the SM's four sub-partitions
// (16K registers each).  More consumer warps hide more of each warp's
// dependent latency; fewer registers spill in the wider rank classes.
// kMode: kModeQ8, the latent pages hold per-token int8 codes and fp32
// scales, and each consumer dequantises a page half by half into its own
// bf16 buffer and runs the bf16 tensor-core tile on it; kModeVA, the pages
// hold key codes and value residual slots (process_tile_va).
template <typename T, int G, bool kDense, int KS, int VB, int kMode = kModePlain>
__global__ void __maxnreg__(168) split_kernel(DecodeArgs a) {
  constexpr int CE = Elem<T>::CE;
  constexpr int NP = CE / 2;
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr bool kTC = std::is_same<T, __nv_bfloat16>::value;
  const SmemPlan sp_ = smem_plan(a.NS, a.stage_bytes, a.B, G, kTC, a.dq_bytes,
                                 kDense ? kHeadDim : a.rw);
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
  volatile int* fail = reinterpret_cast<volatile int*>(smem + sp_.flags);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  pdl_trigger();  // the merge grid may be scheduled; it waits for this grid to finish
  // After a step's append (which also folded the queries) nothing of the
  // cache may be read before that grid is done; after a q-fold the cache was
  // final before it started.
  if (a.wait_first) pdl_wait();
  if (warp == 0) build_prefix(a, start_lat, start_fr);
  if (threadIdx.x == 32) {
    *fail = 0;
    for (int s = 0; s < a.NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      tag[s] = -1;
    }
    mbar_fence_init();
  }
  __syncthreads();

  // The ring carries the latent pages, or the full-rank pages in dense mode.
  constexpr int rsp = kDense ? 1 : 0;
  const int* rstart = rsp == 0 ? start_lat : start_fr;
  const int rtot = rstart[a.B];
  int lo, hi;
  cta_range(c, rtot, a.C, lo, hi);
  const int N = hi - lo;

  if (warp == kProducerWarp) {
    // ---------------- producer: lane l holds the slab address of tile base + l;
    // the next batch's block-table reads are in flight while this batch is
    // issued, kIssue lanes at a time (fetch issues the read, addr consumes it).
    const uint64_t pol = l2_evict_first_policy();
    auto fetch = [&](int kk, int& kvh, int& page) {
      kvh = 0; page = -1;
      if (kk >= N) return;
      int b, i, tiles;
      locate(rstart, a.B, a.H_kv, lo + kk, b, kvh, i, tiles);
      page = rsp == 0 ? __ldg(a.bt_lat + (size_t)b * a.maxp_lat + i)
                      : __ldg(a.bt_fr + (size_t)b * a.maxp_fr + i);
    };
    auto addr = [&](int kk, int kvh, int page, const void*& src, uint32_t& bytes, int& good) {
      src = nullptr; bytes = 0; good = 0;
      if (kk >= N) return;
      if (rsp == 0) {
        good = page >= 0 && page < a.num_pages_lat;
        const size_t slab = (size_t)(good ? page : 0) * a.H_kv + kvh;
        bytes = a.stage_bytes;  // one latent slab (bf16, fp32 or int8 + scales)
        src = static_cast<const uint8_t*>(a.codes) + slab * a.stage_bytes;
      } else {
        good = page >= 0 && page < a.num_pages_fr;
        const size_t slab = (size_t)(good ? page : 0) * a.H_kv + kvh;
        bytes = 2 * kFrTile * kHeadDim * sizeof(T);
        src = static_cast<const T*>(a.fr) + slab * 2 * kFrTile * kHeadDim;
      }
    };
    const void *csrc, *nsrc;
    uint32_t cbytes, nbytes;
    int cgood, ngood;
    int fk, fp;
    fetch(lane, fk, fp);
    addr(lane, fk, fp, csrc, cbytes, cgood);
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < N && ok; base += 32) {
      fetch(base + 32 + lane, fk, fp);
      const int cnt = min(32, N - base);
      for (int j0 = 0; j0 < cnt; j0 += kIssue) {
        int f = 0;
        if (lane >= j0 && lane < min(j0 + kIssue, cnt)) {
          const int k = base + lane, s = k % a.NS, n = k / a.NS;
          if (n > 0 && !mbar_wait_bounded(&empty[s], (n - 1) & 1)) {
            *a.err = kErrTimeout;
            f = 1;
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
        if (__any_sync(0xffffffffu, f) || *fail) {
          ok = false;
          *fail = 1;
          break;
        }
        issued = base + min(j0 + kIssue, cnt);
      }
      addr(base + 32 + lane, fk, fp, nsrc, nbytes, ngood);
      csrc = nsrc; cbytes = nbytes; cgood = ngood;
    }
    // Drain: wait (bounded) for every copy this CTA issued before exiting.
    if (lane == 0)
      for (int s = 0; s < a.NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / a.NS) * a.NS;
        if (!mbar_wait_bounded(&full[s], (last / a.NS) & 1)) *a.err = kErrTimeout;
      }
    return;
  }

  pdl_wait();  // the q-fold results are visible from here on
  const int slot = kTC ? 0 : (warp == kAnchorWarp ? kConsumers : warp - kFirstConsumer);
  float2* pbuf = reinterpret_cast<float2*>(smem + sp_.pbuf) + slot * kLatPage * G;
  float* qv = reinterpret_cast<float*>(smem + sp_.qown) + slot * G * kHeadDim;

  if (warp == kAnchorWarp) {
    // ---------------- anchor warp: this CTA's share of the anchor tiles
    if constexpr (kDense) {
      return;
    } else {
    if (!anchor_mode(a.fr, a.bt_fr)) return;
    const int tot = start_fr[a.B];
    int flo, fhi;
    cta_range(c, tot, a.C, flo, fhi);
    const int rec_stride = hdr_floats(G) + G * kHeadDim;
    int t = flo;
    while (t < fhi) {
      int b, kvh, i0, tiles;
      locate(start_fr, a.B, a.H_kv, t, b, kvh, i0, tiles);
      const int unit = b * a.H_kv + kvh, ustart = t - i0, ce = min(fhi, ustart + tiles);
      const int ntok = space_tokens(a, 1, b);
      fetch_queries_warp<G>(a, 1, b, kvh, qv, lane);
      float m[G], l[G];
      float2 acc[G][NP];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[h][e] = make_float2(0.f, 0.f);
      }
      for (int tt = t; tt < ce; ++tt) {
        const size_t slab = ((size_t)b * a.H_kv + kvh) * a.maxp_fr + (tt - ustart);
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(a.fr) +
                                                          slab * 2 * kFrTile * kHeadDim);
        anchor_tile<T, G>(src, min(kFrTile, ntok - (tt - ustart) * kFrTile), qv, pbuf, m, l,
                          acc, lane);
      }
      write_record<T, G>(a.part_fr + (size_t)(unit + c) * rec_stride, kHeadDim, 32 / (kHeadDim / CE),
                         kHeadDim / CE, m, l, acc, lane);
      t = ce;
    }
    return;
    }
  }

  // ---------------- consumers (bf16 pages on the tensor cores, fp32 on SIMT)
  constexpr bool kTensorTiles = std::is_same<T, __nv_bfloat16>::value;
  const int w = warp - kFirstConsumer;
  float* wrec = reinterpret_cast<float*>(smem + sp_.wrec);
  const int nck = rsp == 0 ? a.rk / CE : kHeadDim / CE;  // (int8 pages: of the bf16 buffer)
  const int ncv = rsp == 0 ? a.rv / CE : kHeadDim / CE;
  const int rvd = rsp == 0 ? a.rw : kHeadDim;
  const int qdim = rsp == 0 ? a.rk : kHeadDim;
  int TS = 1;
  while (TS * 2 * ncv <= 32) TS *= 2;
  float* part = rsp == 0 ? a.part_lat : a.part_fr;
  const int rec_stride = hdr_floats(G) + G * rvd;
  int t = lo;
  while (t < hi) {
    int b, kvh, i0, tiles;
    locate(rstart, a.B, a.H_kv, t, b, kvh, i0, tiles);
    const int unit = b * a.H_kv + kvh, ustart = t - i0, ce = min(hi, ustart + tiles);
    const int ntok = space_tokens(a, rsp, b);
    if constexpr (!kTC) fetch_queries_warp<G>(a, rsp, b, kvh, qv, lane);
    const int k0 = t - lo;
    const int first = t + ((w - k0 % kConsumers) + kConsumers) % kConsumers;
    // Wait (bounded) for tile tt of the ring; nullptr on timeout.
    auto acquire = [&](int tt) -> const uint4* {
      const int k = tt - lo, s = k % a.NS, n = k / a.NS;
      if (!tag_wait_bounded(tag + s, k) || !mbar_wait_bounded(&full[s], n & 1)) {
        *a.err = kErrTimeout;
        *fail = 1;
        return nullptr;
      }
      return reinterpret_cast<const uint4*>(ring + (size_t)s * a.stage_bytes);
    };
    auto release = [&](int tt) {
      if (lane == 0) mbar_arrive(&empty[(tt - lo) % a.NS]);
    };
    // this warp's record: combined below into the CTA's, or written as is
    float* rec = a.combine ? wrec + w * rec_stride
                           : part + ((size_t)(unit + c) * kConsumers + w) * rec_stride;
    if constexpr (kTensorTiles) {
      constexpr int TT = kDense ? kFrTile : kLatPage;
      QFrag<KS> qf;
      load_qfrag<G, KS>((rsp == 0 ? a.qlat : a.qfr) + ((size_t)b * a.H_q + (size_t)kvh * G) * qdim,
                        qdim, lane, qf);
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, acc[2][VB][4];
#pragma unroll
      for (int hl = 0; hl < 2; ++hl)
#pragma unroll
        for (int vb = 0; vb < VB; ++vb)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[hl][vb][i] = 0.f;
      if constexpr (kMode == kModeVA && !kDense) {
        // value-amortised pages: sum p c_k over the key codes and p e over
        // the kept residuals; the merge applies the predictor
        float* pw = reinterpret_cast<float*>(smem + sp_.dq + (size_t)w * a.dq_bytes);
        float acck[2][KS][4], acce[VB][4];
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kb = 0; kb < KS; ++kb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acck[hl][kb][i] = 0.f;
#pragma unroll
        for (int vb = 0; vb < VB; ++vb)
#pragma unroll
          for (int i = 0; i < 4; ++i) acce[vb][i] = 0.f;
        for (int tt = first; tt < ce; tt += kConsumers) {
          const uint4* st = acquire(tt);
          if (!st) break;
          process_tile_va<KS, VB>(st, min(TT, ntok - (tt - ustart) * TT), nck, a.rv / 8, qf, m,
                                  l, acck, acce, pw, lane);
          release(tt);
        }
        write_record_va<G, KS, VB>(rec, a.rk, a.rv, m, l, acck, acce, lane);
      } else if constexpr (kMode == kModeQ8 && !kDense) {
        // int8 pages: each half of 32 tokens is dequantised into this warp's
        // buffer, then run on the tensor cores as a 32-token tile
        uint4* dq = reinterpret_cast<uint4*>(smem + sp_.dq + (size_t)w * a.dq_bytes);
        for (int tt = first; tt < ce; tt += kConsumers) {
          const uint4* st = acquire(tt);
          if (!st) break;
          const int nv = min(TT, ntok - (tt - ustart) * TT);
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const int nh = min(kFrTile, nv - half * kFrTile);
            if (nh <= 0) break;
            dequant_half(st, half, a.rk, a.rv, nh, dq, lane);
            if (half == 1 || nv <= kFrTile) release(tt);
            process_tile_mma<kFrTile, KS, VB>(dq, nh, nck, ncv, qf, m, l, acc, lane);
          }
          if (nv <= 0) release(tt);
        }
      } else {
        for (int tt = first; tt < ce; tt += kConsumers) {
          const uint4* st = acquire(tt);
          if (!st) break;
          process_tile_mma<TT, KS, VB>(st, min(TT, ntok - (tt - ustart) * TT), nck, ncv, qf, m,
                                       l, acc, lane);
          release(tt);
        }
      }
      // This warp's record for (unit, CTA); m = -inf when it had no tile.
      if constexpr (!(kMode == kModeVA && !kDense)) write_record_mma<G, VB>(rec, rvd, m, l, acc, lane);
    } else {
      float m[G], l[G];
      float2 acc[G][NP];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[h][e] = make_float2(0.f, 0.f);
      }
      for (int tt = first; tt < ce; tt += kConsumers) {
        const uint4* st = acquire(tt);
        if (!st) break;
        constexpr int TT = kDense ? kFrTile : kLatPage;
        process_tile<T, G, TT>(st, min(TT, ntok - (tt - ustart) * TT), nck, ncv, TS, qv, qdim,
                               pbuf, m, l, acc, lane);
        release(tt);
      }
      write_record<T, G>(rec, rvd, TS, ncv, m, l, acc, lane);
    }
    if (a.combine) {
      // The CTA's one record for (unit, space).  Every consumer warp passes
      // here once per unit; a failure seen by any of them ends them all.
      if (named_bar_any(kBarRecords, 32 * kConsumers, *fail != 0)) break;
      combine_warp_records<G>(wrec, rec_stride, rvd, part + (size_t)(unit + c) * rec_stride,
                              threadIdx.x - 32 * kFirstConsumer);
      // a warp without tiles in the next unit writes its next record at once
      named_bar(kBarRecords, 32 * kConsumers);
    } else if (*fail) {
      break;
    }
    t = ce;
  }
}

// ------------------------------------------------------------ merge kernel
// Shared-memory plan of the merge kernel (byte offsets from the base).
struct MergePlan {
  int pv, recb, wts, latf, frf, lf, starts, bars, am, uf, total;
};
__host__ __device__ inline int pv_row(int rv) { return rv + 4; }  // padded row of P_v
// rk_va > 0: value-amortised records (key-code sums then residual sums, rw =
// rk_va + rv per head) and the unit's predictor staged beside P_v.
__host__ __device__ inline MergePlan merge_plan(int rv, bool lat, int G, int B, int rk_va = 0) {
  MergePlan p;
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int at = off;
    off += bytes;
    return at;
  };
  p.pv = take(lat ? kHeadDim * pv_row(rv) * 4 : 0, 16);
  p.recb = take(kMergeBuf, 128);
  p.wts = take(kMergeWarps * (kMergeMaxRec + 4) * 4, 16);
  p.latf = take(G * (lat ? rv + rk_va : 0) * 4, 16);
  p.frf = take(G * kHeadDim * 4, 16);
  p.lf = take(G * 4, 16);
  p.starts = take(2 * (B + 1) * 4, 8);
  p.bars = take(8, 8);
  p.am = take(lat ? rk_va * rv * 4 : 0, 16);
  p.uf = take(lat && rk_va ? G * rv * 4 : 0, 16);
  p.total = off;
  return p;
}

// sum over x < n of w[x] * col[x * S] (w 16-byte aligned); a record of
// weight 0 adds nothing even if its words are stale.  Sixteen loads in flight.
__device__ __forceinline__ float weighted_sum(const float* col, int S, const float* w, int n) {
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  int x = 0;
#pragma unroll 2
  for (; x + 4 <= n; x += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(w + x);
    const float ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float c = col[(x + u) * S];
      s[u] = fmaf(ww[u], ww[u] > 0.f ? c : 0.f, s[u]);
    }
  }
  for (; x < n; ++x) {
    const float c = col[x * S];
    s[0] = fmaf(w[x], w[x] > 0.f ? c : 0.f, s[0]);
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// Per unit, over every record (m, l, acc) of both spaces:
//   M_g = max m,  w = exp2(m - M_g),  L_g = sum w l,
//   lat = sum_latent w acc,  fr = sum_full-rank w acc,
//   o = (P_v lat + fr) / L_g   (0 where L_g = 0: a sequence with no tokens).
// A unit's records sit in consecutive slots of each space and arrive in
// shared memory by bulk copies: both spaces at once when they fit (the usual
// case), else space by space in chunks folded into running sums.  Warp w
// owns head g = w % G and the share w / G of the latent and full-rank
// columns; it folds every chunk on its own (warp shuffles, no block barrier),
// so the path after the records land is short.  The product with P_v runs
// once at the end, one thread per output row and several heads, so each
// element of P_v is read from shared memory once per thread.  The sequence
// prefix, the record ranges and P_v are staged before the split grid is
// waited for.
template <typename T, int G>
__global__ void __launch_bounds__(kMergeThreads, 1) merge_kernel(DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int rk_va = a.A ? a.rk : 0;
  const MergePlan mp = merge_plan(a.rv, a.codes != nullptr, G, a.B, rk_va);
  float* pv = reinterpret_cast<float*>(smem + mp.pv);      // [128][r_v + 4]
  float* recb = reinterpret_cast<float*>(smem + mp.recb);  // records of one chunk
  float* latf = reinterpret_cast<float*>(smem + mp.latf);  // [G][r_v]
  float* frf = reinterpret_cast<float*>(smem + mp.frf);    // [G][128]
  float* Lf = reinterpret_cast<float*>(smem + mp.lf);      // [G]
  int* start_lat = reinterpret_cast<int*>(smem + mp.starts);
  int* start_fr = start_lat + (a.B + 1);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + mp.bars);
  pdl_trigger();  // whatever follows may be scheduled now; it waits for this grid itself

  const int unit = blockIdx.x, b = unit / a.H_kv, kvh = unit - b * a.H_kv, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int rv = a.codes ? a.rv : 0, PR = pv_row(a.rv);
  const int rw = a.codes ? a.rw : 0;  // latent record width per head
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (rv) {
    const float4* P = reinterpret_cast<const float4*>(a.P_v + (size_t)b * a.basis_bs +
                                                      (size_t)kvh * kHeadDim * rv);
    const int n4 = rv / 4;
    const uint64_t pol = l2_evict_last_policy();
    for (int x = tid; x < kHeadDim * n4; x += kMergeThreads) {
      const int d = x / n4, j4 = x - d * n4;
      *reinterpret_cast<float4*>(pv + d * PR + 4 * j4) = ldg_f4_hint(P + x, pol);
    }
    if (rk_va) {  // the unit's value predictor A [rk][rv]
      const float4* Ag = reinterpret_cast<const float4*>(a.A + (size_t)unit * rk_va * rv);
      float4* am = reinterpret_cast<float4*>(smem + mp.am);
      for (int x = tid; x < rk_va * rv / 4; x += kMergeThreads) am[x] = __ldg(Ag + x);
    }
  }
  // seq_len was final before the q-fold started (an ordinary launch).
  if (tid < 32) build_prefix(a, start_lat, start_fr);
  __syncthreads();
  const bool anchors = anchor_mode(a.fr, a.bt_fr);
  const int H = hdr_floats(G);
  // records: latent (CTA, warp) pairs, then full-rank (CTA[, warp]) records
  int c0[2] = {0, 0}, ncta[2] = {0, 0}, total[2];
  const int* starts[2] = {start_lat, start_fr};
#pragma unroll
  for (int sp = 0; sp < 2; ++sp) {
    total[sp] = starts[sp][a.B];
    const int tiles = (starts[sp][b + 1] - starts[sp][b]) / a.H_kv;
    if (total[sp] == 0 || tiles == 0) continue;
    const int us = starts[sp][b] + kvh * tiles;
    const int Ce = ctas_for(total[sp], a.C);
    c0[sp] = cta_of(us, total[sp], Ce);
    ncta[sp] = cta_of(us + tiles - 1, total[sp], Ce) - c0[sp] + 1;
  }
  // records per (CTA, unit): the anchor warp writes one; the consumers one
  // (combined) or one per warp
  const int per0 = a.combine ? 1 : kConsumers, per1 = (anchors || a.combine) ? 1 : kConsumers;
  const int S0 = H + G * a.rw, S1 = H + G * kHeadDim;  // floats per record
  const int n0 = ncta[0] * per0, n1 = ncta[1] * per1;
  const float* src0 = a.part_lat + (size_t)(unit + c0[0]) * per0 * S0;
  const float* src1 = a.part_fr + (size_t)(unit + c0[1]) * per1 * S1;
  const bool fused = n0 + n1 <= kMergeMaxRec && (n0 * S0 + n1 * S1) * 4 <= kMergeBuf;

  // this warp: head g, columns [j0, j1) of the latent sums and [d0, d1) of
  // the full-rank sums; lane owns columns j0 + lane + 32 i and d0 + lane + 32 i
  constexpr int kParts = kMergeWarps / G;
  const int g = warp % G, part = warp / G;
  const int jn = (rw + kParts - 1) / kParts, j0 = min(rw, part * jn), j1 = min(rw, j0 + jn);
  constexpr int dn = kHeadDim / kParts, kD = (dn + 31) / 32;
  const int d0 = part * dn;
  float* wts = reinterpret_cast<float*>(smem + mp.wts) + warp * (kMergeMaxRec + 4);
  float M = -INFINITY, L = 0.f, lat[4], fr[kD];
#pragma unroll
  for (int i = 0; i < 4; ++i) lat[i] = 0.f;
#pragma unroll
  for (int i = 0; i < kD; ++i) fr[i] = 0.f;

  pdl_wait();  // every record of the split kernel is visible

  int chunk = 0, sp = 0, q0 = 0;
  bool ok = true;
  while (true) {
    // this chunk: latent records [l0, l0 + nl) and full-rank [f0, f0 + nf)
    int nl = 0, nf = 0, l0 = 0, f0 = 0;
    if (fused) {
      if (chunk > 0 || n0 + n1 == 0) break;
      nl = n0;
      nf = n1;
      if (tid == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)((n0 * S0 + n1 * S1) * 4));
        if (n0) bulk_g2s(recb, src0, (uint32_t)(n0 * S0 * 4), bar);
        if (n1) bulk_g2s(recb + n0 * S0, src1, (uint32_t)(n1 * S1 * 4), bar);
      }
    } else {
      const int n = sp ? n1 : n0;
      if (q0 >= n) {
        if (sp == 1) break;
        sp = 1;
        q0 = 0;
        continue;
      }
      const int S = sp ? S1 : S0;
      const int nq = min(min(kMergeMaxRec, kMergeBuf / (S * 4)), n - q0);
      if (sp) { nf = nq; f0 = q0; } else { nl = nq; l0 = q0; }
      if (tid == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(nq * S * 4));
        bulk_g2s(recb, (sp ? src1 : src0) + (size_t)q0 * S, (uint32_t)(nq * S * 4), bar);
      }
      q0 += nq;
    }
    const bool landed = mbar_wait_bounded(bar, chunk & 1);
    ++chunk;
    if (!__syncthreads_and(landed)) {
      ok = false;
      break;
    }
    const int nq = nl + nf;
    const float* rf = recb + nl * S0;  // full-rank records of this chunk
    // max and weights of head g; a record whose CTA had an empty range was
    // never written and gets weight 0
    auto mval = [&](int x) -> float {
      const bool isf = x >= nl;
      const int q = isf ? f0 + x - nl : l0 + x;
      const int cc = (isf ? c0[1] + q / per1 : c0[0] + q / per0);
      const int tot = isf ? total[1] : total[0];
      const int Ce = ctas_for(tot, a.C);
      const bool v = range_lo(cc, tot, Ce) != range_lo(cc + 1, tot, Ce);
      return v ? (isf ? rf + (x - nl) * S1 : recb + x * S0)[g] : -INFINITY;
    };
    float cm = -INFINITY;
    for (int x = lane; x < nq; x += 32) cm = fmaxf(cm, mval(x));
    const float Mn = fmaxf(M, warp_max(cm));
    float ls = 0.f;
    for (int x = lane; x < nq; x += 32) {
      const float m = mval(x);
      const float w = m > -INFINITY ? exp2f(m - Mn) : 0.f;
      wts[x < nl ? x : x + ((4 - (nl & 3)) & 3)] = w;
      if (w > 0.f) ls = fmaf(w, (x >= nl ? rf + (x - nl) * S1 : recb + x * S0)[G + g], ls);
    }
    ls = warp_sum(ls);
    __syncwarp();
    const float* wts_f = wts + ((nl + 3) & ~3);  // full-rank weights, 16-byte aligned
    const float al = Mn > -INFINITY ? exp2f(M - Mn) : 1.f;
    M = Mn;
    L = fmaf(L, al, ls);
    // weighted sums; records of weight 0 are skipped (their words may be stale)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = j0 + lane + 32 * i;
      if (j < j1) lat[i] = fmaf(lat[i], al, weighted_sum(recb + H + g * a.rw + j, S0, wts, nl));
    }
#pragma unroll
    for (int i = 0; i < kD; ++i) {
      const int d = d0 + lane + 32 * i;
      if (lane + 32 * i < dn)
        fr[i] = fmaf(fr[i], al, weighted_sum(rf + H + g * kHeadDim + d, S1, wts_f, nf));
    }
    __syncthreads();  // the next chunk overwrites recb
  }
  if (!ok) {
    if (tid == 0) {
      *a.err = kErrTimeout;
      mbar_wait_bounded(bar, (chunk - 1) & 1);  // the copy still in flight
    }
    return;
  }
  // hand the sums over to the row-wise product with P_v
  if (warp < kParts * G) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = j0 + lane + 32 * i;
      if (j < j1) latf[g * rw + j] = lat[i];
    }
#pragma unroll
    for (int i = 0; i < kD; ++i)
      if (lane + 32 * i < dn) frf[g * kHeadDim + d0 + lane + 32 * i] = fr[i];
    if (part == 0 && lane == 0) Lf[g] = L;
  }
  __syncthreads();
  // value-amortised: u[g][n] = sum_k A[k][n] keysum[g][k] + ressum[g][n]
  const float* uf = latf;
  if (rk_va && rv) {
    float* u = reinterpret_cast<float*>(smem + mp.uf);
    const float* am = reinterpret_cast<const float*>(smem + mp.am);
    for (int x = tid; x < G * rv; x += kMergeThreads) {
      const int gg = x / rv, n = x - gg * rv;
      float acc = latf[gg * rw + rk_va + n];
      for (int k = 0; k < rk_va; ++k) acc = fmaf(am[k * rv + n], latf[gg * rw + k], acc);
      u[x] = acc;
    }
    __syncthreads();
    uf = u;
  }
  // o[g][d] = (sum_j P_v[d][j] lat[g][j] + fr[g][d]) / L_g: thread -> row d
  // and heads [h0, h0 + kHT)
  constexpr int kHT = (G * kHeadDim + kMergeThreads - 1) / kMergeThreads;
  const int d = tid % kHeadDim, h0 = (tid / kHeadDim) * kHT;
  if (h0 < G) {
    float out[kHT];
#pragma unroll
    for (int h = 0; h < kHT; ++h) out[h] = h0 + h < G ? frf[(h0 + h) * kHeadDim + d] : 0.f;
    const float* prow = pv + d * PR;
    for (int j = 0; j < rv; j += 4) {
      const float4 p4 = *reinterpret_cast<const float4*>(prow + j);
#pragma unroll
      for (int h = 0; h < kHT; ++h) {
        if (h0 + h < G) {
          const float4 l4 = *reinterpret_cast<const float4*>(uf + (h0 + h) * rv + j);
          out[h] = fmaf(p4.x, l4.x, fmaf(p4.y, l4.y, fmaf(p4.z, l4.z, fmaf(p4.w, l4.w, out[h]))));
        }
      }
    }
    T* o = static_cast<T*>(a.o) + ((size_t)b * a.H_q + (size_t)kvh * G) * kHeadDim;
#pragma unroll
    for (int h = 0; h < kHT; ++h) {
      if (h0 + h < G) {
        const float Lg = Lf[h0 + h];
        o[(h0 + h) * kHeadDim + d] = from_f<T>(Lg > 0.f ? out[h] / Lg : 0.f);
      }
    }
  }
}

// ------------------------------------------------------------ host side
struct Plan {
  int C, NS, stage_bytes, dq_bytes, rw, smem, merge_smem;
  size_t off_qlat, off_qfr, off_lat, off_fr, total;
};

// mode: kModePlain, kModeQ8 (int8 codes) or kModeVA (value-amortised slabs).
static int plan_decode(int B, int H_kv, int H_q, int rk, int rv, bool has_lat, bool has_fr,
                       bool anchors, int esize, Plan& p, int mode = kModePlain) {
  int dev = 0;
  DevInfo info;
  const int rc = current_device_info(dev, info);
  if (rc != LRKV_OK) return rc;
  const int sms = info.sms, optin = info.optin;
  const int G = H_q / H_kv;
  // the ring holds latent pages, or dense full-rank pages (no latent space)
  p.stage_bytes = has_lat ? kLatPage * (rk + rv) * esize : 2 * kFrTile * kHeadDim * esize;
  p.dq_bytes = 0;
  int rw = rv;          // latent record width per head
  if (has_lat && mode == kModeQ8) {  // int8 codes + scales; a bf16 half page per consumer
    p.stage_bytes = kLatPage * (rk + rv) + 512;
    p.dq_bytes = kFrTile * (rk + rv) * 2;
  }
  if (has_lat && mode == kModeVA) {  // key codes + residual slots; page weights per consumer
    p.stage_bytes = va_slab_bytes(rk, rv);
    p.dq_bytes = kLatPage * 8 * 4;
    rw = rk + rv;
  }
  p.rw = rw;
  // Leave room for a q-fold CTA beside each split CTA.
  const int budget = optin - 8 * 1024;
  const bool tc = esize == 2;  // bf16: tensor-core consumers
  const int rvd = has_lat ? rw : kHeadDim;  // record width per head of the ring space
  const int fixed = smem_plan(0, p.stage_bytes, B, G, tc, p.dq_bytes, rvd).total + 1024;
  p.NS = std::min(kMaxStages, (budget - fixed) / p.stage_bytes);
  if (p.NS < 2) return LRKV_ERR_UNSUPPORTED;
  p.smem = smem_plan(p.NS, p.stage_bytes, B, G, tc, p.dq_bytes, rvd).total;
  p.C = sms;
  p.merge_smem = merge_plan(rv, has_lat, G, B, mode == kModeVA ? rk : 0).total;
  const int U = B * H_kv;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 256;
  p.off_qlat = off; off = al(off + (size_t)B * H_q * (has_lat ? rk : 0) * 4);
  p.off_qfr = off;  off = al(off + (size_t)B * H_q * (has_fr ? kHeadDim : 0) * 4);
  const size_t slots = (size_t)(U + p.C - 1);
  p.off_lat = off;
  off = al(off + (has_lat ? slots * kConsumers * (hdr_floats(G) + G * rw) * 4 : 0));
  p.off_fr = off;
  off = al(off + (has_fr ? slots * (anchors ? 1 : kConsumers) * (hdr_floats(G) + G * kHeadDim) * 4
                         : 0));
  p.total = off;
  return LRKV_OK;
}

static int mode_of(int dtype) {
  return dtype == LRKV_BF16_Q8 ? kModeQ8 : (dtype == LRKV_BF16_VA ? kModeVA : kModePlain);
}

int decode_plan_check(int B, int H_kv, int H_q, int rk, int rv, bool has_lat, bool has_fr,
                      int dtype) {
  Plan p;
  return plan_decode(B, H_kv, H_q, rk, rv, has_lat, has_fr, has_lat && has_fr,
                     dtype == LRKV_F32 ? 4 : 2, p, mode_of(dtype));
}

size_t decode_workspace_bytes(int B, int H_kv, int H_q, int rk, int rv, bool has_lat,
                              bool has_fr, int dtype) {
  Plan p;
  // anchors: full-rank space present next to a latent one (no block table)
  if (plan_decode(B, H_kv, H_q, rk, rv, has_lat, has_fr, has_lat && has_fr,
                  dtype == LRKV_F32 ? 4 : 2, p, mode_of(dtype)) != LRKV_OK)
    return 0;
  return p.total;
}

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

// The split kernel built for this call: dense or latent ring; for bf16 latent
// pages the smallest rank class that holds (r_k, r_v).
template <typename T, int G>
static const void* split_fn(const DecodeArgs& a) {
  if (!a.codes) return (const void*)split_kernel<T, G, true, 8, 8>;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (a.A) {  // value-amortised slabs
      if (a.rk <= 64 && a.rv <= 32) return (const void*)split_kernel<T, G, false, 4, 2, kModeVA>;
      return (const void*)split_kernel<T, G, false, 8, 8, kModeVA>;
    }
    if (a.dq_bytes) {  // int8 codes
      if (a.rk <= 64 && a.rv <= 32) return (const void*)split_kernel<T, G, false, 4, 2, kModeQ8>;
      return (const void*)split_kernel<T, G, false, 8, 8, kModeQ8>;
    }
    if (a.rk <= 64 && a.rv <= 32) return (const void*)split_kernel<T, G, false, 4, 2>;
  }
  return (const void*)split_kernel<T, G, false, 8, 8>;
}

template <typename T, int G>
static int launch_decode_t(DecodeArgs a, const Plan& p, cudaStream_t st, bool folded) {
  // Keep SMs in the large-shared-memory configuration while the q-fold runs,
  // so the split kernel's CTAs can start beside it without a reconfiguration.
  // (Kernel attributes are set once per device; see prepare_kernel.)
  const void* split = split_fn<T, G>(a);
  int rc = prepare_kernel((const void*)qfold_kernel<T, G>, true);
  if (rc == LRKV_OK) rc = prepare_kernel(split, true);
  if (rc == LRKV_OK) rc = prepare_kernel((const void*)merge_kernel<T, G>, false);
  if (rc != LRKV_OK) return rc;
  if (!folded) {
    qfold_kernel<T, G><<<a.B * a.H_kv * a.fold_split, kFoldThreads, 0, st>>>(a);
    if (cudaGetLastError() != cudaSuccess) return LRKV_ERR_CUDA;
  }
  void* args[] = {&a};
  if (launch_pdl(split, dim3(p.C), dim3(kThreads), p.smem, st, args) != cudaSuccess)
    return LRKV_ERR_CUDA;
  if (launch_pdl((const void*)merge_kernel<T, G>, dim3(a.B * a.H_kv), dim3(kMergeThreads),
                 p.merge_smem, st, args) != cudaSuccess)
    return LRKV_ERR_CUDA;
  return LRKV_OK;
}

template <typename T>
static int launch_decode_g(const DecodeArgs& a, const Plan& p, cudaStream_t st, bool folded) {
  switch (a.G) {
    case 1: return launch_decode_t<T, 1>(a, p, st, folded);
    case 2: return launch_decode_t<T, 2>(a, p, st, folded);
    case 4: return launch_decode_t<T, 4>(a, p, st, folded);
    case 8: return launch_decode_t<T, 8>(a, p, st, folded);
    default: return LRKV_ERR_UNSUPPORTED;
  }
}

// Plan and workspace pointers of a decode call.
static int decode_args(const DecodeLaunch& L, DecodeArgs& a, Plan& p) {
  const bool has_lat = L.codes != nullptr, has_fr = L.fr != nullptr;
  const int es = L.dtype == LRKV_F32 ? 4 : 2;
  int rc = plan_decode(L.B, L.H_kv, L.H_q, L.rk, L.rv, has_lat, has_fr,
                       anchor_mode(L.fr, L.bt_fr), es, p, mode_of(L.dtype));
  if (rc != LRKV_OK) return rc;
  if (L.ws_bytes < p.total) return LRKV_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(L.ws);
  a.B = L.B; a.H_kv = L.H_kv; a.G = L.H_q / L.H_kv; a.H_q = L.H_q;
  a.seq_len = L.seq_len; a.n_sink = L.n_sink; a.W = L.W;
  a.codes = L.codes; a.bt_lat = L.bt_lat; a.maxp_lat = L.maxp_lat;
  a.rk = L.rk; a.rv = L.rv;
  a.fr = L.fr; a.bt_fr = L.bt_fr; a.maxp_fr = L.maxp_fr;
  a.num_pages_lat = L.num_pages_lat; a.num_pages_fr = L.num_pages_fr;
  a.P_v = L.P_v; a.basis_bs = L.basis_bs; a.o = L.o;
  a.q = L.q; a.P_k = L.P_k; a.qscale = L.scale * kLog2e;
  a.err = reinterpret_cast<int*>(ws);
  a.qlat = reinterpret_cast<float*>(ws + p.off_qlat);
  a.qfr = reinterpret_cast<float*>(ws + p.off_qfr);
  a.part_lat = reinterpret_cast<float*>(ws + p.off_lat);
  a.part_fr = reinterpret_cast<float*>(ws + p.off_fr);
  a.C = p.C; a.NS = p.NS; a.stage_bytes = p.stage_bytes; a.dq_bytes = p.dq_bytes;
  a.rw = p.rw;
  a.A = L.dtype == LRKV_BF16_VA ? L.A : nullptr;
  a.wait_first = 0;
  a.fold_split = std::max(kFoldSplit, (L.rk + 31) / 32);
  // Combine the consumer warps' records inside each CTA when a unit spans
  // at least eight CTAs: then the merge would otherwise fold 64 or more
  // records per unit, and its latency chain grows with them (B = 1 at 16K:
  // 20 -> 15 us per call); with fewer CTAs per unit the per-unit barriers
  // cost more than they save.
  a.combine = (long long)L.B * L.H_kv * 8 <= p.C ? 1 : 0;
  return LRKV_OK;
}

int decode_fold_targets(const DecodeLaunch& L, float** qlat, float** qfr, float* qscale) {
  DecodeArgs a;
  Plan p;
  const int rc = decode_args(L, a, p);
  if (rc != LRKV_OK) return rc;
  *qlat = a.qlat;
  *qfr = L.fr ? a.qfr : nullptr;
  *qscale = a.qscale;
  return LRKV_OK;
}

int decode_launch(const DecodeLaunch& L, cudaStream_t st, bool folded) {
  DecodeArgs a;
  Plan p;
  const int rc = decode_args(L, a, p);
  if (rc != LRKV_OK) return rc;
  a.wait_first = folded ? 1 : 0;
  if (L.dtype == LRKV_F32) return launch_decode_g<float>(a, p, st, folded);
  return launch_decode_g<__nv_bfloat16>(a, p, st, folded);
}

}  // namespace lrkv
