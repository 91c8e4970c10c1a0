// Append + compress: new tokens enter the sink / window ring, and every
// token that becomes latent is projected to codes c = P^T x and written into
// its page (Half the Memory, section 04: store the small r-dim codes; OjaKV
// article: first and most recent tokens kept full-rank as anchors).
//
// For a sequence going from L0 to L1 = L0 + n tokens, with latent counts
// lat(L0) and lat(L1), the tokens n_sink + [lat(L0), lat(L1)) become latent:
// those below L0 are read from the window ring (evictions), the others come
// straight from the input.  Ring reads happen before the window writes in
// the same CTA, so a slot is never overwritten before it is compressed.
//
// Launch order per call: bulk_compress (input tokens that go straight to the
// latent pages, only for large n) then append_kernel (evictions, small-n
// input tokens, sink and window writes, and the seq_len advance).  seq_len
// is advanced by the last CTA of each sequence to finish (a per-sequence
// completion counter, reset to zero by that CTA).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "compress.cuh"
#include "internal.h"

namespace lrkv {

constexpr int kSmallN = 16;       // input tokens handled by append_kernel
constexpr int kBulkRows = 64;     // tokens per bulk_compress CTA

constexpr int kRowBatch = 16;  // token rows projected per pass
// Dynamic shared memory of append_kernel: the unit's basis [128][r_k + r_v]
// fp32, rows [kRowBatch][k, v][128] fp32, partial sums [256], and a page per row.
// (+ one row of codes [256] and two scales for int8 codes, a value residual
// [128] and its slot for value-amortised slabs, and the query rows [8][128]
// of a decode step's fold)
inline size_t append_smem_bytes(int rk, int rv) {
  return ((size_t)kHeadDim * (rk + rv) + (size_t)kRowBatch * 2 * kHeadDim + 256 + kRowBatch +
          256 + 4 + kHeadDim + 4 + 8 * kHeadDim) * 4;
}

// One CTA per (KV head, sequence).  Latency matters here (a decode step
// appends one token), so the loads that do not depend on each other are in
// flight together: seq_len with the unit's basis, then the rows to project
// with their block-table entries.  kCluster: the CTAs of one sequence form a
// cluster; each arrives on the cluster barrier once it has read seq_len, and
// rank 0 waits on it before advancing seq_len, so no CTA can read the new
// value.  Without clusters (H_kv > 8) the last CTA to finish, found with a
// per-sequence counter, advances seq_len.
template <typename T, bool kCluster>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a, int do_input_latent) {
  constexpr int CE = Elem<T>::CE, NC = kHeadDim / CE;
  extern __shared__ __align__(16) float sm[];
  const int NJ = a.rk + a.rv;
  float* Ps = sm;                                                      // [128][NJ]
  float* xs = Ps + kHeadDim * NJ;                                      // [row][k, v][128]
  float* red = xs + kRowBatch * 2 * kHeadDim;                          // [seg][NJ]
  int* pg = reinterpret_cast<int*>(red + 256);                         // [row]
  float* crow = red + 256 + kRowBatch;                                 // [NJ] one row's codes
  float* qscale = crow + 256;                                          // [2] its scales
  float* ev = qscale + 4;                                              // [rv] value residual
  int* vslot = reinterpret_cast<int*>(ev + kHeadDim);                  // its slot
  float* qsm = reinterpret_cast<float*>(vslot + 4);                    // [G][128] fold input
  const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;

  // Launched with programmatic dependent launch: wait for the previous grid
  // before reading anything (only the launch latency is hidden).  The next
  // grid may be scheduled from here on; it waits for this one to finish
  // before it reads what this one writes.
  pdl_wait();
  pdl_trigger();
  // 0. a decode step's query rows (G <= 8 heads, four values per thread),
  // in flight together with the loads below
  const int FG = a.fq ? a.fH_q / a.H_kv : 0;
  const size_t fh0 = ((size_t)b * a.fH_q + (size_t)kvh * FG);
  float fqv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int x = tid + e * (int)blockDim.x;
    fqv[e] = x < FG * kHeadDim ? to_f<T>(static_cast<const T*>(a.fq)[fh0 * kHeadDim + x]) : 0.f;
  }
  // 1. seq_len, and the basis into shared memory ([i][o]: P_k columns then P_v),
  // sixteen 16-byte loads in flight per thread (one round at r_k + r_v <= 128)
  const int L0 = __ldcg(a.seq_len + b);
  {
    const float* Pk = a.P_k + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rk;
    const float* Pv = a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rv;
    const int n4 = NJ / 4, total4 = kHeadDim * n4;
    const uint64_t pol = l2_evict_last_policy();
    constexpr int kB = 16;
    for (int x0 = tid; x0 < total4; x0 += kB * (int)blockDim.x) {
      float4 v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int x = x0 + u * (int)blockDim.x;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x < total4) {
          const int i = x / n4, o = 4 * (x - i * n4);
          v[u] = ldg_f4_hint(reinterpret_cast<const float4*>(o < a.rk ? Pk + i * a.rk + o
                                                               : Pv + i * a.rv + o - a.rk),
                             pol);
        }
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int x = x0 + u * (int)blockDim.x;
        if (x < total4) reinterpret_cast<float4*>(Ps)[x] = v[u];
      }
    }
  }
  // This CTA has read seq_len: the cluster's rank 0 may advance it at the end.
  // The arrive (release) comes after the basis loads, which are in flight
  // together with the seq_len load, so it costs no round trip of its own.
  if constexpr (kCluster) cluster_arrive();
  // 1b. a decode step's query fold for unit (b, kvh): q~[g][j] =
  // fqscale sum_i P_k[i][j] q[g][i] from the staged basis (thread -> output
  // (g, j), four partial sums); the scaled rows for the anchors
  if (FG) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int x = tid + e * (int)blockDim.x;
      if (x < FG * kHeadDim) {
        qsm[x] = fqv[e];
        if (a.fqfr) a.fqfr[fh0 * kHeadDim + x] = fqv[e] * a.fqscale;
      }
    }
    __syncthreads();
    for (int x = tid; x < FG * a.rk; x += blockDim.x) {
      const int g = x / a.rk, j = x - g * a.rk;
      const float* qg = qsm + g * kHeadDim;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int i = 0; i < kHeadDim; i += 4)
#pragma unroll
        for (int u = 0; u < 4; ++u) s4[u] = fmaf(Ps[(i + u) * NJ + j], qg[i + u], s4[u]);
      a.fqlat[fh0 * a.rk + x] = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * a.fqscale;
    }
  }
  const int L1 = L0 + appended(a.n_new, a.n, b);
  const Split s0 = split_tokens(L0, a.n_sink, a.W), s1 = split_tokens(L1, a.n_sink, a.W);
  const T* kin = static_cast<const T*>(a.k) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* vin = static_cast<const T*>(a.v) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* anc = static_cast<const T*>(a.anchors);

  // Sink and window writes (step 3): token t of the input goes to slot
  // slot_of(q) for q < wtotal.  The first 16-byte chunk of each thread is
  // loaded now, together with the rows below, and stored after them.
  const int w_lo = max(L0, max(a.n_sink, L1 - a.W));
  const int n_sink_new = a.n_sink + a.W > 0 ? max(0, min(a.n_sink, L1) - L0) : 0;
  const int n_win_new = a.n_sink + a.W > 0 ? max(0, L1 - w_lo) : 0;
  const int wtotal = (n_sink_new + n_win_new) * 2 * NC;
  auto wchunk = [&](int x, int& slot, int& isv, int& ch) -> const uint4* {
    const int q = x / (2 * NC), rem = x - q * 2 * NC;
    isv = rem / NC;
    ch = rem - isv * NC;
    int t;
    if (q < n_sink_new) { t = L0 + q; slot = t; }
    else { t = w_lo + (q - n_sink_new); slot = a.n_sink + (t - a.n_sink) % a.W; }
    return reinterpret_cast<const uint4*>((isv ? vin : kin) + (size_t)(t - L0) * kHeadDim + ch * CE);
  };
  uint4 wfirst = make_uint4(0, 0, 0, 0);
  if (tid < wtotal) {
    int slot, isv, ch;
    wfirst = __ldcg(wchunk(tid, slot, isv, ch));
  }

  // 2. rows that become latent: evictions from the ring (token < L0, oldest
  // first), then input tokens that go straight to latent (small n only)
  const int ev_lo = a.n_sink + s0.lat, ev_hi = min(L0, a.n_sink + s1.lat);
  const int in_lo = max(L0, a.n_sink + s0.lat), in_hi = a.n_sink + s1.lat;
  const int n_ev = max(0, ev_hi - ev_lo), n_in = do_input_latent ? max(0, in_hi - in_lo) : 0;
  const int nrows = n_ev + n_in;
  auto token_of = [&](int r) { return r < n_ev ? ev_lo + r : in_lo + (r - n_ev); };
  for (int r0 = 0; r0 < nrows; r0 += kRowBatch) {
    const int nr = min(kRowBatch, nrows - r0);
    for (int x = tid; x < nr * 2 * NC; x += blockDim.x) {
      const int rr = x / (2 * NC), rem = x - rr * 2 * NC, isv = rem / NC, ch = rem - isv * NC;
      const int r = r0 + rr, t = token_of(r);
      const T* src;
      if (r < n_ev) {
        const int slot = a.n_sink + (t - a.n_sink) % a.W;
        src = anc + anchor_off<T>(a, b, kvh, slot, ch * CE, isv);
      } else {
        src = (isv ? vin : kin) + (size_t)(t - L0) * kHeadDim + ch * CE;
      }
      unpack_chunk<T>(__ldcg(reinterpret_cast<const uint4*>(src)),
                      xs + (rr * 2 + isv) * kHeadDim + ch * CE);
    }
    if (tid < nr) pg[tid] = latent_page(a, b, token_of(r0 + tid) - a.n_sink);
    __syncthreads();
    // c = P^T x, one row at a time: thread (seg, o) sums the dims of segment
    // seg for code column o (nseg a power of two with nseg * NJ <= 256)
    T* codes = static_cast<T*>(a.codes);
    int nseg = 1;
    while (nseg * 2 * NJ <= (int)blockDim.x && nseg < 8) nseg *= 2;
    const int span = kHeadDim / nseg;
    for (int rr = 0; rr < nr; ++rr) {
      if (tid < nseg * NJ) {
        const int seg = tid / NJ, o = tid - seg * NJ, isv = o < a.rk ? 0 : 1;
        const float* x = xs + (rr * 2 + isv) * kHeadDim + seg * span;
        const float* P = Ps + seg * span * NJ + o;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int i = 0; i < span; i += 4)
#pragma unroll
          for (int u = 0; u < 4; ++u) s4[u] = fmaf(P[(i + u) * NJ], x[i + u], s4[u]);
        red[seg * NJ + o] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      }
      __syncthreads();
      if (a.q8) {
        // per-token int8: the row's codes, then one scale per side
        // (max |c| / 127), then the codes under it
        if (tid < NJ) {
          float c = 0.f;
          for (int seg = 0; seg < nseg; ++seg) c += red[seg * NJ + tid];
          crow[tid] = c;
        }
        __syncthreads();
        if (tid < 64) {
          const int isv = tid >> 5, lo_c = isv ? a.rk : 0, hi_c = isv ? NJ : a.rk;
          float m = 0.f;
          for (int o = lo_c + (tid & 31); o < hi_c; o += 32) m = fmaxf(m, fabsf(crow[o]));
          m = warp_max(m);
          if ((tid & 31) == 0) qscale[isv] = __fdiv_rn(m, 127.f);
        }
        __syncthreads();
        if (tid < NJ && pg[rr] >= 0) {
          const int isv = tid < a.rk ? 0 : 1, jj = isv ? tid - a.rk : tid;
          const int j = token_of(r0 + rr) - a.n_sink;
          uint8_t* cb = static_cast<uint8_t*>(a.codes);
          cb[q8_code_off(a, pg[rr], kvh, j, jj, isv)] =
              static_cast<uint8_t>(static_cast<int8_t>(q8_code(crow[tid], qscale[isv])));
          if (jj == 0)
            *reinterpret_cast<float*>(cb + q8_scale_off(a, pg[rr], kvh, j, isv)) = qscale[isv];
        }
      } else if (a.va) {
        // value-amortised slab: the key code is stored; the value residual
        // against the fitted predictor, e = c_v - A^T c_k, enters the page's
        // slots when it is among the page's LRKV_VA_KEEP largest so far
        const int j = token_of(r0 + rr) - a.n_sink;
        if (tid < NJ) {
          float c = 0.f;
          for (int seg = 0; seg < nseg; ++seg) c += red[seg * NJ + tid];
          crow[tid] = c;
          if (tid < a.rk && pg[rr] >= 0) codes[code_off_in<T>(a, pg[rr], kvh, j, tid, 0)] = from_f<T>(c);
        }
        if (a.A && pg[rr] >= 0) {
          __syncthreads();
          const float* Am = a.A + ((size_t)b * a.H_kv + kvh) * a.rk * a.rv;
          if (tid < a.rv) {
            float pr = 0.f;
            for (int k = 0; k < a.rk; ++k) pr = fmaf(__ldg(Am + (size_t)k * a.rv + tid), crow[k], pr);
            ev[tid] = crow[a.rk + tid] - pr;
          }
          __syncthreads();
          uint8_t* slab = static_cast<uint8_t*>(a.codes) +
                          ((size_t)pg[rr] * a.H_kv + kvh) * va_slab_bytes(a.rk, a.rv);
          int* sidx = reinterpret_cast<int*>(slab + (size_t)kLatPage * a.rk * 2 + kVaKeep * a.rv * 2);
          float* snrm = reinterpret_cast<float*>(sidx + kVaKeep);
          if (tid < 32) {
            float ss = 0.f;
            for (int n = tid; n < a.rv; n += 32) ss = fmaf(ev[n], ev[n], ss);
            ss = warp_sum(ss);
            if (tid == 0) {
              const int row = j % kLatPage;
              if (row == 0)  // a fresh page: no slot used yet
                for (int q = 0; q < kVaKeep; ++q) { sidx[q] = -1; snrm[q] = -1.f; }
              int best = -1;
              for (int q = 0; q < kVaKeep && best < 0; ++q)
                if (sidx[q] < 0) best = q;
              if (best < 0) {
                // the smallest kept norm (ties: the later row) gives way to a
                // strictly larger one, so the earlier token wins ties
                best = 0;
                for (int q = 1; q < kVaKeep; ++q)
                  if (snrm[q] < snrm[best] || (snrm[q] == snrm[best] && sidx[q] > sidx[best]))
                    best = q;
                if (!(ss > snrm[best])) best = -1;
              }
              if (best >= 0) {
                sidx[best] = row;
                snrm[best] = ss;
              }
              *vslot = best;
            }
          }
          __syncthreads();
          const int sl = *vslot;
          if (sl >= 0 && tid < a.rv) {
            __nv_bfloat16* res = reinterpret_cast<__nv_bfloat16*>(slab + (size_t)kLatPage * a.rk * 2);
            res[((tid >> 3) * kVaKeep + sl) * 8 + (tid & 7)] = __float2bfloat16_rn(ev[tid]);
          }
        }
      } else if (tid < NJ && pg[rr] >= 0) {
        float c = 0.f;
        for (int seg = 0; seg < nseg; ++seg) c += red[seg * NJ + tid];
        const int isv = tid < a.rk ? 0 : 1, jj = isv ? tid - a.rk : tid;
        const int j = token_of(r0 + rr) - a.n_sink;
        codes[code_off_in<T>(a, pg[rr], kvh, j, jj, isv)] = from_f<T>(c);
      }
      __syncthreads();  // red is reused by the next row
    }
    // (rows and pages are reused by the next batch; ring slots were read
    // before the window writes below)
  }

  // 3. sink and window writes (full-rank, verbatim), 16-byte chunks; the
  // ring slots they overwrite were read in step 2
  {
    T* ancw = static_cast<T*>(a.anchors);
    for (int x = tid; x < wtotal; x += blockDim.x) {
      int slot, isv, ch;
      const uint4* src = wchunk(x, slot, isv, ch);
      const uint4 u = x == tid ? wfirst : __ldcg(src);
      *reinterpret_cast<uint4*>(ancw + anchor_off<T>(a, b, kvh, slot, ch * CE, isv)) = u;
    }
  }

  // 4. advance seq_len
  if constexpr (kCluster) {
    cluster_wait();
    if (cluster_rank() == 0 && tid == 0) a.seq_len[b] = L1;
  } else {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const int old = atomicAdd(&a.counter[b], 1);
      if (old == a.H_kv - 1) {
        a.seq_len[b] = L1;
        a.counter[b] = 0;
        __threadfence();
      }
    }
  }
}

// Input tokens that become latent without passing through the window, in
// tiles of kBulkRows tokens per (tile, kv head, sequence).
template <typename T>
__global__ void __launch_bounds__(256) bulk_compress_kernel(AppendArgs a) {
  __shared__ float xs[kBulkRows][kHeadDim + 1];
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int L0 = a.seq_len[b], L1 = L0 + appended(a.n_new, a.n, b);
  const Split s0 = split_tokens(L0, a.n_sink, a.W), s1 = split_tokens(L1, a.n_sink, a.W);
  const int in_lo = max(L0, a.n_sink + s0.lat) - L0, in_hi = a.n_sink + s1.lat - L0;
  const int r0 = in_lo + blockIdx.x * kBulkRows;
  const int rows = min(kBulkRows, in_hi - r0);
  if (rows <= 0) return;
  for (int pass = 0; pass < 2; ++pass) {
    const T* src = static_cast<const T*>(pass == 0 ? a.k : a.v) + (size_t)b * a.seq_stride +
                   (size_t)kvh * a.head_stride;
    for (int x = threadIdx.x; x < rows * kHeadDim; x += blockDim.x) {
      const int rr = x / kHeadDim, d = x - rr * kHeadDim;
      xs[rr][d] = to_f<T>(src[(size_t)(r0 + rr) * kHeadDim + d]);
    }
    __syncthreads();
    const int r = pass == 0 ? a.rk : a.rv;
    const float* P = (pass == 0 ? a.P_k : a.P_v) + (size_t)b * a.basis_bs +
                     (size_t)kvh * kHeadDim * r;
    T* dst = static_cast<T*>(a.codes);
    for (int o = threadIdx.x; o < rows * r; o += blockDim.x) {
      const int rr = o / r, jj = o - rr * r;
      float s = 0.f;
#pragma unroll 8
      for (int i = 0; i < kHeadDim; ++i) s = fmaf(P[(size_t)i * r + jj], xs[rr][i], s);
      const int j = L0 + r0 + rr - a.n_sink;  // latent index
      long long off = code_off<T>(a, b, kvh, j, jj, pass);
      if (off >= 0) dst[off] = from_f<T>(s);
    }
    __syncthreads();
  }
}

// ---- bf16 prefill compress on the tensor cores
// c = x P for the tokens that go straight to latent pages.  Persistent: one
// CTA per SM; the tiles of TT tokens of every (sequence, KV head) unit are
// laid end to end and each CTA takes an equal contiguous range, so ragged
// prompts balance.  Per tile each warp projects 16 tokens (m16) x the code
// columns (n8 blocks) x 128 dims (eight k16 steps), with P split as hi + lo
// bf16 so the products keep about 16 mantissa bits and accumulate in fp32.
// Token rows are staged by cp.async into padded shared-memory rows (two
// stages); P^T hi/lo sits in padded rows too, rebuilt when the range enters
// a new unit, so ldmatrix reads both operands without bank conflicts.
constexpr int kPadRow = kHeadDim + 8;  // bf16 elements per staged row

// Shared memory of bulk_compress_mma for tiles of TT tokens and B sequences.
inline size_t bulk_mma_smem_bytes(int rk, int rv, int TT, int B) {
  return ((size_t)2 * (round16(rk) + round16(rv)) + (size_t)2 * 2 * TT) * kPadRow * 2 +
         (size_t)4 * (B + 1) * 4;
}

template <int TT>
__global__ void __launch_bounds__(TT * 2) bulk_compress_mma(AppendArgs a) {
  using bf16 = __nv_bfloat16;
  constexpr int kThreadsB = TT * 2;  // TT / 16 warps
  extern __shared__ __align__(16) bf16 smb[];
  const int RK = round16(a.rk), RV = round16(a.rv), NR = RK + RV;
  bf16* PT = smb;                        // [hi, lo][NR][kPadRow]: rows K codes then V codes
  bf16* X = smb + 2 * NR * kPadRow;      // [stage][k, v][TT][kPadRow]
  int* start = reinterpret_cast<int*>(X + 2 * 2 * TT * kPadRow);  // [B + 1] tile prefix
  int* sL0 = start + (a.B + 1);                                    // [B] seq_len before
  int* srlo = sL0 + (a.B + 1);                                     // [B] row range
  int* srhi = srlo + (a.B + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  // tile prefix over sequences (tiles per unit = ceil(rows / TT)), one warp
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
      own += (rh - rl + TT - 1) / TT * a.H_kv;
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
      e += (srhi[b] - srlo[b] + TT - 1) / TT * a.H_kv;
    }
    if (lane == 31) start[a.B] = incl;
  }
  __syncthreads();
  const int total = start[a.B];
  const int lo = bulk_range_lo(blockIdx.x, total, gridDim.x);
  const int hi = bulk_range_lo(blockIdx.x + 1, total, gridDim.x);
  if (lo >= hi) return;

  // tile index -> (sequence, KV head, tile within the unit)
  auto locate = [&](int k, int& b, int& kvh, int& i, int& tiles) {
    int l = 0, h = a.B;
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (start[mid] <= k) l = mid; else h = mid;
    }
    b = l;
    tiles = (start[b + 1] - start[b]) / a.H_kv;
    const int r = k - start[b];
    kvh = r / tiles;
    i = r - kvh * tiles;
  };
  auto stage = [&](int k, int st) {
    int b, kvh, i, tiles;
    locate(k, b, kvh, i, tiles);
    const int rlo = srlo[b], rhi = srhi[b];
    const bf16* kin = static_cast<const bf16*>(a.k) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
    const bf16* vin = static_cast<const bf16*>(a.v) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
    const int t0 = rlo + i * TT;
    for (int x = tid; x < 2 * TT * 16; x += kThreadsB) {
      const int isv = x / (TT * 16), rem = x - isv * TT * 16;
      const int row = rem >> 4, ch = rem & 15;
      const int r = t0 + row;
      const bool ok = r < rhi;  // rows past the range are zero-filled
      const bf16* src = (isv ? vin : kin) + (size_t)(ok ? r : rlo) * kHeadDim + ch * 8;
      cp_async16(X + ((st * 2 + isv) * TT + row) * kPadRow + ch * 8, src, ok ? 16u : 0u);
    }
    cp_async_commit();
  };
  // P^T as hi + lo bf16 for unit (b, kvh); rows past r_k / r_v are zero.
  // Consecutive threads take consecutive dims i, so the transposed stores hit
  // consecutive addresses (no bank conflicts).
  auto load_basis = [&](int b, int kvh) {
    const float* Pk = a.P_k + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rk;
    const float* Pv = a.P_v + (size_t)b * a.basis_bs + (size_t)kvh * kHeadDim * a.rv;
    const int n4 = NR / 4;
#pragma unroll 8
    for (int x = tid; x < kHeadDim * n4; x += kThreadsB) {
      const int i = x & (kHeadDim - 1), o = 4 * (x / kHeadDim);
      float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
      if (o < RK) {
        if (o < a.rk) p = __ldg(reinterpret_cast<const float4*>(Pk + (size_t)i * a.rk + o));
      } else if (o - RK < a.rv) {
        p = __ldg(reinterpret_cast<const float4*>(Pv + (size_t)i * a.rv + (o - RK)));
      }
      const float pv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bf16 h = __float2bfloat16_rn(pv[u]);
        PT[(o + u) * kPadRow + i] = h;
        PT[(NR + o + u) * kPadRow + i] = __float2bfloat16_rn(pv[u] - __bfloat162float(h));
      }
    }
  };

  bf16* codes = static_cast<bf16*>(a.codes);
  int cur_unit = -1;
  stage(lo, 0);
  for (int k = lo; k < hi; ++k) {
    const int st = (k - lo) & 1;
    int b, kvh, i, tiles;
    locate(k, b, kvh, i, tiles);
    const int L0 = sL0[b], rlo = srlo[b], rhi = srhi[b];
    const int unit = b * a.H_kv + kvh;
    if (unit != cur_unit) {  // every warp is past the previous tile (barrier at its end)
      load_basis(b, kvh);
      cur_unit = unit;
    }
    if (k + 1 < hi) {
      stage(k + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // tile k and the basis are in place
    const int tok0 = rlo + i * TT + 16 * warp;  // first input row of this warp
    for (int isv = 0; isv < 2; ++isv) {
      const int r = isv ? a.rv : a.rk, nb = r / 8, RB = isv ? RK : 0;
      const bf16* xt = X + ((st * 2 + isv) * TT + 16 * warp) * kPadRow;
      uint32_t af[8][4];
#pragma unroll
      for (int s = 0; s < 8; ++s)
        ldsm_x4(smem_u32(xt + (lane & 15) * kPadRow + 16 * s + (lane >> 4) * 8), af[s]);
      // pages of the two token rows this lane stores (g and g + 8)
      int jrow[2], prow[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int rin = tok0 + g + 8 * h2;
        jrow[h2] = L0 + rin - a.n_sink;
        prow[h2] = rin < rhi ? latent_page(a, b, jrow[h2]) : -1;
      }
      for (int ng = 0; ng < nb; ng += 8) {
        float acc[8][4];
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][e] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            if (ng + 2 * p < nb) {
              const int o = RB + 8 * (ng + 2 * p) + (lane & 7) + ((lane >> 4) << 3);
              const int koff = 16 * s + ((lane >> 3) & 1) * 8;
              uint32_t bh[4], bl[4];
              ldsm_x4(smem_u32(PT + o * kPadRow + koff), bh);
              ldsm_x4(smem_u32(PT + (NR + o) * kPadRow + koff), bl);
              mma_bf16_16816(acc[2 * p], af[s], bh[0], bh[1]);
              mma_bf16_16816(acc[2 * p + 1], af[s], bh[2], bh[3]);
              mma_bf16_16816(acc[2 * p], af[s], bl[0], bl[1]);
              mma_bf16_16816(acc[2 * p + 1], af[s], bl[2], bl[3]);
            }
          }
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          if (prow[h2] < 0) continue;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (ng + q < nb) {
              const long long off =
                  code_off_in<bf16>(a, prow[h2], kvh, jrow[h2], 8 * (ng + q) + 2 * t, isv);
              *reinterpret_cast<uint32_t*>(codes + off) =
                  pack_bf16x2(acc[q][2 * h2], acc[q][2 * h2 + 1]);
            }
          }
        }
      }
    }
    __syncthreads();  // stage st is refilled, and the basis may be rebuilt, next iteration
  }
}

// Input tokens that go straight to the latent pages (only for large n).
// bf16: the tensor-memory kernel, or the warp-MMA kernel where the former's
// shared memory does not fit; fp32: the SIMT kernel.
template <typename T>
static int bulk_launch(const AppendArgs& a, cudaStream_t st) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    int dev = 0;
    DevInfo info;
    int rc = current_device_info(dev, info);
    if (rc != LRKV_OK) return rc;
    const int sms = info.sms, optin = info.optin;
    rc = bulk_compress_tc_launch(a, sms, optin, st);
    if (rc != LRKV_ERR_UNSUPPORTED || a.q8 || a.va) return rc;
    // persistent: one CTA per SM; 128-token tiles (8 warps) when they fit
    const bool big = bulk_mma_smem_bytes(a.rk, a.rv, 128, a.B) <= (size_t)optin;
    const size_t smem = bulk_mma_smem_bytes(a.rk, a.rv, big ? 128 : 64, a.B);
    if (smem > (size_t)optin) return LRKV_ERR_UNSUPPORTED;
    const void* fn = big ? (const void*)bulk_compress_mma<128> : (const void*)bulk_compress_mma<64>;
    rc = prepare_kernel(fn, false);
    if (rc != LRKV_OK) return rc;
    if (big)
      bulk_compress_mma<128><<<sms, 256, smem, st>>>(a);
    else
      bulk_compress_mma<64><<<sms, 128, smem, st>>>(a);
  } else {
    dim3 g((a.n + kBulkRows - 1) / kBulkRows, a.H_kv, a.B);
    bulk_compress_kernel<T><<<g, 256, 0, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

template <typename T>
static int compress_t(const AppendArgs& a, cudaStream_t st) {
  const bool small = a.n <= kSmallN;
  if (!small) {
    const int rc = bulk_launch<T>(a, st);
    if (rc != LRKV_OK) return rc;
  }
  const size_t smem = append_smem_bytes(a.rk, a.rv);
  const bool cluster = a.H_kv <= 8;
  const void* fn = cluster ? (const void*)append_kernel<T, true> : (const void*)append_kernel<T, false>;
  const int prc = prepare_kernel(fn, false);
  if (prc != LRKV_OK) return prc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.H_kv, a.B);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = a.H_kv;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster ? 2 : 1;
  int small_in = small ? 1 : 0;
  void* args[] = {(void*)&a, (void*)&small_in};
  if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return LRKV_ERR_CUDA;
  return LRKV_OK;
}

int compress_launch(const lrkv_cache& c, const void* k, const void* v, int n, const int* n_new,
                    long long seq_stride, long long head_stride, const float* P_k,
                    const float* P_v, long long basis_bs, cudaStream_t st, const float* A,
                    const StepFold* fold) {
  AppendArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.rk = c.rank_k; a.rv = c.rank_v;
  a.n_sink = c.n_sink; a.W = c.window; a.maxp = c.max_pages_per_seq; a.num_pages = c.num_pages;
  a.n = n; a.anchor_tiles = (c.n_sink + c.window + kFrTile - 1) / kFrTile;
  a.q8 = c.dtype == LRKV_BF16_Q8 ? 1 : 0;
  a.va = c.dtype == LRKV_BF16_VA ? 1 : 0;
  a.A = A;
  a.codes = c.codes; a.anchors = c.anchors;
  a.bt = c.block_table; a.seq_len = c.seq_len; a.counter = c.append_counter; a.n_new = n_new;
  a.k = k; a.v = v; a.seq_stride = seq_stride; a.head_stride = head_stride;
  a.P_k = P_k; a.P_v = P_v; a.basis_bs = basis_bs;
  a.fq = fold ? fold->q : nullptr;
  a.fH_q = fold ? fold->H_q : 0;
  a.fqscale = fold ? fold->qscale : 0.f;
  a.fqlat = fold ? fold->qlat : nullptr;
  a.fqfr = fold ? fold->qfr : nullptr;
  return c.dtype == LRKV_F32 ? compress_t<float>(a, st) : compress_t<__nv_bfloat16>(a, st);
}

// ------------------------------------------------------------ dense baseline
struct DenseAppendArgs {
  int B, H_kv, maxp, num_pages, n;
  void* kvp;
  const int* bt;
  int* seq_len;
  int* counter;
  const int* n_new;
  const void *k, *v;
  long long seq_stride, head_stride;
};

template <typename T>
__global__ void __launch_bounds__(256) dense_append_kernel(DenseAppendArgs a) {
  constexpr int CE = Elem<T>::CE;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int L0 = a.seq_len[b], nb = appended(a.n_new, a.n, b);
  const T* kin = static_cast<const T*>(a.k) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  const T* vin = static_cast<const T*>(a.v) + (size_t)b * a.seq_stride + (size_t)kvh * a.head_stride;
  T* kvp = static_cast<T*>(a.kvp);
  for (int x = threadIdx.x; x < nb * kHeadDim; x += blockDim.x) {
    const int q = x / kHeadDim, d = x - q * kHeadDim;
    const int t = L0 + q, pi = t / kFrTile;
    if (pi >= a.maxp) continue;
    const int page = a.bt[(size_t)b * a.maxp + pi];
    if (page < 0 || page >= a.num_pages) continue;
    const size_t slab = ((size_t)page * a.H_kv + kvh) * (2 * kHeadDim / CE);
    const size_t row = (size_t)(t % kFrTile) * CE + d % CE;
    kvp[(slab + d / CE) * kFrTile * CE + row] = kin[(size_t)q * kHeadDim + d];
    kvp[(slab + kHeadDim / CE + d / CE) * kFrTile * CE + row] = vin[(size_t)q * kHeadDim + d];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(&a.counter[b], 1);
    if (old == a.H_kv - 1) {
      a.seq_len[b] = L0 + nb;
      a.counter[b] = 0;
      __threadfence();
    }
  }
}

int dense_append_launch(const lrkv_dense_cache& c, const void* k, const void* v, int n,
                        const int* n_new, long long seq_stride, long long head_stride, cudaStream_t st) {
  DenseAppendArgs a;
  a.B = c.batch; a.H_kv = c.num_kv_heads; a.maxp = c.max_pages_per_seq;
  a.num_pages = c.num_pages; a.n = n; a.kvp = c.kv_pages;
  a.bt = c.block_table; a.seq_len = c.seq_len; a.counter = c.append_counter; a.n_new = n_new;
  a.k = k; a.v = v; a.seq_stride = seq_stride; a.head_stride = head_stride;
  dim3 g(a.H_kv, a.B);
  if (c.dtype == LRKV_BF16)
    dense_append_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(a);
  else
    dense_append_kernel<float><<<g, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? LRKV_OK : LRKV_ERR_CUDA;
}

}  // namespace lrkv
