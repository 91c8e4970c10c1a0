// Device helpers shared by the latent-KV kernels (sm_100a).
//
// Layouts (all caller-owned device memory):
//  * Latent code pages, chunk-major: [page][kv head][r / CE][64 tokens][CE],
//    where a chunk is 16 bytes (CE = 8 bf16 or 4 fp32 elements).  A page of
//    one head is one contiguous slab, so one bulk copy moves it, and lane t
//    reading chunk j of token t touches consecutive 16-byte words: no bank
//    conflicts without a swizzle.
//  * Full-rank tiles (anchors and the dense baseline) use the same
//    chunk-major form with 32 tokens per tile: [tile][128 / CE][32][CE].
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "lrkv.h"

namespace lrkv {

constexpr int kHeadDim = 128;
constexpr int kLatPage = LRKV_PAGE_TOKENS;     // tokens per latent page
constexpr int kFrTile = LRKV_FULL_RANK_TILE;   // tokens per full-rank tile
constexpr float kLog2e = 1.4426950408889634f;

// Value-amortised slabs (LRKV_BF16_VA): key codes [rk / 8][64][8] bf16,
// residual rows [rv / 8][kVaKeep][8] bf16, slot rows int32 [kVaKeep], slot
// squared norms fp32 [kVaKeep].
constexpr int kVaKeep = LRKV_VA_KEEP;
__host__ __device__ inline int va_slab_bytes(int rk, int rv) {
  return kLatPage * rk * 2 + kVaKeep * rv * 2 + kVaKeep * 8;
}

// Error word values written to the first 4 bytes of a decode workspace.
constexpr int kErrNone = 0;
constexpr int kErrTimeout = 1;
constexpr int kErrBadPage = 2;

template <typename T> struct Elem;
template <> struct Elem<__nv_bfloat16> { static constexpr int CE = 8; };
template <> struct Elem<float> { static constexpr int CE = 4; };

// ------------------------------------------------------------ token split
// Sequence of L tokens: the first min(L, n_sink) are the sink; of the rest
// the most recent min(rest, W) form the window; the others are latent.
struct Split {
  int sink, win, lat;
};
__host__ __device__ inline Split split_tokens(int L, int n_sink, int W) {
  Split s;
  s.sink = L < n_sink ? L : n_sink;
  int rest = L - s.sink;
  s.win = rest < W ? rest : W;
  s.lat = rest - s.win;
  return s;
}

// ------------------------------------------------------------ PTX wrappers
__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ inline void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ inline uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: gives up after ~timeout_ns and returns false.
__device__ inline bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                         uint64_t timeout_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > timeout_ns) return false;
  }
}
// L2 policy for data read once: evict first, so small hot data stays in L2.
// L2 evict-last policy: small arrays every call reads (the bases) stay in
// L2 while the code pages stream past with evict-first.
__device__ inline uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ inline float4 ldg_f4_hint(const float4* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ inline float ldg_f_hint(const float* p, uint64_t pol) {
  float v;
  asm volatile("ld.global.nc.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(p), "l"(pol));
  return v;
}
__device__ inline uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// Bulk copy with an L2 cache-policy hint.
__device__ inline void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                     uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
// One bulk copy global -> shared completing on an mbarrier (no multicast).
__device__ inline void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk copy shared -> global through the async proxy, tracked in the
// issuing thread's bulk groups (commit, then wait for reads or completion).
__device__ inline void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ inline void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// At most N of this thread's committed bulk groups still read shared memory.
template <int N>
__device__ inline void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// At most N of this thread's committed bulk groups are still in flight.
template <int N>
__device__ inline void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Shared-memory writes of this thread (and, after a barrier, of the threads
// it synchronised with) become visible to later async-proxy reads.
__device__ inline void proxy_fence_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ conversions
// bf16 pair in one 32-bit word -> two floats (exact).
__device__ inline float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ inline float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Unpack one 16-byte chunk into CE floats.
template <typename T>
__device__ inline void unpack_chunk(const uint4& c, float* f);
template <>
__device__ inline void unpack_chunk<__nv_bfloat16>(const uint4& c, float* f) {
  f[0] = bf_lo(c.x); f[1] = bf_hi(c.x);
  f[2] = bf_lo(c.y); f[3] = bf_hi(c.y);
  f[4] = bf_lo(c.z); f[5] = bf_hi(c.z);
  f[6] = bf_lo(c.w); f[7] = bf_hi(c.w);
}
template <>
__device__ inline void unpack_chunk<float>(const uint4& c, float* f) {
  f[0] = __uint_as_float(c.x); f[1] = __uint_as_float(c.y);
  f[2] = __uint_as_float(c.z); f[3] = __uint_as_float(c.w);
}

template <typename T> __device__ inline float to_f(T x);
template <> __device__ inline float to_f<float>(float x) { return x; }
template <> __device__ inline float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ inline T from_f(float x);
template <> __device__ inline float from_f<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ------------------------------------------------------------ packed fp32
// d += a * b on two fp32 lanes at once (sm_100 packed FMA).
__device__ __forceinline__ void fma2(float2& d, const float2 a, const float2 b) {
  unsigned long long dd, aa, bb;
  memcpy(&dd, &d, 8); memcpy(&aa, &a, 8); memcpy(&bb, &b, 8);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(dd) : "l"(aa), "l"(bb));
  memcpy(&d, &dd, 8);
}
__device__ __forceinline__ float2 mul2(const float2 a, const float2 b) {
  unsigned long long dd, aa, bb;
  memcpy(&aa, &a, 8); memcpy(&bb, &b, 8);
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(dd) : "l"(aa), "l"(bb));
  float2 d;
  memcpy(&d, &dd, 8);
  return d;
}
// bf16 pair word -> (even, odd) floats as one packed pair.
__device__ __forceinline__ float2 bf2(uint32_t w) { return make_float2(bf_lo(w), bf_hi(w)); }

// Programmatic dependent launch controls.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Named barrier over `threads` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also returns whether any of its threads passed
// pred = true (the same answer in every thread).
__device__ __forceinline__ bool named_bar_any(int id, int threads, bool pred) {
  int r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.s32 p, %1, 0;\n"
      " bar.red.or.pred q, %2, %3, p;\n selp.s32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((int)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- 16-byte asynchronous copies global -> shared (zero-filled when
// src_bytes == 0), committed and awaited in groups
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- thread-block clusters
__device__ __forceinline__ void cluster_arrive() {  // release: prior accesses ordered first
  asm volatile("barrier.cluster.arrive;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {  // acquire
  asm volatile("barrier.cluster.wait;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// ---- warp-level bf16 tensor-core tiles (m16n8k16, fp32 accumulate).
// Fragment ownership, with g = lane / 4 and t = lane % 4:
//   A (16x16, row-major): a0 (g, 2t..2t+1) a1 (g+8, 2t..) a2 (g, 2t+8..) a3 (g+8, 2t+8..)
//   B (16x8, col-major):  b0 (2t..2t+1, g)  b1 (2t+8..2t+9, g)
//   C (16x8):             c0 c1 (g, 2t..2t+1)  c2 c3 (g+8, 2t..2t+1)
// Each 32-bit register holds two bf16, the lower column index in the low half.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm(  // pure register operation: free to schedule
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Transpose of an 8x8 b16 matrix held one row pair per lane (row g, cols 2t..2t+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// 2^x by the PTX approximate base-2 exponential (subnormal results flush to 0;
// exp2(-inf) = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Two floats -> bf16x2, round to nearest even; `lo` goes to the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Element offset of (chunk c, token row, elem e) inside one chunk-major slab.
__host__ __device__ inline int64_t slab_off(int c, int row, int rows, int CE) {
  return ((int64_t)c * rows + row) * CE;
}

}  // namespace lrkv
