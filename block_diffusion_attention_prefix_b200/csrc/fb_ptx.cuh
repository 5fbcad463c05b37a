// fb_ptx.cuh -- thin inline-PTX wrappers used by the sm_100a kernels of libfb.
//
// mbarrier arrive/wait (bounded), TMA tensor loads (cp.async.bulk.tensor, no
// multicast), ldmatrix, bf16 mma.sync and ex2.approx.  Every wait on an mbarrier
// has a time limit: on expiry it records an error code in the device error word
// and reports failure to the caller, which then stops issuing work and returns.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace fb {

// Error codes written to the device error word.
enum : uint32_t {
  DEV_ERR_WAIT_FULL = 1,   // consumer gave up waiting for a TMA tile
  DEV_ERR_WAIT_EMPTY = 2,  // producer gave up waiting for a free stage
  DEV_ERR_WAIT_COMBINE = 3, // the split combine gave up waiting for its bulk copy of the partials
  DEV_ERR_WAIT_PEERS = 4,   // a split CTA gave up waiting for the other splits of its tile
};

// 2 s: far above any legitimate wait (a tile load takes microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, at most kWaitLimitNs.
// Returns false (after recording `code` in *err) if the limit was reached.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* err,
                                                  uint32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      if (err) atomicCAS(err, 0u, code);
      return false;
    }
  }
}

// Wait until the global counter *p reaches `target` (acquire), at most kWaitLimitNs.
// Only for counters that CTAs of the same (cooperative) launch increment.
__device__ __forceinline__ bool wait_count_bounded(const unsigned int* p, unsigned int target, uint32_t* err,
                                                   uint32_t code) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      if (err) atomicCAS(err, 0u, code);
      return false;
    }
  }
}

// 3-D tiled TMA load (no multicast) into shared memory; completion is signalled
// on `bar` as transaction bytes.  c0 is the innermost coordinate (elements).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 1-D bulk copy global -> shared (no multicast); both addresses 16-byte aligned,
// size a multiple of 16.  Completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Orders this thread's view of global memory (generic proxy) before its
// subsequent async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Brings the 128-byte line holding `p` into this SM's L1 (no result, no fault on a
// valid address).
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held one row pair per thread: thread t gives
// {M[t/4][2(t%4)], M[t/4][2(t%4)+1]} and gets {M[2(t%4)][t/4], M[2(t%4)+1][t/4]}.
// A pure register operation (not volatile), so the compiler may schedule the loads
// that feed it early.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// mma.sync as a pure register operation (not volatile): same instruction as
// mma_bf16_16816, free for the compiler to schedule around the loads that feed it.
__device__ __forceinline__ void mma_bf16_16816_free(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                    uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Asynchronous global -> shared copies of 16 or 4 bytes (cp.async), completed by
// cp_async_wait_all() in the issuing thread.
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* sdst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// 8-byte async copy (.ca: the .cg form takes 16 bytes only); both addresses 8-byte aligned.
__device__ __forceinline__ void cp_async8(void* sdst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// 16-byte async copy that zero-fills the destination when `valid` is false (no bytes
// are read then; gsrc must still be a valid address).  Through L1 (.ca), so lines
// an earlier prefetch brought into L1 are served from there.
__device__ __forceinline__ void cp_async16_zfill(void* sdst, const void* gsrc, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(sdst)), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}

// 2^x with the hardware approximation (inputs here are <= 0 or -inf).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes, for softmax exponentials that would otherwise
// queue on the special-function unit.  Range reduction x = n + f with n = round(x)
// (adding and subtracting 1.5 * 2^23 rounds to the nearest integer and leaves n in
// the low mantissa bits of the sum), f in [-1/2, 1/2]; 2^f by a cubic with p(0) = 1
// whose coefficients minimise the largest relative error on [-1/2, 1/2] (Lawson's
// iteratively reweighted least squares; gen_exp2_poly.py in this folder refits
// them); then 2^n is added into the exponent field.  Relative error <= 1.02e-4 for
// x in [-125, 2^22) (below bf16's half ulp, the precision P is kept in); exact at
// integers; 0 for x < -125 and for -inf.
__device__ __forceinline__ float exp2_fma(float x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float t = __fadd_rn(x, kRound);
  const float f = __fsub_rn(x, __fsub_rn(t, kRound));
  const float p = fmaf(f, fmaf(f, fmaf(f, 0.05500892966239863f, 0.2422109719919523f), 0.6932829287944439f), 1.0f);
  const float r = __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
  return x < -125.0f ? 0.0f : r;
}

// Packed pairs of floats for the sm_100 two-wide fp32 instructions (one issue slot
// per pair): f2_pack / f2_unpack only rename registers.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// exp2_fma on a pair, its float steps two-wide: the same roundings, so each half
// equals exp2_fma of that half bit for bit.
__device__ __forceinline__ void exp2_fma2(float x0, float x1, float& y0, float& y1) {
  constexpr float kRound = 12582912.0f;
  const uint64_t X = f2_pack(x0, x1);
  const uint64_t R = f2_pack(kRound, kRound);
  const uint64_t T = f2_add(X, R);
  const uint64_t F = f2_sub(X, f2_sub(T, R));
  uint64_t P = f2_fma(F, f2_pack(0.05500892966239863f, 0.05500892966239863f),
                      f2_pack(0.2422109719919523f, 0.2422109719919523f));
  P = f2_fma(F, P, f2_pack(0.6932829287944439f, 0.6932829287944439f));
  P = f2_fma(F, P, f2_pack(1.0f, 1.0f));
  float p0, p1, t0, t1;
  f2_unpack(P, p0, p1);
  f2_unpack(T, t0, t1);
  const float r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  const float r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
  y0 = x0 < -125.0f ? 0.0f : r0;
  y1 = x1 < -125.0f ? 0.0f : r1;
}

// Largest of three (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier over `nthreads` threads that also returns the AND of `pred` over them,
// so that every participant takes the same branch afterwards.
__device__ __forceinline__ bool named_barrier_and(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

}  // namespace fb
