// block_merge.cu -- the per-step kernels that do not touch the prefix:
//
//  * small_block_kernel: for blocks of up to 64 tokens, one CTA per (b, query
//    head) evaluates the reuse gate, records the decision, computes the in-block
//    attention (A_in, L_in) over the B block keys (bidirectional), and merges it
//    with the cached (A_out, L_out) in log space into A_full.  A reuse step of a
//    dLM-sized layer is this one launch: it reads only Q, the in-block K/V and
//    the cache.  (FlashBlock technical summary, gist.science 2602.05305, "Core
//    mechanism" merge equation and "Adaptive reuse strategies" gates.)
//  * gate_kernel: the gate alone (M^{s+1} and the per-head decisions).
//  * merge_kernel: the merge equation alone, elementwise, 16-byte vectors.
//
// The in-block scores are B x B per head (B <= 64): CUDA cores, fp32 math.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_device.cuh"
#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kSmallThreads = 128;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, size_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// Dynamic shared memory: sK [B][D+1], sV [B][D], sQ [4 warps][D]  (fp32)
template <typename T, int DC>
__global__ void __launch_bounds__(kSmallThreads) small_block_kernel(const SmallBlockArgs a) {
  constexpr int D = 32 * DC;
  extern __shared__ float sm[];
  __shared__ int s_red[32];
  const Dims& d = a.d;
  const int h = blockIdx.x, b = blockIdx.y;
  const int kvh = h / d.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = d.B;
  float* sK = sm;
  float* sV = sK + (size_t)B * (D + 1);
  float* sQ = sV + (size_t)B * D;

  // Gate and decision record.
  if (a.gate.enabled) {
    const int M = block_updated_count(a.gate.mask + (size_t)b * B, B, s_red);
    if (tid == 0) {
      const bool t = tau_reuse(a.gate, M);
      if (a.dec_reuse) a.dec_reuse[(size_t)b * d.hq + h] = head_reuse(a.gate, t, b, d.hq, h) ? 1 : 0;
      if (a.dec_M && h == 0) a.dec_M[b] = M;
    }
  }

  const T* kb = static_cast<const T*>(a.k_blk) + (size_t)(b * d.hkv + kvh) * B * D;
  const T* vb = static_cast<const T*>(a.v_blk) + (size_t)(b * d.hkv + kvh) * B * D;
  for (int i = tid; i < B * D; i += kSmallThreads) {
    const int j = i / D, dd = i - j * D;
    sK[(size_t)j * (D + 1) + dd] = ldf(kb, i);
    sV[i] = ldf(vb, i);
  }
  __syncthreads();

  const T* qh = static_cast<const T*>(a.q) + (size_t)(b * d.hq + h) * B * D;
  float* sq = sQ + warp * D;
  for (int i = warp; i < B; i += kSmallThreads / 32) {
#pragma unroll
    for (int t = 0; t < DC; ++t) sq[lane + 32 * t] = ldf(qh, (size_t)i * D + lane + 32 * t);
    __syncwarp();
    // scores: lane j handles keys j, j + 32 (B <= 64)
    float s0 = -CUDART_INF_F, s1 = -CUDART_INF_F;
    if (lane < B) {
      float acc = 0.f;
      const float* kr = sK + (size_t)lane * (D + 1);
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) acc = fmaf(sq[dd], kr[dd], acc);
      s0 = acc * d.scale;
    }
    if (lane + 32 < B) {
      float acc = 0.f;
      const float* kr = sK + (size_t)(lane + 32) * (D + 1);
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) acc = fmaf(sq[dd], kr[dd], acc);
      s1 = acc * d.scale;
    }
    const float mx = warp_max(fmaxf(s0, s1));
    const float p0 = lane < B ? expf(s0 - mx) : 0.f;
    const float p1 = lane + 32 < B ? expf(s1 - mx) : 0.f;
    const float z = warp_sum(p0 + p1);
    const float inv = 1.f / z;
    const float Lin = mx + logf(z);
    float ain[DC];
#pragma unroll
    for (int t = 0; t < DC; ++t) ain[t] = 0.f;
    for (int j = 0; j < B; ++j) {
      const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
      for (int t = 0; t < DC; ++t) ain[t] = fmaf(pj, sV[(size_t)j * D + lane + 32 * t], ain[t]);
    }
    const size_t grow = (size_t)(b * d.hq + h) * B + i;
    if (a.ep.mode == 0) {
#pragma unroll
      for (int t = 0; t < DC; ++t) a.ep.a_dst[grow * D + lane + 32 * t] = ain[t] * inv;
      if (lane == 0) a.ep.l_dst[grow] = Lin;
    } else {
      const float lp = __ldg(a.ep.l_prev + grow);
      const float m = fmaxf(lp, Lin);  // Lin is finite (B >= 1)
      const float wp = expf(lp - m), wi = expf(Lin - m);
      const float den = wp + wi;
      const float rden = 1.f / den;
#pragma unroll
      for (int t = 0; t < DC; ++t) {
        const size_t off = grow * D + lane + 32 * t;
        const float v = (wp * __ldg(a.ep.a_prev + off) + wi * ain[t] * inv) * rden;
        if (a.ep.out_bf16)
          static_cast<__nv_bfloat16*>(a.ep.a_full)[off] = __float2bfloat16_rn(v);
        else
          static_cast<float*>(a.ep.a_full)[off] = v;
      }
      if (lane == 0 && a.ep.l_full) a.ep.l_full[grow] = m + logf(den);
    }
    __syncwarp();
  }
}

__global__ void gate_kernel(const Dims d, const GateParams g, int32_t* dec_M, uint8_t* dec_reuse) {
  __shared__ int s_red[32];
  const int b = blockIdx.x;
  const int M = block_updated_count(g.mask + (size_t)b * d.B, d.B, s_red);
  const bool t = tau_reuse(g, M);
  if (threadIdx.x == 0 && dec_M) dec_M[b] = M;
  if (dec_reuse)
    for (int h = threadIdx.x; h < d.hq; h += blockDim.x)
      dec_reuse[(size_t)b * d.hq + h] = head_reuse(g, t, b, d.hq, h) ? 1 : 0;
}

__global__ void merge_kernel(const Dims d, const float* a1, const float* l1, const float* a2,
                             const float* l2, void* a_full, float* l_full, size_t rows) {
  const int D4 = d.D / 4;
  const size_t n = rows * D4;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < n;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t r = idx / D4;
    const int d4 = (int)(idx - r * D4);
    const size_t off = r * d.D + (size_t)d4 * 4;
    float4 a;
    float l;
    merge4(__ldg(reinterpret_cast<const float4*>(a1 + off)), __ldg(l1 + r),
           __ldg(reinterpret_cast<const float4*>(a2 + off)), __ldg(l2 + r), a, l);
    store4(a_full, off, a, d.dtype == 1);
    if (d4 == 0 && l_full) l_full[r] = l;
  }
}

template <typename T>
cudaError_t launch_small_t(const SmallBlockArgs& a, cudaStream_t s) {
  const int DC = a.d.D / 32;
  const size_t smem = ((size_t)a.d.B * (a.d.D + 1) + (size_t)a.d.B * a.d.D + 4 * (size_t)a.d.D) * 4;
  dim3 grid(a.d.hq, a.d.b);
#define FB_SMALL_CASE(X)                                                                              \
  case X: {                                                                                           \
    auto k = small_block_kernel<T, X>;                                                                \
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                   \
    k<<<grid, kSmallThreads, smem, s>>>(a);                                                           \
    break;                                                                                            \
  }
  switch (DC) {
    FB_SMALL_CASE(1)
    FB_SMALL_CASE(2)
    FB_SMALL_CASE(3)
    FB_SMALL_CASE(4)
    default:
      return cudaErrorInvalidValue;
  }
#undef FB_SMALL_CASE
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_small_block(const SmallBlockArgs& a, cudaStream_t s) {
  return a.d.dtype == 1 ? launch_small_t<__nv_bfloat16>(a, s) : launch_small_t<float>(a, s);
}

cudaError_t launch_gate_eval(const Dims& d, const GateParams& g, int32_t* dec_M, uint8_t* dec_reuse,
                             cudaStream_t s) {
  gate_kernel<<<d.b, 128, 0, s>>>(d, g, dec_M, dec_reuse);
  return cudaGetLastError();
}

cudaError_t launch_merge(const Dims& d, const float* a1, const float* l1, const float* a2, const float* l2,
                         void* a_full, float* l_full, cudaStream_t s) {
  const size_t rows = (size_t)d.b * d.hq * d.B;
  const size_t n = rows * (d.D / 4);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  size_t blocks = (n + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  merge_kernel<<<(unsigned)blocks, threads, 0, s>>>(d, a1, l1, a2, l2, a_full, l_full, rows);
  return cudaGetLastError();
}

}  // namespace fb
