// similarity.cu -- the per-head similarity estimate behind the gamma gate, and the
// refresh of the reference queries it compares against.
//
// FlashBlock technical summary (gist.science 2602.05305), "Adaptive reuse
// strategies": in the video setting each head's similarity between the current
// step and the cached one is estimated, and only heads above gamma reuse.  The
// pages give no estimator; the one here (readings S1-S4) is the cosine between a
// head's block queries now and the queries its cache was computed with:
//   sim = <Q, R> / sqrt(<Q, Q> <R, R>)   (float64, rounded to float32).
// The sums run in one fixed order so the float32 result -- and the gate decision
// taken on it -- is reproducible bit for bit: per row ascending d (exact products,
// one rounding per term), rows in chunks of 256 summed as a pairwise tree
// (neighbours first; rows past B are zero), chunk totals in ascending order.
//
// similarity_kernel: grid (chunks, b * H_q), 256 threads, one row per thread; the
// last CTA of a head (arrival counter, self-resetting) adds the chunk totals and
// writes sim.  refresh_kernel: one CTA per (b, head); heads that recomputed copy
// their block queries into the reference.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fb_device.cuh"
#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kSimChunk = 256;

template <typename T>
__global__ void __launch_bounds__(kSimChunk) similarity_kernel(const Dims d, const T* q, const T* q_ref, float* sim,
                                                               double* part, unsigned int* counters, int chunks) {
  __shared__ double s[3][kSimChunk];
  __shared__ int s_last;
  const int c = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int row = c * kSimChunk + t;
  double dqr = 0.0, dqq = 0.0, drr = 0.0;
  if (row < d.B) {
    // 16-byte vector loads of the row; terms still added in ascending d
    constexpr int V = 16 / sizeof(T);
    const uint4* qv = reinterpret_cast<const uint4*>(q + ((size_t)bh * d.B + row) * d.D);
    const uint4* rv = reinterpret_cast<const uint4*>(q_ref + ((size_t)bh * d.B + row) * d.D);
    for (int k = 0; k < d.D / V; ++k) {
      const uint4 x = __ldg(qv + k), y = __ldg(rv + k);
      const T* xa = reinterpret_cast<const T*>(&x);
      const T* ya = reinterpret_cast<const T*>(&y);
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const double a = (double)ldf<T>(xa, e), b = (double)ldf<T>(ya, e);
        dqr = fma(a, b, dqr);  // the product is exact in float64: one rounding per term
        dqq = fma(a, a, dqq);
        drr = fma(b, b, drr);
      }
    }
  }
  s[0][t] = dqr;
  s[1][t] = dqq;
  s[2][t] = drr;
  __syncthreads();
  for (int n = kSimChunk / 2; n >= 1; n >>= 1) {  // pairwise tree, neighbours first
    double v0 = 0.0, v1 = 0.0, v2 = 0.0;
    if (t < n) {
      v0 = s[0][2 * t] + s[0][2 * t + 1];
      v1 = s[1][2 * t] + s[1][2 * t + 1];
      v2 = s[2][2 * t] + s[2][2 * t + 1];
    }
    __syncthreads();
    if (t < n) {
      s[0][t] = v0;
      s[1][t] = v1;
      s[2][t] = v2;
    }
    __syncthreads();
  }
  if (t == 0) {
    double* pc = part + ((size_t)bh * chunks + c) * 3;
    pc[0] = s[0][0];
    pc[1] = s[1][0];
    pc[2] = s[2][0];
    __threadfence();
    const unsigned prev = atomicAdd(counters + bh, 1u);
    __threadfence();
    s_last = prev == (unsigned)chunks - 1u;
  }
  __syncthreads();
  if (!s_last || t != 0) return;
  double tqr = 0.0, tqq = 0.0, trr = 0.0;  // chunk totals in ascending chunk order
  for (int k = 0; k < chunks; ++k) {
    const double* pk = part + ((size_t)bh * chunks + k) * 3;
    tqr = tqr + __ldcg(pk);
    tqq = tqq + __ldcg(pk + 1);
    trr = trr + __ldcg(pk + 2);
  }
  const double den = sqrt(tqq * trr);
  sim[bh] = den > 0.0 ? (float)(tqr / den) : 0.f;
  counters[bh] = 0u;
}

__global__ void refresh_kernel(const Dims d, const uint8_t* q, uint8_t* q_ref, const uint8_t* dec_reuse, int eb) {
  const int bh = blockIdx.x;
  if (dec_reuse[bh]) return;  // the head reused: its reference stays
  const size_t bytes = (size_t)d.B * d.D * eb;
  const uint4* src = reinterpret_cast<const uint4*>(q + bh * bytes);
  uint4* dst = reinterpret_cast<uint4*>(q_ref + bh * bytes);
  for (size_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) dst[i] = __ldg(src + i);
}

}  // namespace

size_t similarity_bytes(const Dims& d) {
  const size_t heads = (size_t)d.b * d.hq;
  const size_t chunks = (d.B + kSimChunk - 1) / kSimChunk;
  return (heads * 4 + 255) / 256 * 256 + heads * chunks * 3 * sizeof(double);
}

cudaError_t launch_similarity(const Dims& d, const void* q, const void* q_ref, float* sim, void* ws, cudaStream_t s) {
  const size_t heads = (size_t)d.b * d.hq;
  const int chunks = (d.B + kSimChunk - 1) / kSimChunk;
  unsigned int* counters = static_cast<unsigned int*>(ws);
  double* part = reinterpret_cast<double*>(static_cast<char*>(ws) + (heads * 4 + 255) / 256 * 256);
  dim3 grid(chunks, (unsigned)heads);
  if (d.dtype == 1)
    similarity_kernel<__nv_bfloat16><<<grid, kSimChunk, 0, s>>>(d, static_cast<const __nv_bfloat16*>(q),
                                                                 static_cast<const __nv_bfloat16*>(q_ref), sim, part,
                                                                 counters, chunks);
  else
    similarity_kernel<float><<<grid, kSimChunk, 0, s>>>(d, static_cast<const float*>(q),
                                                         static_cast<const float*>(q_ref), sim, part, counters, chunks);
  return cudaGetLastError();
}

cudaError_t launch_refresh(const Dims& d, const void* q, void* q_ref, const uint8_t* dec_reuse, cudaStream_t s) {
  refresh_kernel<<<d.b * d.hq, 256, 0, s>>>(d, static_cast<const uint8_t*>(q), static_cast<uint8_t*>(q_ref), dec_reuse,
                                            d.dtype == 1 ? 2 : 4);
  return cudaGetLastError();
}

}  // namespace fb
