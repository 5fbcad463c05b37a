// similarity.cu -- the per-head similarity estimate behind the gamma gate, and the
// refresh of the reference queries it compares against.
//
// FlashBlock technical summary (gist.science 2602.05305), "Adaptive reuse
// strategies": in the video setting each head's similarity between the current
// step and the cached one is estimated, and only heads above gamma reuse.  The
// pages give no estimator; the one here (readings S1-S4) is the cosine between a
// head's block queries now and the queries its cache was computed with:
//   sim = <Q, R> / sqrt(<Q, Q> <R, R>)   (float64, rounded to float32).
// The sums run in one plain order so the float32 result -- and the gate decision
// taken on it -- is reproducible bit for bit: each row's products in ascending d
// (exact products, one rounding per term) give the row's dot product, and the row
// dot products are added one after another in ascending row order.
//
// similarity_kernel: grid (ceil(B / 256), b * H_q), 256 threads, one row per
// thread: the three row dot products go to the workspace.  The last CTA of a head
// to arrive (arrival counter, self-resetting) stages the head's row sums through
// shared memory in tiles and adds them in row order -- one thread per sum, a chain
// of B float64 additions -- then writes sim.  refresh_kernel: one CTA per
// (b, head); heads that recomputed copy their block queries into the reference.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fb_device.cuh"
#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kSimRows = 256;   // rows per CTA (one per thread)
constexpr int kSimTile = 1024;  // row sums staged per tile by the finishing CTA

template <typename T>
__global__ void __launch_bounds__(kSimRows) similarity_kernel(const Dims d, const T* q, const T* q_ref, float* sim,
                                                              double* rows, unsigned int* counters, int chunks) {
  __shared__ double s[kSimTile][4];
  __shared__ int s_last;
  const int c = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int row = c * kSimRows + t;
  if (row < d.B) {
    double dqr = 0.0, dqq = 0.0, drr = 0.0;
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
    double2* dst = reinterpret_cast<double2*>(rows) + ((size_t)bh * d.B + row) * 2;  // 16-byte aligned
    dst[0] = make_double2(dqr, dqq);
    dst[1] = make_double2(drr, 0.0);
  }
  __threadfence();
  __syncthreads();
  if (t == 0) {
    const unsigned prev = atomicAdd(counters + bh, 1u);
    s_last = prev == (unsigned)chunks - 1u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // Every row sum of the head is written: add them in ascending row order.
  const double2* src = reinterpret_cast<const double2*>(rows) + (size_t)bh * d.B * 2;
  double acc = 0.0;  // thread t < 3 carries sum t
  for (int r0 = 0; r0 < d.B; r0 += kSimTile) {
    const int n = min(kSimTile, d.B - r0);
    for (int i = t; i < n; i += kSimRows) {
      const double2 v0 = __ldcg(src + (size_t)(r0 + i) * 2), v1 = __ldcg(src + (size_t)(r0 + i) * 2 + 1);
      s[i][0] = v0.x;
      s[i][1] = v0.y;
      s[i][2] = v1.x;
    }
    __syncthreads();
    if (t < 3) {
#pragma unroll 8
      for (int i = 0; i < n; ++i) acc = acc + s[i][t];
    }
    __syncthreads();
  }
  if (t < 3) s[0][t] = acc;
  __syncthreads();
  if (t == 0) {
    const double tqr = s[0][0], tqq = s[0][1], trr = s[0][2];
    const double den = sqrt(tqq * trr);
    sim[bh] = den > 0.0 ? (float)(tqr / den) : 0.f;
    counters[bh] = 0u;
  }
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
  return (heads * 4 + 255) / 256 * 256 + heads * (size_t)d.B * 4 * sizeof(double);
}

cudaError_t launch_similarity(const Dims& d, const void* q, const void* q_ref, float* sim, void* ws, cudaStream_t s) {
  const size_t heads = (size_t)d.b * d.hq;
  const int chunks = (d.B + kSimRows - 1) / kSimRows;
  unsigned int* counters = static_cast<unsigned int*>(ws);
  double* rows = reinterpret_cast<double*>(static_cast<char*>(ws) + (heads * 4 + 255) / 256 * 256);
  dim3 grid(chunks, (unsigned)heads);
  if (d.dtype == 1)
    similarity_kernel<__nv_bfloat16><<<grid, kSimRows, 0, s>>>(d, static_cast<const __nv_bfloat16*>(q),
                                                                static_cast<const __nv_bfloat16*>(q_ref), sim, rows,
                                                                counters, chunks);
  else
    similarity_kernel<float><<<grid, kSimRows, 0, s>>>(d, static_cast<const float*>(q),
                                                        static_cast<const float*>(q_ref), sim, rows, counters, chunks);
  return cudaGetLastError();
}

cudaError_t launch_refresh(const Dims& d, const void* q, void* q_ref, const uint8_t* dec_reuse, cudaStream_t s) {
  refresh_kernel<<<d.b * d.hq, 256, 0, s>>>(d, static_cast<const uint8_t*>(q), static_cast<uint8_t*>(q_ref), dec_reuse,
                                            d.dtype == 1 ? 2 : 4);
  return cudaGetLastError();
}

}  // namespace fb
