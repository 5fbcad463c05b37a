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
//  * merge_parts_kernel: the context-parallel combine -- the prefix split into P
//    key ranges (one per GPU), each range's partial (A, L), and the cache rows of
//    the heads that recompute set to the merge of all P partials in range order
//    (the merge equation over a partition of J_out).
//  * append_block_kernel: the block transition -- once a block's last step is
//    done its tokens belong to the prefix: their K/V rows are copied to the end
//    of the prefix cache (the prefix J_out grows by B; FlashBlock technical
//    summary, "1. Problem definition").
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

// One CTA per (b, query head): gate, decision record, in-block rows of that head
// (one warp per row).
template <typename T, int DC>
__global__ void __launch_bounds__(kSmallThreads) small_block_kernel(const SmallBlockArgs a) {
  constexpr int D = 32 * DC;
  __shared__ int s_red[32];
  const Dims& d = a.d;
  const int h = blockIdx.x, b = blockIdx.y;
  const int kvh = h / d.G;
  const int tid = threadIdx.x;
  if (a.gate.enabled) {
    const int M = block_updated_count(a.gate.mask + (size_t)b * d.B, d.B, s_red);
    if (tid == 0) {
      const bool t = tau_reuse(a.gate, M);
      if (a.dec_reuse) a.dec_reuse[(size_t)b * d.hq + h] = head_reuse(a.gate, t, b, d.hq, h) ? 1 : 0;
      if (a.dec_M && h == 0) a.dec_M[b] = M;
    }
  }
  extern __shared__ __align__(16) uint8_t tile_smem[];  // bf16: a tile memory per warp
  inblock_rows<T, D>(d, static_cast<const T*>(a.q), static_cast<const T*>(a.k_blk),
                     static_cast<const T*>(a.v_blk), b, kvh, (h - kvh * d.G) * d.B, 0, d.B, a.ep, tid >> 5,
                     kSmallThreads / 32, tid & 31, tile_smem);
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

// One CTA per (query head, b), a warp per row: the merge of the P partials of each
// row in range order -- M = max_p L_p, e_p = e^{L_p - M}, den = sum_p e_p (in order),
// A = (sum_p e_p A_p) / den, L = M + ln den -- written to the cache, for the heads
// whose gate decision is "recompute" (all heads without a gate).  Rows of reusing
// heads are left untouched.
template <int DC>
__global__ void __launch_bounds__(128) merge_parts_kernel(const Dims d, const GateParams g, const float* a_parts,
                                                           long long a_stride, const float* l_parts,
                                                           long long l_stride, int P, float* a_out, float* l_out) {
  constexpr int D = 32 * DC;
  __shared__ int s_red[32];
  const int h = blockIdx.x, b = blockIdx.y;
  if (g.enabled) {
    const int M = block_updated_count(g.mask + (size_t)b * d.B, d.B, s_red);
    if (head_reuse(g, tau_reuse(g, M), b, d.hq, h)) return;  // uniform over the CTA
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < d.B; i += 4) {
    const size_t grow = ((size_t)b * d.hq + h) * d.B + i;
    float M = -CUDART_INF_F;
    for (int p = 0; p < P; ++p) M = fmaxf(M, __ldg(l_parts + p * l_stride + grow));
    float acc[DC], den = 0.f;
#pragma unroll
    for (int t = 0; t < DC; ++t) acc[t] = 0.f;
    if (M != -CUDART_INF_F) {
      for (int p = 0; p < P; ++p) {
        const float e = expf(__ldg(l_parts + p * l_stride + grow) - M);
        float a[DC];
        load_vec<DC>(a_parts + p * a_stride + grow * D + lane * DC, a);
        den += e;
#pragma unroll
        for (int t = 0; t < DC; ++t) acc[t] = fmaf(e, a[t], acc[t]);
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int t = 0; t < DC; ++t) a_out[grow * D + lane * DC + t] = acc[t] * inv;
    if (lane == 0) l_out[grow] = den > 0.f ? M + logf(den) : -CUDART_INF_F;
  }
}

// Block transition: CTA (chunk, b * H_kv) copies rows [64 chunk, 64 chunk + 64) of the
// block's K and V into cache rows N + those (16-byte vectors; cache rows may be padded).
constexpr int kAppendRows = 64;
__global__ void append_block_kernel(const Dims d, uint8_t* k_cache, uint8_t* v_cache, const uint8_t* k_blk,
                                    const uint8_t* v_blk, int elem_bytes) {
  const int bg = blockIdx.y;
  const int row0 = blockIdx.x * kAppendRows;
  const int rows = min(kAppendRows, d.B - row0);
  const int vec_per_row = d.D * elem_bytes / 16;
  const size_t n = (size_t)rows * vec_per_row;
  const size_t src0 = ((size_t)bg * d.B + row0) * d.D * elem_bytes;
  const size_t dst0 = ((size_t)bg * d.head_stride + (size_t)(d.N + row0) * d.row_stride) * elem_bytes;
  for (size_t i = threadIdx.x; i < 2 * n; i += blockDim.x) {
    const bool isv = i >= n;
    const size_t j = isv ? i - n : i;
    const size_t row = j / vec_per_row, c = j - row * vec_per_row;
    const uint4 x = __ldg(reinterpret_cast<const uint4*>((isv ? v_blk : k_blk) + src0 + row * d.D * elem_bytes) + c);
    reinterpret_cast<uint4*>((isv ? v_cache : k_cache) + dst0 + row * d.row_stride * elem_bytes)[c] = x;
  }
}

template <typename T, int DC>
cudaError_t launch_small_dc(const SmallBlockArgs& a, const dim3& grid, cudaStream_t s) {
  // bf16 takes a tensor-core tile memory per warp (dynamic shared memory)
  constexpr size_t smem = std::is_same<T, __nv_bfloat16>::value ? (kSmallThreads / 32) * TileSmem<32 * DC>::kBytes : 0;
  if (smem > 48 * 1024) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      const cudaError_t e =
          cudaFuncSetAttribute(small_block_kernel<T, DC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  small_block_kernel<T, DC><<<grid, kSmallThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_small_t(const SmallBlockArgs& a, cudaStream_t s) {
  dim3 grid(a.d.hq, a.d.b);
  switch (a.d.D / 32) {
    case 1: return launch_small_dc<T, 1>(a, grid, s);
    case 2: return launch_small_dc<T, 2>(a, grid, s);
    case 3: return launch_small_dc<T, 3>(a, grid, s);
    case 4: return launch_small_dc<T, 4>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
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

cudaError_t launch_append_block(const Dims& d, void* k_cache, void* v_cache, const void* k_blk, const void* v_blk,
                                cudaStream_t s) {
  const dim3 grid((d.B + kAppendRows - 1) / kAppendRows, d.b * d.hkv);
  append_block_kernel<<<grid, 256, 0, s>>>(d, static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache),
                                                   static_cast<const uint8_t*>(k_blk),
                                                   static_cast<const uint8_t*>(v_blk), d.dtype == 1 ? 2 : 4);
  return cudaGetLastError();
}

cudaError_t launch_merge_parts(const Dims& d, const GateParams& g, const float* a_parts, long long a_stride,
                               const float* l_parts, long long l_stride, int P, float* a_out, float* l_out,
                               cudaStream_t s) {
  const dim3 grid(d.hq, d.b);
  switch (d.D / 32) {
    case 1: merge_parts_kernel<1><<<grid, 128, 0, s>>>(d, g, a_parts, a_stride, l_parts, l_stride, P, a_out, l_out); break;
    case 2: merge_parts_kernel<2><<<grid, 128, 0, s>>>(d, g, a_parts, a_stride, l_parts, l_stride, P, a_out, l_out); break;
    case 3: merge_parts_kernel<3><<<grid, 128, 0, s>>>(d, g, a_parts, a_stride, l_parts, l_stride, P, a_out, l_out); break;
    case 4: merge_parts_kernel<4><<<grid, 128, 0, s>>>(d, g, a_parts, a_stride, l_parts, l_stride, P, a_out, l_out); break;
    default: return cudaErrorInvalidValue;
  }
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
