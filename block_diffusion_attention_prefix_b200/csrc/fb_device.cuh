// fb_device.cuh -- device code shared by the attention passes of libfb:
// the reuse gate, warp reductions, and the deterministic log-space combine of
// split-KV partials with its epilogues (write the cache, or merge into A_full).
//
// Gate: FlashBlock technical summary (gist.science 2602.05305), "Adaptive reuse
// strategies": reuse iff M^{s+1} < tau; in the video setting only heads whose
// similarity is above gamma reuse; step 0 of a block always recomputes.
// Combine and merge: same page, "Core mechanism", the log-space merge equation,
// applied to split-KV partials (each split is a key subset of J_out).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_internal.h"

namespace fb {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// M^{s+1} of batch element b, computed by all `nthreads` threads of the block
// (blockDim.x must be a multiple of 32); every thread gets the result.
__device__ __forceinline__ int block_updated_count(const uint8_t* mask_row, int B, int* s_red) {
  int part = 0;
  for (int i = threadIdx.x; i < B; i += blockDim.x) part += mask_row[i] != 0;
  part = warp_sum_int(part);
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_red[warp] = part;
  __syncthreads();
  int M = 0;
  for (int w = 0; w < nwarps; ++w) M += s_red[w];
  __syncthreads();
  return M;
}

__device__ __forceinline__ bool tau_reuse(const GateParams& g, int M) {
  return !g.first && M < g.tau;
}

__device__ __forceinline__ bool head_reuse(const GateParams& g, bool tau_ok, int b, int hq, int h) {
  if (!tau_ok) return false;
  if (g.sim == nullptr) return true;
  return g.sim[(size_t)b * hq + h] > g.gamma;
}

// Row flags of one CTA: s_flags[r] = 1 iff row (row0 + r) of KV group g must be
// (re)computed.  Returns nonzero iff any row of the tile needs work.  Called by
// every thread of the block.
__device__ __forceinline__ int gate_row_flags(const GateParams& g, const Dims& d, int b, int kvh,
                                              int row0, int rows_valid, int row_tile, int* s_flags,
                                              int* s_red) {
  bool tau_ok = false;
  if (g.enabled) {
    const int M = block_updated_count(g.mask + (size_t)b * d.B, d.B, s_red);
    tau_ok = tau_reuse(g, M);
  }
  int mine = 0;
  for (int r = threadIdx.x; r < row_tile; r += blockDim.x) {
    int f = 0;
    if (r < rows_valid) {
      const int h = kvh * d.G + (row0 + r) / d.B;
      f = g.enabled ? !head_reuse(g, tau_ok, b, d.hq, h) : 1;
    }
    s_flags[r] = f;
    mine |= f;
  }
  return __syncthreads_or(mine);
}

// Store a float4 of outputs as fp32 or bf16.
__device__ __forceinline__ void store4(void* base, size_t idx, float4 v, int bf16) {
  if (bf16) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(base) + idx) = u;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(base) + idx) = v;
  }
}

// The merge equation on one float4 of a row: (A1, L1) and (A2, L2) -> (A, L).
__device__ __forceinline__ void merge4(float4 a1, float l1, float4 a2, float l2, float4& a, float& l) {
  const float m = fmaxf(l1, l2);
  if (m == -CUDART_INF_F) {
    a = make_float4(0.f, 0.f, 0.f, 0.f);
    l = -CUDART_INF_F;
    return;
  }
  const float w1 = expf(l1 - m), w2 = expf(l2 - m);  // exp(-inf) = 0
  const float inv = 1.f / (w1 + w2);
  a.x = (w1 * a1.x + w2 * a2.x) * inv;
  a.y = (w1 * a1.y + w2 * a2.y) * inv;
  a.z = (w1 * a1.z + w2 * a2.z) * inv;
  a.w = (w1 * a1.w + w2 * a2.w) * inv;
  l = m + logf(w1 + w2);
}

// Epilogue for one float4 (cols d4*4 .. d4*4+3) of global row `grow` (index into
// [b, H_q, B]) holding the combined (A, L) of a pass.
__device__ __forceinline__ void epilogue4(const Epilogue& ep, int D, size_t grow, int d4, float4 A,
                                          float L) {
  const size_t off = grow * (size_t)D + (size_t)d4 * 4;
  if (ep.mode == 0) {
    *reinterpret_cast<float4*>(ep.a_dst + off) = A;
    if (d4 == 0) ep.l_dst[grow] = L;
  } else {
    const float4 ap = __ldg(reinterpret_cast<const float4*>(ep.a_prev + off));
    const float lp = __ldg(ep.l_prev + grow);
    float4 af;
    float lf;
    merge4(ap, lp, A, L, af, lf);
    store4(ep.a_full, off, af, ep.out_bf16);
    if (d4 == 0 && ep.l_full) ep.l_full[grow] = lf;
  }
}

// Combine the `splits` partials of one (b, kv head, row tile) in fixed split
// order (deterministic) and run the epilogue on flagged rows.  Partials are
// [splits][row_tile][D + 4] fp32: A normalised in cols 0..D-1, L (natural log) in
// col D.  Executed by threads [0, nthr) of the CTA.
__device__ __forceinline__ void combine_splits(const float* part, int splits, int row_tile, int D,
                                               int rows_valid, const int* s_flags, size_t grow0,
                                               const Epilogue& ep, int tid, int nthr) {
  const int D4 = D / 4;
  const size_t rstride = (size_t)D + 4;
  const size_t sstride = (size_t)row_tile * rstride;
  for (int idx = tid; idx < rows_valid * D4; idx += nthr) {
    const int r = idx / D4, d4 = idx - r * D4;
    if (!s_flags[r]) continue;
    const float* pr = part + (size_t)r * rstride;
    float M = -CUDART_INF_F;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(pr + s * sstride + D));
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = -CUDART_INF_F;
    if (M != -CUDART_INF_F) {
      float den = 0.f;
      for (int s = 0; s < splits; ++s) {
        const float Ls = __ldcg(pr + s * sstride + D);
        const float w = expf(Ls - M);
        const float4 a = __ldcg(reinterpret_cast<const float4*>(pr + s * sstride) + d4);
        A.x += w * a.x;
        A.y += w * a.y;
        A.z += w * a.z;
        A.w += w * a.w;
        den += w;
      }
      const float inv = 1.f / den;
      A.x *= inv;
      A.y *= inv;
      A.z *= inv;
      A.w *= inv;
      L = M + logf(den);
    }
    epilogue4(ep, D, grow0 + r, d4, A, L);
  }
}

}  // namespace fb
