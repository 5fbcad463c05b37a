// prefix_f32.cu -- split-KV attention pass over an fp32 KV cache on CUDA cores.
//
// Same contract as the bf16 pass (prefix_bf16.cu): (A, L) of every query row of
// a KV-head group over a key range, partials per split, deterministic
// last-CTA combine.  fp32 keeps the 1e-5 tolerance of fp32 workloads (tf32 tensor
// cores would not), and the fp32 workload is small, so CUDA cores suffice.
// Softmax is computed in natural units with expf/logf.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_device.cuh"
#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kThreads = 128;
constexpr int kRowTileF32 = 16;
constexpr int kKeyTileF32 = 32;

// Dynamic shared memory (floats): Q tile, K and V key tiles.
__host__ __device__ constexpr size_t f32_smem_floats(int D) {
  return (size_t)kRowTileF32 * D + (size_t)kKeyTileF32 * (D + 1) + (size_t)kKeyTileF32 * D;
}

template <int DC>  // D = 32 * DC
__global__ void __launch_bounds__(kThreads) pass_f32_kernel(const PassArgs args) {
  constexpr int D = 32 * DC;
  constexpr int RT = kRowTileF32;
  constexpr int KT = kKeyTileF32;
  extern __shared__ float fsm[];
  float (*sQ)[D] = reinterpret_cast<float (*)[D]>(fsm);
  float (*sK)[D + 1] = reinterpret_cast<float (*)[D + 1]>(fsm + RT * D);
  float (*sV)[D] = reinterpret_cast<float (*)[D]>(fsm + RT * D + KT * (D + 1));
  __shared__ int s_flags[RT];
  __shared__ int s_red[32];
  __shared__ int s_last;
  __shared__ int s_M;

  const Dims& d = args.d;
  const SplitPlan& plan = args.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, rt = blockIdx.y, bg = blockIdx.z;
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int row0 = rt * RT;
  const int rows_valid = min(RT, d.R - row0);

  Epilogue step_ep;
  step_ep.mode = 1;
  step_ep.a_dst = nullptr;
  step_ep.l_dst = nullptr;
  step_ep.a_prev = args.ep.a_dst;
  step_ep.l_prev = args.ep.l_dst;
  step_ep.a_full = args.step.a_full;
  step_ep.l_full = args.step.l_full;
  step_ep.out_bf16 = 0;
  const int per = (rows_valid + plan.splits - 1) / plan.splits;
  const int ib0 = min(rows_valid, split * per), ib1 = min(rows_valid, ib0 + per);
  const size_t unit = (size_t)bg * plan.n_row_tiles + rt;

  if (!gate_row_flags(args.gate, d, b, kvh, row0, rows_valid, RT, &s_flags[0], s_red, &s_M)) {
    // Every row reuses its cache: in a fused step, merge this split's rows with it
    // (unless the reuse-rows kernel already did).
    if (args.step.enabled && !args.step.reuse_done) {
      inblock_rows<float, D>(d, static_cast<const float*>(args.q), static_cast<const float*>(args.step.k_blk),
                             static_cast<const float*>(args.step.v_blk), b, kvh, row0, ib0, ib1, step_ep, warp,
                             kThreads / 32, lane);
      if (split == 0)
        record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, s_M, args.step.dec_M,
                         args.step.dec_reuse, kvh == 0 && rt == 0, tid, kThreads);
    }
    return;
  }
  if (args.step.enabled)
    inblock_rows_to_ws<float, D>(d, static_cast<const float*>(args.q), static_cast<const float*>(args.step.k_blk),
                                 static_cast<const float*>(args.step.v_blk), b, kvh, row0, ib0, ib1,
                                 args.inblock + unit * RT * (D + 4), warp, kThreads / 32, lane);

  const float* q = static_cast<const float*>(args.q) + ((size_t)(b * d.hq + kvh * d.G) * d.B + row0) * D;
  for (int i = tid; i < RT * D; i += kThreads) {
    const int r = i / D;
    sQ[r][i - r * D] = r < rows_valid ? q[i] : 0.f;
  }
  const float* kbase = static_cast<const float*>(args.k) + (size_t)bg * d.head_stride;
  const float* vbase = static_cast<const float*>(args.v) + (size_t)bg * d.head_stride;

  const long long key_begin = (long long)split * plan.tiles_per_split * KT;
  const long long key_end = min(d.N, key_begin + (long long)plan.tiles_per_split * KT);

  // Each warp owns rows warp*4 .. warp*4+3 of the tile.
  float m[4], l[4], acc[4][DC];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m[j] = -CUDART_INF_F;
    l[j] = 0.f;
#pragma unroll
    for (int t = 0; t < DC; ++t) acc[j][t] = 0.f;
  }

  for (long long k0 = key_begin; k0 < key_end; k0 += KT) {
    __syncthreads();
    for (int i = tid; i < KT * D; i += kThreads) {
      const int kk = i / D, dd = i - kk * D;
      const long long key = k0 + kk;
      const bool ok = key < key_end;
      sK[kk][dd] = ok ? kbase[key * d.row_stride + dd] : 0.f;
      sV[kk][dd] = ok ? vbase[key * d.row_stride + dd] : 0.f;
    }
    __syncthreads();
    const bool valid = (k0 + lane) < key_end;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = warp * 4 + j;
      if (r >= rows_valid) continue;  // warp-uniform
      float s = 0.f;
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) s = fmaf(sQ[r][dd], sK[lane][dd], s);
      s = valid ? s * d.scale : -CUDART_INF_F;
      const float mnew = fmaxf(m[j], warp_max(s));
      const float p = valid ? expf(s - mnew) : 0.f;
      const float alpha = (m[j] == -CUDART_INF_F) ? 0.f : expf(m[j] - mnew);
      l[j] = l[j] * alpha + warp_sum(p);
#pragma unroll
      for (int t = 0; t < DC; ++t) acc[j][t] *= alpha;
      for (int kk = 0; kk < KT; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
        for (int t = 0; t < DC; ++t) acc[j][t] = fmaf(pk, sV[kk][lane + 32 * t], acc[j][t]);
      }
      m[j] = mnew;
    }
  }

  const size_t rstride = (size_t)D + 4;
  float* part_base = args.partials + unit * (size_t)plan.splits * RT * rstride;
  float* mypart = part_base + (size_t)split * RT * rstride;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = warp * 4 + j;
    const bool has = l[j] > 0.f;
    const float inv = has ? 1.f / l[j] : 0.f;
#pragma unroll
    for (int t = 0; t < DC; ++t) mypart[(size_t)r * rstride + lane + 32 * t] = acc[j][t] * inv;
    if (lane == 0) mypart[(size_t)r * rstride + D] = has ? m[j] + logf(l[j]) : -CUDART_INF_F;
  }

  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(args.counters + unit, 1u);
    s_last = (prev == (unsigned)plan.splits - 1u);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  combine_splits(part_base, plan.splits, RT, D, rows_valid, s_flags, grow0, args.ep, tid, kThreads);
  if (args.step.enabled) {
    __syncthreads();  // the recomputed cache rows are written
    merge_tile_from_ws<D>(step_ep, grow0, rows_valid, args.inblock + unit * RT * (D + 4), tid, kThreads);
    if (!args.step.reuse_done)
      record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, s_M, args.step.dec_M, args.step.dec_reuse,
                       kvh == 0 && rt == 0, tid, kThreads);
  }
  if (tid == 0) args.counters[unit] = 0u;
}

}  // namespace

template <int DC>
cudaError_t launch_f32_dc(const PassArgs& a, cudaStream_t s) {
  const size_t smem = f32_smem_floats(32 * DC) * sizeof(float);
  auto kern = pass_f32_kernel<DC>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.plan.splits, a.plan.n_row_tiles, a.d.b * a.d.hkv);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_pass_f32(const PassArgs& a, cudaStream_t s) {
  switch (a.d.D / 32) {
    case 1: return launch_f32_dc<1>(a, s);
    case 2: return launch_f32_dc<2>(a, s);
    case 3: return launch_f32_dc<3>(a, s);
    case 4: return launch_f32_dc<4>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fb
