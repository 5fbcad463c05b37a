// reuse.cu -- the reusing rows of a denoising step, for many problems at once.
//
// FlashBlock technical summary (gist.science 2602.05305), "2. Methodology / Core
// mechanism": a row whose cache is reused gets A_full = merge(cached (A_out,
// L_out), fresh in-block (A_in, L_in)); the prefix K/V are not read.  "Adaptive
// reuse strategies": the row's head reuses iff the step is not the block's first,
// M^{s+1} < tau and (with a per-head gate) its similarity is above gamma.
//
// When one call carries many independent (b, KV head) groups -- the batch of a
// serving step, or every layer of a model stacked on the batch axis -- the pass
// kernel's one-CTA-per-SM shared-memory ring would hold a whole SM per reusing
// tile.  These kernels instead need no dynamic shared memory: the gate, the
// decision record (dec_M, dec_reuse), and for every reusing row the in-block
// attention merged with its cached row, in the same arithmetic as the pass kernels'
// fused epilogue, so the results agree bit for bit.  Rows that recompute are left to
// the prefix pass that follows.
//  * bf16 (reuse_tiles_kernel): a warp per 16-row tile of a group, the in-block
//    part on the tensor cores (inblock_rows_tc), two tiles per CTA and up to six CTAs
//    per SM (their tile memories fill shared memory); each warp starts
//    its tile's copies into its shared memory while it reads the gate, so one DRAM
//    latency covers the tile.
//  * fp32 (reuse_rows_kernel): a CTA per group, a warp per row on CUDA cores
//    (inblock_merge_row), three CTAs per SM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "fb_device.cuh"
#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kReuseThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kReuseThreads, 3) reuse_rows_kernel(const PassArgs args) {
  __shared__ int s_red[32];
  const Dims& d = args.d;
  const GateParams& g = args.gate;
  const int bg = blockIdx.x, b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B;
  {
    // Pull the group's rows into L1 while the gate reads the mask, so each row's
    // loads below hit L1 instead of paying a DRAM latency each: the q rows, the
    // cached rows (A and L) and the block's keys and values.  Every prefetched
    // address lies inside its buffer (a range's last byte covers its last line).
    const char* base[5] = {reinterpret_cast<const char*>(static_cast<const T*>(args.q) + grow0 * D),
                           reinterpret_cast<const char*>(args.ep.a_dst + grow0 * D),
                           reinterpret_cast<const char*>(args.ep.l_dst + grow0),
                           reinterpret_cast<const char*>(static_cast<const T*>(args.step.k_blk) + (size_t)bg * d.B * D),
                           reinterpret_cast<const char*>(static_cast<const T*>(args.step.v_blk) + (size_t)bg * d.B * D)};
    const size_t bytes[5] = {(size_t)d.R * D * sizeof(T), (size_t)d.R * D * 4, (size_t)d.R * 4,
                             (size_t)d.B * D * sizeof(T), (size_t)d.B * D * sizeof(T)};
#pragma unroll
    for (int t = 0; t < 5; ++t) {
      const int lines = (int)((bytes[t] + 127) / 128);
      for (int i = tid; i <= lines; i += kReuseThreads)
        prefetch_l1(base[t] + (i < lines ? (size_t)i * 128 : bytes[t] - 1));
    }
  }
  const int M = block_updated_count(g.mask + (size_t)b * d.B, d.B, s_red);
  const bool tau_ok = tau_reuse(g, M);
  if (kvh == 0 && tid == 0 && args.step.dec_M) args.step.dec_M[b] = M;
  if (args.step.dec_reuse)
    for (int j = tid; j < d.G; j += kReuseThreads) {
      const int h = kvh * d.G + j;
      args.step.dec_reuse[(size_t)b * d.hq + h] = head_reuse(g, tau_ok, b, d.hq, h) ? 1 : 0;
    }
  if (!tau_ok) return;  // every head of this batch element recomputes: the prefix pass writes its rows

  Epilogue ep;
  ep.mode = 1;
  ep.a_dst = nullptr;
  ep.l_dst = nullptr;
  ep.a_prev = args.ep.a_dst;  // the cache
  ep.l_prev = args.ep.l_dst;
  ep.a_full = args.step.a_full;
  ep.l_full = args.step.l_full;
  ep.out_bf16 = d.dtype == 1;
  const T* q = static_cast<const T*>(args.q);
  const T* kb = static_cast<const T*>(args.step.k_blk) + (size_t)bg * d.B * D;
  const T* vb = static_cast<const T*>(args.step.v_blk) + (size_t)bg * d.B * D;
  constexpr int kWarps = kReuseThreads / 32;
  for (int r = warp; r < d.R; r += kWarps) {
    if (!head_reuse(g, true, b, d.hq, kvh * d.G + r / d.B)) continue;  // warp-uniform
    inblock_merge_row<T, D>(d, q, kb, vb, grow0 + r, ep, lane);
  }
}

constexpr int kTileWarps = 2;

template <int D>
__global__ void __launch_bounds__(kTileWarps * 32, 6) reuse_tiles_kernel(const PassArgs args, long long items) {
  using bf16 = __nv_bfloat16;
  const Dims& d = args.d;
  const GateParams& g = args.gate;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (d.R + 15) >> 4;
  const long long item = (long long)blockIdx.x * kTileWarps + warp;
  if (item >= items) return;
  const int bg = (int)(item / tiles), t = (int)(item - (long long)bg * tiles);
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int r0 = t * 16, r1 = min(d.R, r0 + 16);
  Epilogue ep;
  ep.mode = 1;
  ep.a_dst = nullptr;
  ep.l_dst = nullptr;
  ep.a_prev = args.ep.a_dst;  // the cache
  ep.l_prev = args.ep.l_dst;
  ep.a_full = args.step.a_full;
  ep.l_full = args.step.l_full;
  ep.out_bf16 = 1;
  const TileOut out = tile_out_ep(ep);
  const bf16* q = static_cast<const bf16*>(args.q);
  const bf16* kb = static_cast<const bf16*>(args.step.k_blk);
  const bf16* vb = static_cast<const bf16*>(args.step.v_blk);
  extern __shared__ __align__(16) uint8_t tile_smem[];  // a tile memory per warp
  uint8_t* wsm = tile_smem + (size_t)warp * TileSmem<D>::bytes(d.B);
  // the tile's copies (query rows, block keys and values, cached rows) start while
  // the gate reads the mask
  inblock_rows_prestage<D>(d, q, kb, vb, b, kvh, r0, r1, out, 0, lane, wsm);
  int cnt = 0;
  for (int i = lane; i < d.B; i += 32) cnt += g.mask[(size_t)b * d.B + i] != 0;
  const int M = warp_sum_int(cnt);
  const bool tau_ok = tau_reuse(g, M);
  if (t == 0) {
    if (kvh == 0 && lane == 0 && args.step.dec_M) args.step.dec_M[b] = M;
    if (args.step.dec_reuse)
      for (int j = lane; j < d.G; j += 32)
        args.step.dec_reuse[(size_t)b * d.hq + kvh * d.G + j] = head_reuse(g, tau_ok, b, d.hq, kvh * d.G + j) ? 1 : 0;
  }
  if (!tau_ok) {  // every head of this batch element recomputes: the prefix pass writes its rows
    cp_async_wait_all();  // no copy may still be landing when the warp leaves
    return;
  }
  auto keep = [&](int r) { return head_reuse(g, true, b, d.hq, kvh * d.G + r / d.B); };
  inblock_rows_tc<D>(d, q, kb, vb, b, kvh, r0, r1, out, keep, 0, 1, lane, wsm, true);
}

template <typename T, int D>
cudaError_t launch_typed(const PassArgs& a, cudaStream_t s) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    const long long items = (long long)a.d.b * a.d.hkv * ((a.d.R + 15) / 16);
    const int smem = kTileWarps * TileSmem<D>::bytes(a.d.B);  // narrower for blocks of at most 8 keys
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      const cudaError_t e = cudaFuncSetAttribute(reuse_tiles_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kTileWarps * TileSmem<D>::kBytes);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    reuse_tiles_kernel<D><<<(unsigned)((items + kTileWarps - 1) / kTileWarps), kTileWarps * 32, smem, s>>>(a, items);
  } else {
    reuse_rows_kernel<T, D><<<(unsigned)(a.d.b * a.d.hkv), kReuseThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

int reuse_rows_supported(int dtype, int D) {
  return dtype == 1 ? (D == 64 || D == 128) : (D == 32 || D == 64 || D == 96 || D == 128);
}

cudaError_t launch_reuse_rows(const PassArgs& a, cudaStream_t s) {
  const int D = a.d.D;
  if (a.d.dtype == 1) {
    if (D == 128) return launch_typed<__nv_bfloat16, 128>(a, s);
    if (D == 64) return launch_typed<__nv_bfloat16, 64>(a, s);
  } else {
    if (D == 128) return launch_typed<float, 128>(a, s);
    if (D == 96) return launch_typed<float, 96>(a, s);
    if (D == 64) return launch_typed<float, 64>(a, s);
    if (D == 32) return launch_typed<float, 32>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fb
