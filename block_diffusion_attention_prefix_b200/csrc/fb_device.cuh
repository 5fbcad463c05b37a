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

#include <type_traits>

#include "fb_internal.h"
#include "fb_ptx.cuh"

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
                                              int* s_red, int* s_M = nullptr) {
  bool tau_ok = false;
  if (g.enabled) {
    const int M = block_updated_count(g.mask + (size_t)b * d.B, d.B, s_red);
    tau_ok = tau_reuse(g, M);
    if (s_M && threadIdx.x == 0) *s_M = M;
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

// The merge equation for one row, in the one rounding order every dense merge of
// the library uses (so a fused step and the separate calls agree bit for bit):
// m = max(L1, L2), w_i = e^{L_i - m}, A = (w1 A1 + w2 A2) / (w1 + w2),
// L = m + ln(w1 + w2).
struct MergeRow {
  float w1, w2, rden, l;
};
__device__ __forceinline__ MergeRow merge_row(float l1, float l2) {
  const float m = fmaxf(l1, l2);
  MergeRow w;
  w.w1 = m == -CUDART_INF_F ? 0.f : expf(l1 - m);
  w.w2 = m == -CUDART_INF_F ? 0.f : expf(l2 - m);
  const float den = w.w1 + w.w2;
  w.rden = den > 0.f ? 1.f / den : 0.f;
  w.l = den > 0.f ? m + logf(den) : -CUDART_INF_F;
  return w;
}
__device__ __forceinline__ float merge_val(const MergeRow& w, float a1, float a2) {
  return fmaf(w.w1, a1, w.w2 * a2) * w.rden;
}

// The merge equation on one float4 of a row: (A1, L1) and (A2, L2) -> (A, L).
__device__ __forceinline__ void merge4(float4 a1, float l1, float4 a2, float l2, float4& a, float& l) {
  const MergeRow w = merge_row(l1, l2);
  l = w.l;
  if (w.l == -CUDART_INF_F) {
    a = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  a = make_float4(merge_val(w, a1.x, a2.x), merge_val(w, a1.y, a2.y), merge_val(w, a1.z, a2.z),
                  merge_val(w, a1.w, a2.w));
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

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// Load DC consecutive elements as floats.
template <int DC>
__device__ __forceinline__ void load_vec(const float* p, float (&x)[DC]) {
  if constexpr (DC == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else if constexpr (DC == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x; x[1] = v.y;
  } else {
#pragma unroll
    for (int t = 0; t < DC; ++t) x[t] = p[t];
  }
}
template <int DC>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&x)[DC]) {
  if constexpr (DC == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = lo.x; x[1] = lo.y; x[2] = hi.x; x[3] = hi.y;
  } else if constexpr (DC == 2) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    x[0] = v.x; x[1] = v.y;
  } else {
#pragma unroll
    for (int t = 0; t < DC; ++t) x[t] = __bfloat162float(p[t]);
  }
}

// Store DC consecutive floats (as fp32, or rounded to bf16) with one vector store
// where the width allows (the caller's offset is DC-element aligned).
template <int DC>
__device__ __forceinline__ void store_vec(float* p, const float (&x)[DC]) {
  if constexpr (DC == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  } else if constexpr (DC == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  } else {
#pragma unroll
    for (int t = 0; t < DC; ++t) p[t] = x[t];
  }
}
template <int DC>
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&x)[DC]) {
  if constexpr (DC == 4) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]), hi = __floats2bfloat162_rn(x[2], x[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
  } else if constexpr (DC == 2) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x[0], x[1]);
  } else {
#pragma unroll
    for (int t = 0; t < DC; ++t) p[t] = __float2bfloat16_rn(x[t]);
  }
}

// In-block attention of one query row by one warp (FlashBlock "Core mechanism":
// A_in over J_in, the B tokens of the current block, bidirectional; fp32 math).
// Lane l owns dims [l*DC, l*DC + DC).  Keys go in chunks of KC whose dot products
// are reduced across the warp together (independent butterflies), with an online
// softmax across chunks.  Returns L_in (natural log); `a` gets the lane's dims of
// the normalised A_in.  `kb` / `vb` point at the KV group's [B][D] block keys.
template <typename T, int D, int KC>
__device__ __forceinline__ float inblock_row_kc(const T* qrow, const T* kb, const T* vb, int B, float scale,
                                                float (&a)[D / 32], int lane) {
  constexpr int DC = D / 32;
  float q[DC];
  load_vec<DC>(qrow + lane * DC, q);
  float m = -CUDART_INF_F, l = 0.f, acc[DC];
#pragma unroll
  for (int t = 0; t < DC; ++t) acc[t] = 0.f;
  for (int j0 = 0; j0 < B; j0 += KC) {
    const int nj = min(KC, B - j0);
    float s[KC], v[KC][DC];
#pragma unroll
    for (int jj = 0; jj < KC; ++jj) {
      s[jj] = 0.f;
#pragma unroll
      for (int t = 0; t < DC; ++t) v[jj][t] = 0.f;
      if (jj < nj) {
        float k[DC];
        load_vec<DC>(kb + (size_t)(j0 + jj) * D + lane * DC, k);
        load_vec<DC>(vb + (size_t)(j0 + jj) * D + lane * DC, v[jj]);
#pragma unroll
        for (int t = 0; t < DC; ++t) s[jj] = fmaf(q[t], k[t], s[jj]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int jj = 0; jj < KC; ++jj) s[jj] += __shfl_xor_sync(0xffffffffu, s[jj], o);
    }
    float cm = -CUDART_INF_F;
#pragma unroll
    for (int jj = 0; jj < KC; ++jj) {
      s[jj] = jj < nj ? s[jj] * scale : -CUDART_INF_F;
      cm = fmaxf(cm, s[jj]);
    }
    const float mn = fmaxf(m, cm);
    const float alpha = m == -CUDART_INF_F ? 0.f : expf(m - mn);
    l *= alpha;
#pragma unroll
    for (int t = 0; t < DC; ++t) acc[t] *= alpha;
#pragma unroll
    for (int jj = 0; jj < KC; ++jj) {
      const float p = jj < nj ? expf(s[jj] - mn) : 0.f;
      l += p;
#pragma unroll
      for (int t = 0; t < DC; ++t) acc[t] = fmaf(p, v[jj][t], acc[t]);
    }
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int t = 0; t < DC; ++t) a[t] = acc[t] * inv;
  return m + logf(l);
}

// In-block row with chunks of 8 keys.  Blocks of at most 4 keys take chunks of 4:
// the same result bit for bit (a chunk's unused key slots add exact zeros to the
// row sum and the accumulators, and -inf to the chunk max), with half the shuffles.
template <typename T, int D>
__device__ __forceinline__ float inblock_row(const T* qrow, const T* kb, const T* vb, int B, float scale,
                                             float (&a)[D / 32], int lane) {
  if (B <= 4) return inblock_row_kc<T, D, 4>(qrow, kb, vb, B, scale, a, lane);
  return inblock_row_kc<T, D, 8>(qrow, kb, vb, B, scale, a, lane);
}

// ---------------------------------------------------------------------------
// In-block attention on the tensor cores (bf16): 16 query rows of one KV group by
// one warp.  FlashBlock "Core mechanism": (A_in, L_in) over J_in, the B tokens of
// the current block, bidirectional.  The operands are staged in the warp's own
// shared memory with coalesced 16-byte async copies (one pass over the 16 query
// rows, then the keys and values 16 at a time), and mma.sync m16n8k16 (bf16
// operands, fp32 accumulation) reads them with ldmatrix:
//   S = Q K^T over D in k16 steps, keys in chunks of 16 (two n8 tiles);
//   online softmax across the chunks in fp32, base 2 (scale * log2 e folded in),
//   keys past B masked; the running max m, sum l and the output are rescaled by
//   2^(m_old - m_new) when a chunk raises the max;
//   O += P V with P split into bf16 hi and lo parts (P = hi + lo to about 2^-17),
//   two products per step, so the rounding of P to bf16 costs no accuracy;
//   A_in = O / l, L_in = (m + log2 l) ln 2.
// Each row's result depends only on that row's query and the block's keys and
// values (the MMA computes each output element the same way for every row, and the
// row reductions run inside the row's thread quad), so every caller that covers a
// row with any 16-row tile gets the same bits.
// Output, accumulator layout: thread (g = lane / 4, c = lane % 4) holds for d-tile n
// o[n][0..1] = A_in[row g][8n + 2c, +1] and o[n][2..3] = the same of row g + 8, and
// L[0] / L[1] = L_in of rows g / g + 8 (tile rows).

// One warp's shared memory for in-block tiles: 16 staged query rows, the keys and
// values of one chunk (16 rows, or 8 when the block has at most 8 keys; bf16 rows
// padded to D + 8 elements: 16-byte aligned, ldmatrix without bank conflicts) and 16
// cached rows of D + 4 floats (the merge of mode 1).  kBytes / kOperandBytes are the
// sizes for any block (16-row chunks); bytes(B) / operand_bytes(B) for a given B.
template <int D>
struct TileSmem {
  static constexpr int kRow = D + 8;  // bf16 elements per staged row
  static constexpr int kQBytes = 16 * kRow * 2;
  __host__ __device__ static constexpr int kv_rows(int B) { return B <= 8 ? 8 : 16; }
  __host__ __device__ static constexpr int k_off(int) { return kQBytes; }
  __host__ __device__ static constexpr int v_off(int B) { return kQBytes + kv_rows(B) * kRow * 2; }
  __host__ __device__ static constexpr int cache_off(int B) { return kQBytes + 2 * kv_rows(B) * kRow * 2; }
  __host__ __device__ static constexpr int operand_bytes(int B) { return cache_off(B); }
  __host__ __device__ static constexpr int bytes(int B) { return cache_off(B) + 16 * (D + 4) * 4; }
  static constexpr int kBytes = bytes(64);
  static constexpr int kOperandBytes = operand_bytes(64);  // enough for callers that merge nothing
  static_assert(kBytes % 16 == 0 && kOperandBytes % 16 == 0 && bytes(1) % 16 == 0, "16-byte aligned regions");
};

// `rows` rows [row0, row0 + rows) of a [n][D] bf16 array into a staged [rows][D + 8]
// tile; rows >= n are zero-filled.  Asynchronous (cp.async); the caller waits.
template <int D>
__device__ __forceinline__ void stage_rows(__nv_bfloat16* dst, const __nv_bfloat16* src, int row0, int n, int rows,
                                           int lane) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  for (int i = lane; i < rows * kChunks; i += 32) {
    const int r = i / kChunks, c = i - r * kChunks;
    const bool valid = row0 + r < n;
    const __nv_bfloat16* g = src + (size_t)(valid ? row0 + r : 0) * D + c * 8;
    cp_async16_zfill(dst + r * TileSmem<D>::kRow + c * 8, g, valid);
  }
}

// The first copies of a tile: its 16 query rows and the block's first 16 keys and
// values, into the warp's tile memory (asynchronous).
template <int D>
__device__ __forceinline__ void inblock_tile_stage(const __nv_bfloat16* q, int R, int row0, const __nv_bfloat16* kb,
                                                   const __nv_bfloat16* vb, int B, int lane, uint8_t* wsm) {
  using TS = TileSmem<D>;
  const int kvr = TS::kv_rows(B);
  __syncwarp();  // the warp's previous reads of its tile memory are done
  stage_rows<D>(reinterpret_cast<__nv_bfloat16*>(wsm), q, row0, R, 16, lane);
  stage_rows<D>(reinterpret_cast<__nv_bfloat16*>(wsm + TS::k_off(B)), kb, 0, B, kvr, lane);
  stage_rows<D>(reinterpret_cast<__nv_bfloat16*>(wsm + TS::v_off(B)), vb, 0, B, kvr, lane);
}

// `staged`: inblock_tile_stage already ran for this tile (same arguments).
template <int D>
__device__ __forceinline__ void inblock_tile_tc(const __nv_bfloat16* q, int R, int row0, const __nv_bfloat16* kb,
                                                const __nv_bfloat16* vb, int B, float scale, float (&o)[D / 8][4],
                                                float (&L)[2], int lane, uint8_t* wsm, bool staged = false) {
  using TS = TileSmem<D>;
  const bool narrow = TS::kv_rows(B) == 8;  // at most 8 keys: one n8 tile of scores, 8 value rows
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(wsm);
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(wsm + TS::k_off(B));
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(wsm + TS::v_off(B));
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
  const int c = lane & 3;
  if (!staged) inblock_tile_stage<D>(q, R, row0, kb, vb, B, lane, wsm);
  const float sl2 = scale * 1.4426950408889634f;
  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  uint32_t qf[D / 16][4];
  for (int k0 = 0; k0 < B; k0 += 16) {
    if (k0 > 0) {  // the first chunk came with the query rows (chunks past it: 16 rows)
      __syncwarp();  // the previous chunk's reads of sK / sV are done
      stage_rows<D>(sK, kb, k0, B, 16, lane);
      stage_rows<D>(sV, vb, k0, B, 16, lane);
    }
    cp_async_wait_all();
    __syncwarp();
    if (k0 == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(aQ + (uint32_t)(((lane & 15) * TS::kRow + kk * 16 + (lane >> 4) * 8) * 2), qf[kk][0], qf[kk][1],
                qf[kk][2], qf[kk][3]);
    }
    // S for this chunk's 16 keys (n-tiles 0: keys k0..k0+7, 1: k0+8..k0+15).  With at
    // most 8 keys the second n-tile is all masked and is not computed (its scores are
    // -inf either way; the skipped products are exact zeros in the sums).
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int key = (lane & 7) + ((lane >> 4) << 3);
      const int col = kk * 16 + ((lane >> 3) & 1) * 8;
      if (narrow) {
        uint32_t b0, b1;
        ldsm_x2(aK + (uint32_t)(((lane & 7) * TS::kRow + col) * 2), b0, b1);
        mma_bf16_16816_free(s[0], qf[kk], b0, b1);
      } else {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(aK + (uint32_t)((key * TS::kRow + col) * 2), b0, b1, b2, b3);
        mma_bf16_16816_free(s[0], qf[kk], b0, b1);
        mma_bf16_16816_free(s[1], qf[kk], b2, b3);
      }
    }
    float cm0 = -CUDART_INF_F, cm1 = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + j * 8 + 2 * c + (e & 1);
        const float v = key < B ? s[j][e] * sl2 : -CUDART_INF_F;
        s[j][e] = v;
        if (e < 2) cm0 = fmaxf(cm0, v); else cm1 = fmaxf(cm1, v);
      }
    }
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 1));
    cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, 2));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 1));
    cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, 2));
    const float n0 = fmaxf(m0, cm0), n1 = fmaxf(m1, cm1);  // every chunk has a valid key: finite
    const float al0 = ex2_approx(m0 - n0), al1 = ex2_approx(m1 - n1);  // 0 on the first chunk
    float cs0 = 0.f, cs1 = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      s[j][0] = ex2_approx(s[j][0] - n0);
      s[j][1] = ex2_approx(s[j][1] - n0);
      s[j][2] = ex2_approx(s[j][2] - n1);
      s[j][3] = ex2_approx(s[j][3] - n1);
      cs0 += s[j][0] + s[j][1];
      cs1 += s[j][2] + s[j][3];
    }
    cs0 += __shfl_xor_sync(0xffffffffu, cs0, 1);
    cs0 += __shfl_xor_sync(0xffffffffu, cs0, 2);
    cs1 += __shfl_xor_sync(0xffffffffu, cs1, 1);
    cs1 += __shfl_xor_sync(0xffffffffu, cs1, 2);
    l0 = l0 * al0 + cs0;
    l1 = l1 * al1 + cs1;
    m0 = n0;
    m1 = n1;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= al0;
      o[n][1] *= al0;
      o[n][2] *= al1;
      o[n][3] *= al1;
    }
    // O += P V, P = hi + lo in bf16
    uint32_t hi[4], lo[4];
    {
      const float pv[8] = {s[0][0], s[0][1], s[0][2], s[0][3], s[1][0], s[1][1], s[1][2], s[1][3]};
      float rest[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) rest[e] = pv[e] - __bfloat162float(__float2bfloat16_rn(pv[e]));
      hi[0] = pack_bf16x2(pv[0], pv[1]);
      hi[1] = pack_bf16x2(pv[2], pv[3]);
      hi[2] = pack_bf16x2(pv[4], pv[5]);
      hi[3] = pack_bf16x2(pv[6], pv[7]);
      lo[0] = pack_bf16x2(rest[0], rest[1]);
      lo[1] = pack_bf16x2(rest[2], rest[3]);
      lo[2] = pack_bf16x2(rest[4], rest[5]);
      lo[3] = pack_bf16x2(rest[6], rest[7]);
    }
#pragma unroll
    for (int dn = 0; dn < D / 8; dn += 2) {
      uint32_t b0, b1 = 0u, b2, b3 = 0u;  // with at most 8 keys, value rows 8..15 are zero
      if (narrow) {
        ldsm_x2_t(aV + (uint32_t)(((lane & 7) * TS::kRow + dn * 8 + ((lane >> 3) & 1) * 8) * 2), b0, b2);
      } else {
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = dn * 8 + (lane >> 4) * 8;
        ldsm_x4_t(aV + (uint32_t)((key * TS::kRow + col) * 2), b0, b1, b2, b3);
      }
      mma_bf16_16816_free(o[dn], hi, b0, b1);
      mma_bf16_16816_free(o[dn], lo, b0, b1);
      mma_bf16_16816_free(o[dn + 1], hi, b2, b3);
      mma_bf16_16816_free(o[dn + 1], lo, b2, b3);
    }
  }
  const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    o[n][0] *= i0;
    o[n][1] *= i0;
    o[n][2] *= i1;
    o[n][3] *= i1;
  }
  L[0] = (m0 + __log2f(l0)) * 0.6931471805599453f;
  L[1] = (m1 + __log2f(l1)) * 0.6931471805599453f;
}

// The in-block rows [r_begin, r_end) of KV group (b, kvh) (group rows, 0 .. G*B),
// computed on the tensor cores in 16-row tiles by warps [warp, nwarps); for each
// tile row r that `keep(r)` accepts, the threads holding it write their columns.
// `wsm`: this warp's TileSmem<D>::kBytes of shared memory (16-byte aligned).  In
// mode 1 the tile's cached rows are copied there asynchronously while the tile is
// computed.  Modes:
//   to_ws: (A_in, L_in) into slot rows r - slot_row0 ([.][D + 4] fp32, L at col D);
//   ep mode 0: (A_in, L_in) into ep.a_dst / ep.l_dst;
//   ep mode 1: A_full = merge(cache row, in-block row) into ep.a_full / ep.l_full.
struct TileOut {
  int kind;            // 0: workspace slot, 1: epilogue
  float* slot;         // kind 0
  int slot_row0;       // kind 0: group row of slot row 0
  Epilogue ep;         // kind 1
};

// The copies inblock_rows_tc makes first for this warp's first tile (query rows, the
// first 16 keys and values, and in mode 1 the cached rows), issued ahead -- e.g. while
// the gate is still being read; the matching call then passes prestaged = true.
template <int D>
__device__ void inblock_rows_prestage(const Dims& d, const __nv_bfloat16* q, const __nv_bfloat16* k_blk,
                                      const __nv_bfloat16* v_blk, int b, int kvh, int r_begin, int r_end,
                                      const TileOut& out, int warp, int lane, uint8_t* wsm) {
  using TS = TileSmem<D>;
  const int t0 = r_begin + warp * 16;
  if (t0 >= r_end) return;
  const size_t grow_base = (size_t)(b * d.hq + kvh * d.G) * d.B;
  if (out.kind == 1 && out.ep.mode == 1) {
    float* sC = reinterpret_cast<float*>(wsm + TS::cache_off(d.B));
    const int nr = min(16, r_end - t0);
    for (int i = lane; i < nr * (D / 4); i += 32) {
      const int rr = i / (D / 4), c4 = i - rr * (D / 4);
      cp_async16(sC + rr * (D + 4) + c4 * 4, out.ep.a_prev + (grow_base + t0 + rr) * D + c4 * 4);
    }
    for (int rr = lane; rr < nr; rr += 32) cp_async4(sC + rr * (D + 4) + D, out.ep.l_prev + grow_base + t0 + rr);
  }
  inblock_tile_stage<D>(q + grow_base * D, min(r_end, d.R), t0, k_blk + (size_t)(b * d.hkv + kvh) * d.B * D,
                        v_blk + (size_t)(b * d.hkv + kvh) * d.B * D, d.B, lane, wsm);
}

template <int D, typename Keep>
__device__ void inblock_rows_tc(const Dims& d, const __nv_bfloat16* q, const __nv_bfloat16* k_blk,
                                const __nv_bfloat16* v_blk, int b, int kvh, int r_begin, int r_end,
                                const TileOut& out, Keep keep, int warp, int nwarps, int lane, uint8_t* wsm,
                                bool prestaged = false) {
  using TS = TileSmem<D>;
  const __nv_bfloat16* kb = k_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const __nv_bfloat16* vb = v_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const size_t grow_base = (size_t)(b * d.hq + kvh * d.G) * d.B;  // global row of group row 0
  const __nv_bfloat16* qg = q + grow_base * D;
  float* sC = reinterpret_cast<float*>(wsm + TS::cache_off(d.B));
  const int g = lane >> 2, c = lane & 3;
  for (int t0 = r_begin + warp * 16; t0 < r_end; t0 += nwarps * 16) {
    const bool merge = out.kind == 1 && out.ep.mode == 1;
    const bool pre = prestaged && t0 == r_begin + warp * 16;
    if (merge && !pre) {
      // the tile's cached rows are needed after the in-block math: copy them now
      __syncwarp();  // the previous tile's reads of sC are done
      const int nr = min(16, r_end - t0);
      for (int i = lane; i < nr * (D / 4); i += 32) {
        const int rr = i / (D / 4), c4 = i - rr * (D / 4);
        cp_async16(sC + rr * (D + 4) + c4 * 4, out.ep.a_prev + (grow_base + t0 + rr) * D + c4 * 4);
      }
      for (int rr = lane; rr < nr; rr += 32) cp_async4(sC + rr * (D + 4) + D, out.ep.l_prev + grow_base + t0 + rr);
    }
    float o[D / 8][4], L[2];
    inblock_tile_tc<D>(qg, min(r_end, d.R), t0, kb, vb, d.B, d.scale, o, L, lane, wsm, pre);
    if (merge) {
      cp_async_wait_all();
      __syncwarp();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = t0 + g + 8 * h;
      if (r >= r_end || !keep(r)) continue;
      const size_t grow = grow_base + r;
      if (out.kind == 0) {
        float* dst = out.slot + (size_t)(r - out.slot_row0) * (D + 4);
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
          *reinterpret_cast<float2*>(dst + n * 8 + 2 * c) = make_float2(o[n][2 * h], o[n][2 * h + 1]);
        if (c == 0) dst[D] = L[h];
      } else if (out.ep.mode == 0) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
          *reinterpret_cast<float2*>(out.ep.a_dst + grow * D + n * 8 + 2 * c) =
              make_float2(o[n][2 * h], o[n][2 * h + 1]);
        if (c == 0) out.ep.l_dst[grow] = L[h];
      } else {
        const float* srow = sC + (r - t0) * (D + 4);
        const MergeRow w = merge_row(srow[D], L[h]);
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const size_t off = grow * D + n * 8 + 2 * c;
          const float2 ap = *reinterpret_cast<const float2*>(srow + n * 8 + 2 * c);
          const float v0 = merge_val(w, ap.x, o[n][2 * h]), v1 = merge_val(w, ap.y, o[n][2 * h + 1]);
          if (out.ep.out_bf16)
            *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out.ep.a_full) + off) =
                __floats2bfloat162_rn(v0, v1);
          else
            *reinterpret_cast<float2*>(static_cast<float*>(out.ep.a_full) + off) = make_float2(v0, v1);
        }
        if (c == 0 && out.ep.l_full) out.ep.l_full[grow] = w.l;
      }
    }
  }
}

__device__ __forceinline__ TileOut tile_out_ep(const Epilogue& ep) {
  TileOut out;
  out.kind = 1;
  out.slot = nullptr;
  out.slot_row0 = 0;
  out.ep = ep;
  return out;
}

struct KeepAll {
  __device__ bool operator()(int) const { return true; }
};

// One in-block row of a step, by one warp: A_full = merge(cache row, in-block
// row) (mode 1), or (A_in, L_in) written out (mode 0).  `grow` indexes [b, H_q, B];
// `kb` / `vb` are the KV group's [B][D] block keys and values.  In mode 1 the cache
// row is loaded before the in-block math so the two latencies overlap.  Every
// mode-1 caller reads a cache that an earlier launch wrote and that no CTA of its
// own launch writes (a reusing row's cache is left alone), so the cache is read
// through the read-only L1 path.
template <typename T, int D>
__device__ __forceinline__ void inblock_merge_row(const Dims& d, const T* q, const T* kb, const T* vb, size_t grow,
                                                  const Epilogue& ep, int lane) {
  constexpr int DC = D / 32;
  float ap[DC], lp = 0.f;
  if (ep.mode == 1) {
    lp = __ldg(ep.l_prev + grow);
#pragma unroll
    for (int t = 0; t < DC; ++t) ap[t] = __ldg(ep.a_prev + grow * D + lane * DC + t);
  }
  float a[DC];
  const float L = inblock_row<T, D>(q + grow * D, kb, vb, d.B, d.scale, a, lane);
  const size_t off = grow * D + (size_t)lane * DC;
  if (ep.mode == 0) {
    store_vec<DC>(ep.a_dst + off, a);
    if (lane == 0) ep.l_dst[grow] = L;
    return;
  }
  const MergeRow w = merge_row(lp, L);
  float o[DC];
#pragma unroll
  for (int t = 0; t < DC; ++t) o[t] = merge_val(w, ap[t], a[t]);
  if (ep.out_bf16)
    store_vec<DC>(static_cast<__nv_bfloat16*>(ep.a_full) + off, o);
  else
    store_vec<DC>(static_cast<float*>(ep.a_full) + off, o);
  if (lane == 0 && ep.l_full) ep.l_full[grow] = w.l;
}

// In-block rows [r_begin, r_end) of tile rows (group rows row0 + r) of KV group
// (b, kvh), one warp per row (inblock_merge_row), executed by warps [0, nwarps) of
// the CTA.
// `tsm` (bf16 only): shared memory of TileSmem<D>::kBytes per warp (warp w uses
// tsm + w * TileSmem<D>::kBytes) for the tensor-core tiles.
template <typename T, int D>
__device__ void inblock_rows(const Dims& d, const T* q, const T* k_blk, const T* v_blk, int b, int kvh,
                             int row0, int r_begin, int r_end, const Epilogue& ep, int warp, int nwarps,
                             int lane, uint8_t* tsm = nullptr, bool prestaged = false) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {  // bf16: tensor-core tiles
    TileOut out;
    out.kind = 1;
    out.slot = nullptr;
    out.slot_row0 = 0;
    out.ep = ep;
    inblock_rows_tc<D>(d, q, k_blk, v_blk, b, kvh, row0 + r_begin, row0 + r_end, out, KeepAll(), warp, nwarps,
                       lane, tsm + (size_t)warp * TileSmem<D>::kBytes, prestaged);
    return;
  }
  const T* kb = k_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const T* vb = v_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  for (int r = r_begin + warp; r < r_end; r += nwarps) inblock_merge_row<T, D>(d, q, kb, vb, grow0 + r, ep, lane);
}

// In-block rows [r_begin, r_end) of one tile written as (A_in, L_in) into the
// tile's [RT][D + 4] fp32 slot of the workspace (the fused step merges them later).
// `tsm` as for inblock_rows.
template <typename T, int D>
__device__ void inblock_rows_to_ws(const Dims& d, const T* q, const T* k_blk, const T* v_blk, int b, int kvh,
                                   int row0, int r_begin, int r_end, float* slot, int warp, int nwarps,
                                   int lane, uint8_t* tsm = nullptr) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {  // bf16: tensor-core tiles
    TileOut out;
    out.kind = 0;
    out.slot = slot;
    out.slot_row0 = row0;
    inblock_rows_tc<D>(d, q, k_blk, v_blk, b, kvh, row0 + r_begin, row0 + r_end, out, KeepAll(), warp, nwarps,
                       lane, tsm + (size_t)warp * TileSmem<D>::kBytes);
    return;
  }
  constexpr int DC = D / 32;
  const T* kb = k_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const T* vb = v_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  for (int r = r_begin + warp; r < r_end; r += nwarps) {
    float a[DC];
    const float L = inblock_row<T, D>(q + (grow0 + r) * D, kb, vb, d.B, d.scale, a, lane);
    float* dst = slot + (size_t)r * (D + 4);
#pragma unroll
    for (int t = 0; t < DC; ++t) dst[lane * DC + t] = a[t];
    if (lane == 0) dst[D] = L;
  }
}

// Fused-step merge of a finished tile: A_full = merge(cache row, in-block row) for
// rows [0, rows_valid), reading the cache (possibly just written by this CTA) and
// the in-block slot with L2-coherent loads.  Threads [0, nthr).
template <int D>
__device__ void merge_tile_from_ws(const Epilogue& ep, size_t grow0, int rows_valid, const float* slot, int tid,
                                   int nthr) {
  constexpr int D4 = D / 4;
  for (int idx = tid; idx < rows_valid * D4; idx += nthr) {
    const int r = idx / D4, d4 = idx - r * D4;
    const size_t grow = grow0 + r;
    const size_t off = grow * D + (size_t)d4 * 4;
    const float4 ap = __ldcg(reinterpret_cast<const float4*>(ep.a_prev + off));
    const float lp = __ldcg(ep.l_prev + grow);
    const float4 ai = __ldcg(reinterpret_cast<const float4*>(slot + (size_t)r * (D + 4)) + d4);
    const float li = __ldcg(slot + (size_t)r * (D + 4) + D);
    float4 af;
    float lf;
    merge4(ap, lp, ai, li, af, lf);
    store4(ep.a_full, off, af, ep.out_bf16);
    if (d4 == 0 && ep.l_full) ep.l_full[grow] = lf;
  }
}

// Rows [r0, r1) of a tile assigned to split `split` for the in-block pass.
__device__ __forceinline__ void split_rows(int rows_valid, int splits, int split, int& r0, int& r1) {
  const int per = (rows_valid + splits - 1) / splits;
  r0 = min(rows_valid, split * per);
  r1 = min(rows_valid, r0 + per);
}

__device__ __forceinline__ Epilogue step_epilogue(const PassArgs& args) {
  Epilogue ep;
  ep.mode = 1;
  ep.a_dst = nullptr;
  ep.l_dst = nullptr;
  ep.a_prev = args.ep.a_dst;
  ep.l_prev = args.ep.l_dst;
  ep.a_full = args.step.a_full;
  ep.l_full = args.step.l_full;
  ep.out_bf16 = 1;
  return ep;
}

// Record the gate's decisions for the rows of one tile: dec_reuse[b, h] for every
// head with a row in the tile, and dec_M[b] when `write_M`.
__device__ __forceinline__ void record_decisions(const GateParams& g, const Dims& d, int b, int kvh, int row0,
                                                 int nrows, const int* s_flags, int M, int32_t* dec_M,
                                                 uint8_t* dec_reuse, bool write_M, int tid, int nthr) {
  if (!g.enabled) return;
  if (dec_reuse) {
    for (int r = tid; r < nrows; r += nthr) {
      const int gr = row0 + r;
      if (r == 0 || gr % d.B == 0) {
        const int h = kvh * d.G + gr / d.B;
        dec_reuse[(size_t)b * d.hq + h] = s_flags[r] ? 0 : 1;
      }
    }
  }
  if (write_M && dec_M && tid == 0) dec_M[b] = M;
}

// Split-KV combine spread over the split CTAs of one (b, kv head, row tile)
// (`unit`).  Called by the threads [0, NT) of every split CTA once its partial
// ([RT][D + 4] fp32, A normalised, natural-log L) and its share of the in-block
// rows are in the workspace.  The launch is cooperative -- every CTA of the grid
// is resident -- so a CTA may wait for the other splits of its tile:
//   1. arrive on arrive[0] (release); wait (acquire, bounded) until all `splits`
//      CTAs have arrived; depart on depart[0] -- the last to depart resets both
//      counters for the next launch;
//   2. bring rows [r0, r1) of every split's partial (the rows whose in-block part
//      this CTA computed), and those in-block rows, into shared memory with one
//      1-D bulk copy per split;
//   3. per row (one warp): M = max_s L_s, e_s = e^{L_s - M}, den = sum_s e_s (a
//      fixed warp tree), L = M + ln den -- the FlashBlock merge equation over all
//      splits; per item sum_s e_s A_s in split order, times 1/den.  The order is
//      fixed, so the result does not depend on timing;
//   4. epilogue: rows flagged for recompute go through `ep`; in a fused step
//      (`step_ep`) A_full = merge(cache row, in-block row), the cache row being the
//      one just combined (flagged rows) or the cached one (rows of reusing heads).
// `sbuf` (1024-byte aligned, `sbuf_bytes`) is idle shared memory; `mbar` an
// initialised mbarrier (count 1) whose phases this function alone uses, next
// parity `*phase`; barrier `bar_id` over NT threads.
template <int D, int NT>
__device__ void coop_finish_rows(const float* part, int splits, int RT, int r0, int r1, const float* inblock_slot,
                                 const int* s_flags, size_t grow0, const Epilogue& ep, const Epilogue* step_ep,
                                 uint8_t* sbuf, int sbuf_bytes, uint64_t* mbar, uint32_t* phase,
                                 unsigned int* arrive, unsigned int* depart, uint32_t* err, int tid, int bar_id) {
  constexpr int RS = D + 4;
  constexpr int D4 = D / 4;
  constexpr int NW = NT / 32;
  const int n = r1 - r0 > 0 ? r1 - r0 : 0;
  const bool step = step_ep != nullptr;
  // Shared layout: [splits][n][RS] partial rows | [n][RS] in-block rows | [n][splits] e_s | 5 x [n] row scalars.
  const size_t a_floats = (size_t)splits * n * RS;
  const size_t in_floats = step ? (size_t)n * RS : 0;
  float* sA = reinterpret_cast<float*>(sbuf);
  float* sIn = sA + a_floats;
  float* sE = sIn + in_floats;
  float* sL = sE + (size_t)n * splits;
  float* sInv = sL + n;
  float* sWo = sInv + n;  // fused step: the merge of the cache row with the in-block row
  float* sWi = sWo + n;
  float* sWr = sWi + n;
  const bool staged = (a_floats + in_floats + (size_t)n * splits + 5 * (size_t)n) * 4 <= (size_t)sbuf_bytes;
  fence_proxy_async_smem();         // generic writes to `sbuf` before the bulk copies land there
  named_barrier_sync(bar_id, NT);  // this CTA's partial and in-block rows are written
  bool ok = true;
  unsigned int dep = 0;
  if (tid == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
    ok = wait_count_bounded(arrive, (unsigned)splits, err, DEV_ERR_WAIT_PEERS);
    dep = atomicAdd(depart, 1u);  // result checked at the end
    if (ok && staged && n > 0) {
      fence_proxy_async_global();  // the partials were written through the generic proxy
      const uint32_t row_bytes = (uint32_t)n * RS * 4;
      mbar_arrive_expect_tx(mbar, row_bytes * (uint32_t)(splits + (step ? 1 : 0)));
      for (int sp = 0; sp < splits; ++sp)
        bulk_load(sA + (size_t)sp * n * RS, part + ((size_t)sp * RT + r0) * RS, row_bytes, mbar);
      if (step) bulk_load(sIn, inblock_slot + (size_t)r0 * RS, row_bytes, mbar);
    }
  }
  ok = named_barrier_and(bar_id, NT, ok);
  if (ok && n > 0) {
    if (staged) {
      ok = mbar_wait_bounded(mbar, *phase, err, DEV_ERR_WAIT_COMBINE);
      *phase ^= 1u;
    }
    ok = named_barrier_and(bar_id, NT, ok);
    // Source rows: shared memory when staged, else the workspace itself (L2).
    auto ld1 = [&](int sp, int rr) -> float {
      return staged ? sA[((size_t)sp * n + rr) * RS + D] : __ldcg(part + ((size_t)sp * RT + r0 + rr) * RS + D);
    };
    auto ld4 = [&](int sp, int rr, int d4) -> float4 {
      return staged ? reinterpret_cast<const float4*>(sA + ((size_t)sp * n + rr) * RS)[d4]
                    : __ldcg(reinterpret_cast<const float4*>(part + ((size_t)sp * RT + r0 + rr) * RS) + d4);
    };
    auto in1 = [&](int rr) -> float {
      return staged ? sIn[(size_t)rr * RS + D] : __ldcg(inblock_slot + (size_t)(r0 + rr) * RS + D);
    };
    auto in4 = [&](int rr, int d4) -> float4 {
      return staged ? reinterpret_cast<const float4*>(sIn + (size_t)rr * RS)[d4]
                    : __ldcg(reinterpret_cast<const float4*>(inblock_slot + (size_t)(r0 + rr) * RS) + d4);
    };
    const int warp = tid >> 5, lane = tid & 31;
    for (int rr = warp; rr < n && ok; rr += NW) {
      float M = -CUDART_INF_F;
      for (int sp = lane; sp < splits; sp += 32) M = fmaxf(M, ld1(sp, rr));
      M = warp_max(M);
      float den = 0.f;
      for (int sp = lane; sp < splits; sp += 32) {
        const float e = M == -CUDART_INF_F ? 0.f : expf(ld1(sp, rr) - M);
        sE[(size_t)rr * splits + sp] = e;
        den += e;
      }
      den = warp_sum(den);
      if (lane == 0) {
        const int r = r0 + rr;
        const float L = den > 0.f ? M + logf(den) : -CUDART_INF_F;
        sL[rr] = L;
        sInv[rr] = den > 0.f ? 1.f / den : 0.f;
        if (step) {
          const float lo = s_flags[r] ? L : __ldcg(step_ep->l_prev + grow0 + r);
          const MergeRow w = merge_row(lo, in1(rr));
          if (step_ep->l_full) step_ep->l_full[grow0 + r] = w.l;
          sWo[rr] = w.w1;
          sWi[rr] = w.w2;
          sWr[rr] = w.rden;
        }
      }
    }
    named_barrier_sync(bar_id, NT);
    for (int idx = tid; idx < n * D4 && ok; idx += NT) {
      const int rr = idx / D4, d4 = idx - rr * D4;
      const int r = r0 + rr;
      const float* er = sE + (size_t)rr * splits;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < splits; ++sp) {
        const float w = er[sp];
        const float4 x = ld4(sp, rr, d4);
        a.x = fmaf(w, x.x, a.x);
        a.y = fmaf(w, x.y, a.y);
        a.z = fmaf(w, x.z, a.z);
        a.w = fmaf(w, x.w, a.w);
      }
      const float sc = sInv[rr];
      const float4 A = make_float4(a.x * sc, a.y * sc, a.z * sc, a.w * sc);
      const size_t grow = grow0 + r;
      if (s_flags[r]) epilogue4(ep, D, grow, d4, A, sL[rr]);
      if (step) {
        const size_t off = grow * D + (size_t)d4 * 4;
        const float4 ap = s_flags[r] ? A : __ldcg(reinterpret_cast<const float4*>(step_ep->a_prev + off));
        const float4 ai = in4(rr, d4);
        MergeRow w;
        w.w1 = sWo[rr];
        w.w2 = sWi[rr];
        w.rden = sWr[rr];
        store4(step_ep->a_full, off,
               make_float4(merge_val(w, ap.x, ai.x), merge_val(w, ap.y, ai.y), merge_val(w, ap.z, ai.z),
                           merge_val(w, ap.w, ai.w)),
               step_ep->out_bf16);
      }
    }
  }
  if (tid == 0 && dep == (unsigned)splits - 1u) {  // every split has seen the full count
    *arrive = 0u;
    *depart = 0u;
  }
}

}  // namespace fb
