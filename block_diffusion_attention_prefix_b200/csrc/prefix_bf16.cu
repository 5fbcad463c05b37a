// prefix_bf16.cu -- split-KV attention pass over a bf16 KV cache (sm_100a).
//
// Computes (A, L) of every query row of a KV-head group over a key range: the
// out-of-block pass over the prefix J_out (FlashBlock technical summary,
// gist.science 2602.05305, "Core mechanism": A_out and L_out = log Z_out), and
// the in-block pass over J_in when the block is large (video blocks).
//
// Design (B200):
//  * Grid = (splits, row tiles, b * H_kv).  Each CTA streams one contiguous key
//    range of one KV head.  The G query heads of the group share every K/V tile
//    (GQA packing: row_tile = 16..64 rows = B * G).
//  * One producer warp issues TMA tensor loads (128-byte swizzle, no multicast)
//    of 64-key K and V tiles into a STAGES-deep ring guarded by full/empty
//    mbarriers.  Waits are time-bounded (fb_ptx.cuh).  One aux warp computes the
//    CTA's share of the in-block rows meanwhile (fused step).
//  * Consumer warps (WARPS_M x WARPS_N) run bf16 mma.sync m16n8k16 on the tiles:
//    warp (wm, wn) owns query rows [16 wm, 16 wm + 16) and keys
//    [wn * KW, (wn + 1) * KW) of every tile; Q stays in registers; the online
//    softmax (running max / sum in base 2) stays in registers.
//  * At the end, warps of the same rows merge in shared memory and the CTA writes
//    its partial (A normalised, L natural) to the workspace.  The launch is
//    cooperative (every CTA resident), so the split CTAs of a (b, kv head, row
//    tile) wait for one another on a counter and then each combines its share of
//    the tile's rows over all splits in fixed order (deterministic) and runs the
//    epilogue (write the cache, or merge with the cache into A_full).
//  * Fused step (small blocks): the in-block rows of a tile are spread over its
//    split CTAs (aux warps), the same rows each CTA combines, so each CTA also
//    merges them with the combined cache rows into A_full; split 0 records the
//    decisions, so a denoising step is one launch.  When every row of a tile reuses the cache,
//    its CTAs read no K/V at all: they merge their in-block rows with the cache.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_device.cuh"
#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {
namespace {

constexpr int kKeyTile = 64;

// Byte offset of element (key, d) inside a [64 x D] bf16 tile stored as D/64
// boxes of [64 keys x 64 d] with the TMA 128-byte swizzle: within each 1024-byte
// group of 8 rows, 16-byte chunk c of row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int key, int d) {
  return (uint32_t)((d >> 6) * (kKeyTile * 128) + key * 128 + ((((d & 63) >> 3) ^ (key & 7)) << 4) +
                    (d & 7) * 2);
}

template <int D, int WARPS_M, int WARPS_N, int STAGES>
struct Cfg {
  static constexpr int kConsumerWarps = WARPS_M * WARPS_N;
  static constexpr int kProducerWarp = kConsumerWarps;
  static constexpr int kAuxWarp = kConsumerWarps + 1;
  static constexpr int kThreads = 32 * (kConsumerWarps + 2);
  static constexpr int kFinishThreads = 32 * (kConsumerWarps + 1);  // consumers + aux
  static constexpr int kRowTile = 16 * WARPS_M;
  static constexpr int KW = kKeyTile / WARPS_N;  // keys per warp per tile
  static constexpr int kTileBytes = kKeyTile * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K then V
  static constexpr int kScratchBytes = kConsumerWarps * 16 * (D + 2) * 4;
  static constexpr int kRingBytes = STAGES * kStageBytes;
  // the aux warp's in-block tile memory, past the ring (which is busy while it works)
  static constexpr int kAuxOff = kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes;
  static constexpr int kSmemBytes = kAuxOff + TileSmem<D>::kOperandBytes + 1024;
  static_assert(kConsumerWarps + 2 <= kRingBytes / TileSmem<D>::kBytes, "reuse path: a tile memory per warp");
  static_assert(KW % 16 == 0, "each warp needs whole k16 steps of keys");
  static_assert(D % 64 == 0, "D must be a multiple of 64");
  // The combine stages (rows x (splits + 1)) partial rows, rows <= ceil(RT / splits):
  // at most 2 RT + 149 rows for up to 148 splits (it reads the workspace directly
  // when they do not fit).
  static_assert(kRingBytes >= (2 * kRowTile + 149) * (D + 4) * 4 + 8192, "combine staging");
};

// Barrier ids: 0 = whole CTA, 1 = consumer warps, 2 = consumer + aux warps.
constexpr int kBarConsumers = 1;
constexpr int kBarFinish = 2;

// Shared state of one CTA of the pass, kept across the work items of a persistent CTA.
template <int RT>
struct PassShared {
  uint64_t full_bar[8];
  uint64_t empty_bar[8];
  uint64_t fin_bar;
  int flags[RT];
  int red[32];
  int M;
};

// One work item of the pass -- split `split` of row tile `rt` of (b, KV head) `bg`
// -- executed by every thread of the CTA (the producer warp included).  `tile_base`
// counts the K/V tiles this CTA pushed through its ring before this item, so the
// ring's mbarrier phases continue from one item to the next.  `init_bars`: the
// mbarriers are initialised here, once the gate says the item has work (single-item
// CTAs); persistent CTAs initialise them once up front.  Returns false when a
// bounded wait of this thread gave up.
template <int D, int WARPS_M, int WARPS_N, int STAGES>
__device__ __forceinline__ bool pass_unit(const CUtensorMap* tmK, const CUtensorMap* tmV, const PassArgs& args,
                                          int split, int rt, int bg, uint8_t* smem,
                                          PassShared<Cfg<D, WARPS_M, WARPS_N, STAGES>::kRowTile>& sh,
                                          uint32_t& fin_phase, long long tile_base, bool init_bars) {
  using C = Cfg<D, WARPS_M, WARPS_N, STAGES>;
  constexpr int NCW = C::kConsumerWarps;
  constexpr int KW = C::KW;
  constexpr int RT = C::kRowTile;
  using bf16 = __nv_bfloat16;
  uint64_t* full_bar = sh.full_bar;
  uint64_t* empty_bar = sh.empty_bar;
  int* s_flags = sh.flags;

  const Dims& d = args.d;
  const SplitPlan& plan = args.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int row0 = rt * RT;
  const int rows_valid = min(RT, d.R - row0);
  const size_t unit = (size_t)bg * plan.n_row_tiles + rt;
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  const bf16* q = static_cast<const bf16*>(args.q);
  const bf16* k_blk = static_cast<const bf16*>(args.step.k_blk);
  const bf16* v_blk = static_cast<const bf16*>(args.step.v_blk);
  if (args.step.enabled && !plan.persistent && warp == C::kAuxWarp) {
    // Whatever the gate decides, this CTA computes its share of the in-block rows:
    // pull their q rows, the group's block keys and values and the cached rows into
    // L1 while the gate reads the mask.
    int r0, r1;
    split_rows(rows_valid, plan.splits, split, r0, r1);
    const int lines_row = D * (int)sizeof(bf16) / 128;  // 128-byte lines per bf16 row
    const int nq = (min(r0 + 16, d.R - row0) - r0) * lines_row;  // the 16-row tile the in-block part stages
    const int nkv = d.B * lines_row;  // per tensor
    const int nc = (r1 - r0) * (D * 4 / 128);
    const bf16* kb = k_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
    const bf16* vb = v_blk + (size_t)(b * d.hkv + kvh) * d.B * D;
    for (int i = lane; i < nq + 2 * nkv + nc; i += 32) {
      const void* p;
      if (i < nq)
        p = q + (grow0 + r0) * D + (size_t)i * (128 / sizeof(bf16));
      else if (i < nq + nkv)
        p = kb + (size_t)(i - nq) * (128 / sizeof(bf16));
      else if (i < nq + 2 * nkv)
        p = vb + (size_t)(i - nq - nkv) * (128 / sizeof(bf16));
      else
        p = args.ep.a_dst + (grow0 + r0) * D + (size_t)(i - nq - 2 * nkv) * 32;
      prefetch_l1(p);
    }
  }

  if (!gate_row_flags(args.gate, d, b, kvh, row0, rows_valid, RT, s_flags, sh.red, &sh.M)) {
    // Every row of this tile reuses its cache: no K/V is read.  In a fused step the
    // tile's CTAs still produce the step's output from the cache.
    // (When the reusing rows were handled by the reuse-rows kernel, nothing is left.)
    if (args.step.enabled && !args.step.reuse_done) {
      int r0, r1;
      split_rows(rows_valid, plan.splits, split, r0, r1);
      inblock_rows<bf16, D>(d, q, k_blk, v_blk, b, kvh, row0, r0, r1, step_epilogue(args), warp, C::kThreads / 32,
                            lane, smem);  // the ring is idle: a tile memory per warp
      if (split == 0)
        record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, sh.M, args.step.dec_M,
                         args.step.dec_reuse, kvh == 0 && rt == 0, tid, C::kThreads);
    }
    return true;
  }

  const long long key_begin = (long long)split * plan.tiles_per_split * kKeyTile;
  const long long key_end = min(d.N, key_begin + (long long)plan.tiles_per_split * kKeyTile);
  const int ntiles = key_end > key_begin ? (int)((key_end - key_begin + kKeyTile - 1) / kKeyTile) : 0;

  if (init_bars) {
    if (tid == 0) {
      for (int s = 0; s < STAGES; ++s) {
        mbar_init(&full_bar[s], 1);
        mbar_init(&empty_bar[s], NCW);
      }
      mbar_init(&sh.fin_bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
  }
  bool ok = true;

  if (warp == C::kProducerWarp) {
    // ---------------- producer warp: TMA loads into the ring ----------------
    if (lane == 0 && ntiles > 0) {
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const long long gi = tile_base + i;  // ring position across work items
        const int s = (int)(gi % STAGES);
        const uint32_t ph = (uint32_t)(gi / STAGES) & 1u;
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, args.err, DEV_ERR_WAIT_EMPTY)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
        const int key0 = (int)(key_begin + (long long)i * kKeyTile);
        uint8_t* st = smem + s * C::kStageBytes;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_load_3d(st + h * (kKeyTile * 128), tmK, &full_bar[s], h * 64, key0, bg);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(st + C::kTileBytes + h * (kKeyTile * 128), tmV, &full_bar[s], h * 64, key0, bg);
        ++issued;
      }
      // Do not leave while copies issued by this CTA may still be landing.
      for (int i = max(0, issued - STAGES); i < issued; ++i) {
        const long long gi = tile_base + i;
        ok &= mbar_wait_bounded(&full_bar[gi % STAGES], (uint32_t)(gi / STAGES) & 1u, args.err, DEV_ERR_WAIT_FULL);
      }
    }
    return ok;
  }

  if (warp == C::kAuxWarp) {
    // ---------------- aux warp: this split's share of the in-block rows ------
    if (args.step.enabled) {
      int r0, r1;
      split_rows(rows_valid, plan.splits, split, r0, r1);
      inblock_rows_to_ws<bf16, D>(d, q, k_blk, v_blk, b, kvh, row0, r0, r1, args.inblock + unit * RT * (D + 4),
                                  0, 1, lane, smem + C::kAuxOff);
    }
  } else {
    // ---------------------------- consumer warps ----------------------------
    const int wm = warp / WARPS_N, wn = warp - (warp / WARPS_N) * WARPS_N;
    const int c = lane & 3;
    const int r0 = wm * 16 + (lane >> 2), r1 = r0 + 8;

    // Q fragments (A operand, row-major), rows beyond the group are zero.
    uint32_t qf[D / 16][4];
    {
      const bf16* qb = q + grow0 * D;
      const bool v0 = r0 < rows_valid, v1 = r1 < rows_valid;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int col = kk * 16 + 2 * c;
        qf[kk][0] = v0 ? *reinterpret_cast<const uint32_t*>(qb + (size_t)r0 * D + col) : 0u;
        qf[kk][1] = v1 ? *reinterpret_cast<const uint32_t*>(qb + (size_t)r1 * D + col) : 0u;
        qf[kk][2] = v0 ? *reinterpret_cast<const uint32_t*>(qb + (size_t)r0 * D + col + 8) : 0u;
        qf[kk][3] = v1 ? *reinterpret_cast<const uint32_t*>(qb + (size_t)r1 * D + col + 8) : 0u;
      }
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    const float sl2 = d.scale * 1.4426950408889634f;  // scale * log2(e)

    for (int i = 0; i < ntiles && ok; ++i) {
      const long long gi = tile_base + i;
      const int s = (int)(gi % STAGES);
      if (!mbar_wait_bounded(&full_bar[s], (uint32_t)(gi / STAGES) & 1u, args.err, DEV_ERR_WAIT_FULL)) {
        ok = false;
        break;
      }
      const uint32_t sK = smem_u32(smem + s * C::kStageBytes);
      const uint32_t sV = sK + C::kTileBytes;
      const long long tkey0 = key_begin + (long long)i * kKeyTile + wn * KW;

      // S = Q K^T for this warp's KW keys.
      float sc[KW / 8][4];
#pragma unroll
      for (int n = 0; n < KW / 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int n = 0; n < KW / 8; n += 2) {
          const int key = wn * KW + n * 8 + (lane & 7) + ((lane >> 4) << 3);
          const int dd = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sK + swz(key, dd), b0, b1, b2, b3);
          mma_bf16_16816(sc[n], qf[kk], b0, b1);
          mma_bf16_16816(sc[n + 1], qf[kk], b2, b3);
        }
      }

      // Online softmax in base 2; keys past the range end are masked.
      const long long kvalid = key_end - tkey0;  // keys of this warp slice still in range
      float mx0 = m0, mx1 = m1;
#pragma unroll
      for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = n * 8 + 2 * c + (j & 1);
          const float v = (col < kvalid) ? sc[n][j] * sl2 : -CUDART_INF_F;
          sc[n][j] = v;
          if (j < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float base0 = (mx0 == -CUDART_INF_F) ? 0.f : mx0;
      const float base1 = (mx1 == -CUDART_INF_F) ? 0.f : mx1;
      const float al0 = ex2_approx(m0 - base0), al1 = ex2_approx(m1 - base1);
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int n = 0; n < KW / 8; ++n) {
        sc[n][0] = ex2_approx(sc[n][0] - base0);
        sc[n][1] = ex2_approx(sc[n][1] - base0);
        sc[n][2] = ex2_approx(sc[n][2] - base1);
        sc[n][3] = ex2_approx(sc[n][3] - base1);
        ps0 += sc[n][0] + sc[n][1];
        ps1 += sc[n][2] + sc[n][3];
      }
      l0 = l0 * al0 + ps0;
      l1 = l1 * al1 + ps1;
      m0 = mx0;
      m1 = mx1;
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        o[dn][0] *= al0;
        o[dn][1] *= al0;
        o[dn][2] *= al1;
        o[dn][3] *= al1;
      }

      // O += P V.
#pragma unroll
      for (int k2 = 0; k2 < KW / 16; ++k2) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[2 * k2][0], sc[2 * k2][1]);
        pa[1] = pack_bf16x2(sc[2 * k2][2], sc[2 * k2][3]);
        pa[2] = pack_bf16x2(sc[2 * k2 + 1][0], sc[2 * k2 + 1][1]);
        pa[3] = pack_bf16x2(sc[2 * k2 + 1][2], sc[2 * k2 + 1][3]);
#pragma unroll
        for (int dn = 0; dn < D / 8; dn += 2) {
          const int key = wn * KW + k2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int dd = dn * 8 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + swz(key, dd), b0, b1, b2, b3);
          mma_bf16_16816(o[dn], pa, b0, b1);
          mma_bf16_16816(o[dn + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }

    // Row sums: reduce the per-thread partial sums over the quad.
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

    // Every issued tile has been consumed, so the ring is free: reuse it as scratch.
    named_barrier_sync(kBarConsumers, NCW * 32);
    float* scr = reinterpret_cast<float*>(smem);  // [NCW][16][D + 2]: O, then m, l
    {
      float* w = scr + (size_t)warp * 16 * (D + 2);
      const int q0 = lane >> 2, q1 = q0 + 8;
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        w[q0 * (D + 2) + dn * 8 + 2 * c] = o[dn][0];
        w[q0 * (D + 2) + dn * 8 + 2 * c + 1] = o[dn][1];
        w[q1 * (D + 2) + dn * 8 + 2 * c] = o[dn][2];
        w[q1 * (D + 2) + dn * 8 + 2 * c + 1] = o[dn][3];
      }
      if (c == 0) {
        w[q0 * (D + 2) + D] = m0;
        w[q0 * (D + 2) + D + 1] = l0;
        w[q1 * (D + 2) + D] = m1;
        w[q1 * (D + 2) + D + 1] = l1;
      }
    }
    named_barrier_sync(kBarConsumers, NCW * 32);

    // CTA partial for this split: merge the WARPS_N key slices of each row.
    const size_t rstride = (size_t)D + 4;
    float* mypart = args.partials + (unit * plan.splits + split) * RT * rstride;
    for (int idx = tid; idx < RT * (D / 4); idx += NCW * 32) {
      const int r = idx / (D / 4), d4 = idx - r * (D / 4);
      const int wmr = r >> 4, rr = r & 15;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int x = 0; x < WARPS_N; ++x) M = fmaxf(M, scr[((size_t)(wmr * WARPS_N + x) * 16 + rr) * (D + 2) + D]);
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
      float L = -CUDART_INF_F;
      if (M != -CUDART_INF_F) {
        float den = 0.f;
#pragma unroll
        for (int x = 0; x < WARPS_N; ++x) {
          const float* w = scr + ((size_t)(wmr * WARPS_N + x) * 16 + rr) * (D + 2);
          const float scl = ex2_approx(w[D] - M);
          den += scl * w[D + 1];
          A.x += scl * w[d4 * 4 + 0];
          A.y += scl * w[d4 * 4 + 1];
          A.z += scl * w[d4 * 4 + 2];
          A.w += scl * w[d4 * 4 + 3];
        }
        if (den > 0.f) {
          const float inv = 1.f / den;
          A.x *= inv;
          A.y *= inv;
          A.z *= inv;
          A.w *= inv;
          L = (M + __log2f(den)) * 0.6931471805599453f;
        } else {
          A = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      *reinterpret_cast<float4*>(mypart + (size_t)r * rstride + d4 * 4) = A;
      if (d4 == 0) mypart[(size_t)r * rstride + D] = L;
    }
  }

  // ---- consumers + aux: once every split has arrived, combine this CTA's share of the rows ----
  // Finisher threads are the consumer warps and the aux warp: number them 0..kFinishThreads-1.
  const int ftid = warp < NCW ? tid : NCW * 32 + lane;
  int r0, r1;
  split_rows(rows_valid, plan.splits, split, r0, r1);
  const Epilogue sep = step_epilogue(args);
  const size_t nunits = (size_t)d.b * d.hkv * plan.n_row_tiles;
  coop_finish_rows<D, C::kFinishThreads>(args.partials + unit * plan.splits * RT * (D + 4), plan.splits, RT, r0, r1,
                                         args.step.enabled ? args.inblock + unit * RT * (D + 4) : nullptr, s_flags,
                                         grow0, args.ep, args.step.enabled ? &sep : nullptr, smem, C::kRingBytes,
                                         &sh.fin_bar, &fin_phase, args.counters + unit, args.counters + nunits + unit,
                                         args.err, ftid, kBarFinish);
  if (args.step.enabled && !args.step.reuse_done && split == 0)
    record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, sh.M, args.step.dec_M, args.step.dec_reuse,
                     kvh == 0 && rt == 0, ftid, C::kFinishThreads);
  return ok;
}


// PERSIST = false: one work item per CTA, grid (splits, row tiles, b * H_kv).
// PERSIST = true: the batched fused step's persistent CTAs (plan.persistent).
template <int D, int WARPS_M, int WARPS_N, int STAGES, bool PERSIST>
__global__ void __launch_bounds__(Cfg<D, WARPS_M, WARPS_N, STAGES>::kThreads, 1)
    pass_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const PassArgs args) {
  using C = Cfg<D, WARPS_M, WARPS_N, STAGES>;
  constexpr int RT = C::kRowTile;
  static_assert(STAGES <= 8, "PassShared holds up to 8 stages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) PassShared<RT> sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == C::kProducerWarp && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  uint32_t fin_phase = 0;
  const SplitPlan& plan = args.plan;
  if constexpr (!PERSIST) {
    pass_unit<D, WARPS_M, WARPS_N, STAGES>(&tmK, &tmV, args, blockIdx.x, blockIdx.y, blockIdx.z, smem, sh,
                                           fin_phase, 0, true);
    return;
  }
  // Persistent CTA (one split per tile, many tiles): work items u = blockIdx.x + k * gridDim.x.
  // First the gate of each of them, one thread per item, so that items whose rows all
  // reuse cost no pass at all; then the remaining items one after another.
  __shared__ int s_units[kMaxUnitsPerCta];
  __shared__ int s_nunits, s_abort;
  const Dims& d = args.d;
  const GateParams& g = args.gate;
  if (tid == 0) {
    s_nunits = 0;
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      mbar_init(&sh.empty_bar[s], C::kConsumerWarps);
    }
    mbar_init(&sh.fin_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const long long units = (long long)d.b * d.hkv * plan.n_row_tiles;
  for (long long u = blockIdx.x + (long long)tid * gridDim.x; u < units; u += (long long)C::kThreads * gridDim.x) {
    const int bg = (int)(u / plan.n_row_tiles), rt = (int)(u - (long long)bg * plan.n_row_tiles);
    const int b = bg / d.hkv, kvh = bg - b * d.hkv;
    const int row0 = rt * RT, rows_valid = min(RT, d.R - row0);
    bool need = true;
    if (g.enabled) {
      int M = 0;
      for (int i = 0; i < d.B; ++i) M += g.mask[(size_t)b * d.B + i] != 0;
      const bool tau_ok = tau_reuse(g, M);
      need = false;
      const int h0 = kvh * d.G + row0 / d.B, h1 = kvh * d.G + (row0 + rows_valid - 1) / d.B;
      for (int h = h0; h <= h1 && !need; ++h) need = !head_reuse(g, tau_ok, b, d.hq, h);
    }
    if (need) s_units[atomicAdd(&s_nunits, 1)] = (int)u;
  }
  __syncthreads();
  const int n = s_nunits;
  long long tile_base = 0;
  for (int li = 0; li < n; ++li) {
    const int u = s_units[li];
    const int bg = u / plan.n_row_tiles, rt = u - bg * plan.n_row_tiles;
    const bool ok =
        pass_unit<D, WARPS_M, WARPS_N, STAGES>(&tmK, &tmV, args, 0, rt, bg, smem, sh, fin_phase, tile_base, false);
    tile_base += plan.tiles_per_split;
    fence_proxy_async_smem();  // generic writes to the ring (scratch, staging) before the next item's TMA loads
    if (!ok) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
  }
}

template <int D, int WM, int WN, int STAGES>
cudaError_t launch_cfg(const PassArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  using C = Cfg<D, WM, WN, STAGES>;
  auto kern = a.plan.persistent ? pass_bf16_kernel<D, WM, WN, STAGES, true> : pass_bf16_kernel<D, WM, WN, STAGES, false>;
  static bool attr_set[2][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int pi = a.plan.persistent ? 1 : 0;
  if (dev < 0 || dev >= 64 || !attr_set[pi][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[pi][dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = a.plan.persistent ? dim3(a.plan.grid) : dim3(a.plan.splits, a.plan.n_row_tiles, a.d.b * a.d.hkv);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the split CTAs of a tile wait for one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.plan.splits > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, a);
}

}  // namespace

int bf16_pass_supported(int D, int row_tile) {
  return (D == 64 || D == 128) && (row_tile == 16 || row_tile == 32 || row_tile == 64);
}

cudaError_t launch_pass_bf16(const PassArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  const int D = a.d.D, rt = a.plan.row_tile;
  if (D == 128) {
    if (rt == 16) return launch_cfg<128, 1, 4, 6>(a, tk, tv, s);
    if (rt == 32) return launch_cfg<128, 2, 2, 6>(a, tk, tv, s);
    if (rt == 64) return launch_cfg<128, 4, 1, 6>(a, tk, tv, s);
  } else if (D == 64) {
    if (rt == 16) return launch_cfg<64, 1, 4, 8>(a, tk, tv, s);
    if (rt == 32) return launch_cfg<64, 2, 2, 8>(a, tk, tv, s);
    if (rt == 64) return launch_cfg<64, 4, 1, 8>(a, tk, tv, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fb
