// flash_tc.cu -- attention pass on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Used when more than 16 query rows share a KV head (GQA packing: B x G rows), so
// the tiles are a real dense contraction: 128 x 128 x 128 score tiles and
// 128 x 128 x 128 output tiles on tcgen05.mma with fp32 accumulators in tensor
// memory.  Same contract as the mma.sync pass (prefix_bf16.cu): (A, L) per query
// row over a key set -- the out-of-block part over J_out, or the in-block part
// over J_in -- and, in a fused step, the in-block rows, the merge with the cache
// and the decision record (FlashBlock technical summary, gist.science
// 2602.05305, "Core mechanism" and "Adaptive reuse strategies").
//
// A CTA owns a row tile of RT = 32, 64 or 128 rows of one KV group (the MMA is
// always M = 128; TMEM lanes past RT are padding whose softmax is skipped) and
//   SPLIT:  one key range of the split-KV grid (splits, row tiles, b * H_kv).  It
//           writes a normalised partial; once all splits of the tile have arrived
//           (cooperative launch: all CTAs resident), each split CTA combines its
//           share of the rows in fixed split order (deterministic) and runs the
//           epilogue -- small blocks, where row tiles alone cannot fill the GPU;
//   !SPLIT: all keys, epilogue directly (large blocks: video, 4680 rows per head).
// 352 threads:
//   warp 0     TMA producer: Q once; 128-key K tiles into a 3-slot ring and V tiles
//              into a 2-slot ring (128-byte swizzle, no multicast).  A K slot frees
//              when its score MMAs finish, a V slot when its output MMAs do.
//   warp 1     TMEM owner and MMA issuer (one thread):
//                S_w  = Q K_j^T   (M=128, N=128 keys, K=128 d; A, B K-major in
//                                  shared memory)
//                O_w += P_w V_j   (M=128, N=128 d,  K=128 keys; A = P_w in TMEM,
//                                  B = V MN-major in shared memory)
//              for key tiles j split between two softmax warpgroups w = j % 2,
//              so that one group's softmax overlaps the other's MMAs;
//              completions signalled with tcgen05.commit on mbarriers.  An MMA
//              with N = 64 runs at half the rate of N = 128 on this tensor core,
//              which is why the key tile is 128 wide.
//   warps 2-5, 6-9  softmax warpgroups a and b, one query row per thread (TMEM
//              lane = row): read S_w with tcgen05.ld, online softmax in base 2, and
//              P_w as bf16 pairs written back (tcgen05.st) over 64 of S_w's columns
//              whose scores have been read, where the output MMA reads it; the next
//              score MMA of the group is issued after that output MMA, and MMAs of
//              one thread run in issue order.  The exponentials run on the
//              special-function unit (kPolyPair can route pairs to the FMA pipe,
//              exp2_fma2; measured slower here).  O_w is rescaled in TMEM only when
//              a row's max grows by more than 2^8 (otherwise the stale max is kept;
//              p <= 2^8 is exact enough in bf16 and cannot overflow fp32).  At the
//              end group a merges the two partial results (the FlashBlock log-space
//              merge).
//   warp 10    fused step: this split's share of the tile's in-block rows.
// TMEM: 512 columns (S_a / P_a [0,128), S_b / P_b [128,256), O_a [256,384),
// O_b [384,512)).  Every mbarrier wait is time bounded; on expiry the roles fall
// through to the common exit, which frees TMEM.
#include <algorithm>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_device.cuh"
#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {
namespace {

constexpr int kM = 128;
constexpr int kKT = 128;  // keys per tile
constexpr int kD = 128;
constexpr int kKSlots = 3;  // K ring
constexpr int kVSlots = 2;  // V ring
constexpr int kThreads = 352;  // 11 warps
constexpr int kAuxWarp = 10;
constexpr int kBarSoftmax = 1;  // the 8 softmax warps
constexpr int kBarFinish = 2;   // every warp (split combine)
constexpr uint32_t kTmemCols = 512;
// Pairs of keys (t, t + 1) within a 32-key chunk whose exponentials run on the FMA
// pipe (exp2_fma2) instead of the special-function unit.  None: on the video
// workload every fraction tried (1/4, 3/8, 1/2) made the pass slower (0.55, 0.54,
// 0.52 of the burst tensor peak against 0.59 with none) -- the softmax is bound by
// issue slots and latency, not by the special-function unit.
__host__ __device__ constexpr bool kPolyPair(int) { return false; }
// First TMEM column (within S_w) of the P of keys [32c, 32c + 32), c = 0..3: the
// softmax writes each chunk over scores it has already read.
__device__ constexpr uint32_t kPCol[4] = {112, 0, 16, 96};
constexpr uint32_t kOCol = 256;                  // O_a at column 256, O_b at 384
constexpr int kQBlock = 128 * 128;               // Q: [128 rows][128 B] per 64-column block
constexpr int kQBytes = 2 * kQBlock;
constexpr int kKVBlock = kKT * 128;              // K or V: [128 keys][128 B] per 64-column block
constexpr int kKVBytes = 2 * kKVBlock;           // one 128 x 128 tile
constexpr int kQOff = 0;
constexpr int kKOff = kQBytes;
constexpr int kVOff = kKOff + kKSlots * kKVBytes;
constexpr int kAuxOff = kVOff + kVSlots * kKVBytes;  // the aux warp's in-block tile memory
constexpr int kSmemBytes = kAuxOff + TileSmem<kD>::kOperandBytes + 1024;
constexpr int kBufBytes = kSmemBytes - 1024;  // all of it, reused by the split combine
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2, version 1),
// as two 32-bit words.  Low word: start address >> 4 (bits 0-13) and the leading
// byte offset >> 4 (bits 16-29); high word: the stride byte offset >> 4 (bits 0-13),
// the version bit (14) and the swizzle mode (bits 29-31).  K-major: 8-row groups
// 1024 B apart (SBO); LBO unused (1).  MN-major: LBO is the stride between
// 64-element blocks along M/N, SBO the stride between 8-row groups along K.
// Shared addresses are below 2^18, so adding (byte offset >> 4) to the low word
// moves the start without a carry into the LBO field: one add per MMA.
__host__ __device__ constexpr uint32_t desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint64_t desc(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

// Instruction descriptor of kind::f16: fp32 accumulate, bf16 A and B, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Same MMA with A read from tensor memory: a_tmem addresses the 128 x 16 A slice,
// row m in lane m, two bf16 of a row per 32-bit column in k order (low half first).
__device__ __forceinline__ void umma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Bounded wait taken by a whole warp: every lane waits, then all agree (tcgen05.ld /
// st are warp-collective, so a warp must never split on a timeout).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const bool ok = mbar_wait_bounded(bar, parity, err, DEV_ERR_WAIT_FULL);
  return __all_sync(0xffffffffu, ok);
}

template <int RT, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    pass_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PassArgs args) {
  static_assert(RT % 32 == 0 && RT <= kM, "row tile: whole TMEM lane quarters of the 128-row accumulator");
  constexpr int kRealWarps = RT / 32;  // softmax warps per group whose TMEM lanes hold tile rows
  using bf16 = __nv_bfloat16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t k_full[kKSlots];
  __shared__ __align__(8) uint64_t k_empty[kKSlots];
  __shared__ __align__(8) uint64_t v_full[kVSlots];
  __shared__ __align__(8) uint64_t v_empty[kVSlots];
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t p_full[2];
  __shared__ __align__(8) uint64_t o_done[2];
  __shared__ __align__(8) uint64_t fin_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_flags[RT];
  __shared__ int s_red[32];
  __shared__ int s_M;
  __shared__ float s_mb[RT], s_lb[RT];  // group b's row max / sum for the final merge

  const Dims& d = args.d;
  const SplitPlan& plan = args.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = SPLIT ? (int)blockIdx.x : 0;
  const int rt = SPLIT ? (int)blockIdx.y : (int)blockIdx.x;
  const int bg = SPLIT ? (int)blockIdx.z : (int)blockIdx.y;
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int row0 = rt * RT;
  const int rows_valid = min(RT, d.R - row0);
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  const size_t unit = (size_t)bg * plan.n_row_tiles + rt;
  const long long key_begin = SPLIT ? (long long)split * plan.tiles_per_split * kKT : 0;
  const long long key_end = SPLIT ? min(d.N, key_begin + (long long)plan.tiles_per_split * kKT) : d.N;
  const int T = key_end > key_begin ? (int)((key_end - key_begin + kKT - 1) / kKT) : 0;
  const bf16* q = static_cast<const bf16*>(args.q);
  const bf16* k_blk = static_cast<const bf16*>(args.step.k_blk);
  const bf16* v_blk = static_cast<const bf16*>(args.step.v_blk);

  if (SPLIT && args.step.enabled && warp == kAuxWarp) {
    // Whatever the gate decides, this CTA computes its share of the in-block rows:
    // pull their q rows, the group's block keys and values and the cached rows into
    // L1 while the gate reads the mask.
    int r0, r1;
    split_rows(rows_valid, plan.splits, split, r0, r1);
    constexpr int kLinesRow = kD * (int)sizeof(bf16) / 128;  // 128-byte lines per bf16 row
    const int nq = (min(r0 + 16, d.R - row0) - r0) * kLinesRow;  // the 16-row tile the in-block part stages
    const int nkv = d.B * kLinesRow;  // per tensor
    const int nc = (r1 - r0) * (kD * 4 / 128);
    const bf16* kb = k_blk + (size_t)(b * d.hkv + kvh) * d.B * kD;
    const bf16* vb = v_blk + (size_t)(b * d.hkv + kvh) * d.B * kD;
    for (int i = lane; i < nq + 2 * nkv + nc; i += 32) {
      const void* p;
      if (i < nq)
        p = q + (grow0 + r0) * kD + (size_t)i * (128 / sizeof(bf16));
      else if (i < nq + nkv)
        p = kb + (size_t)(i - nq) * (128 / sizeof(bf16));
      else if (i < nq + 2 * nkv)
        p = vb + (size_t)(i - nq - nkv) * (128 / sizeof(bf16));
      else
        p = args.ep.a_dst + (grow0 + r0) * kD + (size_t)(i - nq - 2 * nkv) * 32;
      prefetch_l1(p);
    }
  }

  if (!gate_row_flags(args.gate, d, b, kvh, row0, rows_valid, RT, s_flags, s_red, &s_M)) {
    // Every row of this tile reuses its cache: no K/V is read.  In a fused step the
    // tile's CTAs still produce the step's output from the cache.
    if (SPLIT && args.step.enabled) {
      int r0, r1;
      split_rows(rows_valid, plan.splits, split, r0, r1);
      constexpr int kTileWarps = 8;  // tile memories that fit the idle shared memory
      static_assert(kTileWarps * TileSmem<kD>::kBytes <= kSmemBytes - 1024, "tile memory per warp");
      if (warp < kTileWarps)
        inblock_rows<bf16, kD>(d, q, k_blk, v_blk, b, kvh, row0, r0, r1, step_epilogue(args), warp, kTileWarps,
                               lane, smem);  // nothing else uses shared memory here
      if (split == 0)
        record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, s_M, args.step.dec_M,
                         args.step.dec_reuse, kvh == 0 && rt == 0, tid, kThreads);
    }
    return;
  }

  if (tid == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], kRealWarps);
      mbar_init(&o_done[w], 1);
    }
    mbar_init(&fin_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t sQ = smem_u32(smem + kQOff);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && T > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&q_full, kQBytes);
      for (int h = 0; h < 2; ++h) tma_load_3d(smem + kQOff + h * kQBlock, &tmQ, &q_full, h * 64, (int)grow0, 0);
      // K tiles run up to three ahead, V tiles two: K(j + 3) once the score MMAs of
      // tile j are done, then V(j + 2) once its output MMAs are.
      auto load_k = [&](int n) -> bool {
        const int sl = n % kKSlots;
        if (!mbar_wait_bounded(&k_empty[sl], ((uint32_t)(n / kKSlots) & 1u) ^ 1u, args.err, DEV_ERR_WAIT_EMPTY))
          return false;
        mbar_arrive_expect_tx(&k_full[sl], kKVBytes);
        uint8_t* st = smem + kKOff + sl * kKVBytes;
        const int key0 = (int)(key_begin + (long long)n * kKT);
        for (int h = 0; h < 2; ++h) tma_load_3d(st + h * kKVBlock, &tmK, &k_full[sl], h * 64, key0, bg);
        return true;
      };
      auto load_v = [&](int n) -> bool {
        const int sl = n % kVSlots;
        if (!mbar_wait_bounded(&v_empty[sl], ((uint32_t)(n / kVSlots) & 1u) ^ 1u, args.err, DEV_ERR_WAIT_EMPTY))
          return false;
        mbar_arrive_expect_tx(&v_full[sl], kKVBytes);
        uint8_t* st = smem + kVOff + sl * kKVBytes;
        const int key0 = (int)(key_begin + (long long)n * kKT);
        for (int h = 0; h < 2; ++h) tma_load_3d(st + h * kKVBlock, &tmV, &v_full[sl], h * 64, key0, bg);
        return true;
      };
      int nk = 0, nv = 0;  // tiles issued
      bool ok = true;
      for (; nk < min(T, kKSlots) && ok; ++nk) ok = load_k(nk);
      for (; nv < min(T, kVSlots) && ok; ++nv) ok = load_v(nv);
      while (ok && (nk < T || nv < T)) {
        if (nk < T) {
          ok = load_k(nk);
          if (ok) ++nk;
        }
        if (ok && nv < T) {
          ok = load_v(nv);
          if (ok) ++nv;
        }
      }
      // No copy may still be landing when the CTA leaves (on a timeout above too).
      for (int n = max(0, nk - kKSlots); n < nk; ++n)
        mbar_wait_bounded(&k_full[n % kKSlots], (uint32_t)(n / kKSlots) & 1u, args.err, DEV_ERR_WAIT_FULL);
      for (int n = max(0, nv - kVSlots); n < nv; ++n)
        mbar_wait_bounded(&v_full[n % kVSlots], (uint32_t)(n / kVSlots) & 1u, args.err, DEV_ERR_WAIT_FULL);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && T > 0) {
      constexpr uint32_t kIdQK = idesc_bf16(kM, kKT, false);
      constexpr uint32_t kIdPV = idesc_bf16(kM, kD, true);
      const uint32_t q_lo = desc_lo(sQ, 16);
      const uint32_t k_lo = desc_lo(smem_u32(smem + kKOff), 16);
      const uint32_t v_lo = desc_lo(smem_u32(smem + kVOff), kKVBlock);
      auto wait_k = [&](int j) -> bool {
        return mbar_wait_bounded(&k_full[j % kKSlots], (uint32_t)(j / kKSlots) & 1u, args.err, DEV_ERR_WAIT_FULL);
      };
      auto issue_qk = [&](int j) {  // K_j has landed
        const int sl = j % kKSlots;
        const uint32_t b_lo = k_lo + (uint32_t)sl * (kKVBytes >> 4);
        const uint32_t tS = tmem + (uint32_t)((j & 1) * kKT);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          constexpr uint32_t kHi = desc_hi(1024);
          const uint32_t off = (uint32_t)(((kk >> 2) * kKVBlock + (kk & 3) * 32) >> 4);
          const uint32_t aoff = (uint32_t)(((kk >> 2) * kQBlock + (kk & 3) * 32) >> 4);
          umma(tS, desc(q_lo + aoff, kHi), desc(b_lo + off, kHi), kIdQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[sl]);
        umma_commit(&s_full[j & 1]);
      };
      bool ok = mbar_wait_bounded(&q_full, 0u, args.err, DEV_ERR_WAIT_FULL) && wait_k(0);
      if (ok) issue_qk(0);
      if (ok && T > 1) {
        ok = wait_k(1);
        if (ok) issue_qk(1);
      }
      for (int j = 0; j < T && ok; ++j) {
        const int w = j & 1;
        // The tiles this step reads (V_j, K_{j+2}) are normally in place long before
        // group w hands over P_w: wait for them first, so that only the hand-over
        // stands between the previous MMAs and these.
        const int sl = j % kVSlots;
        if (!mbar_wait_bounded(&v_full[sl], (uint32_t)(j / kVSlots) & 1u, args.err, DEV_ERR_WAIT_FULL)) break;
        if (j + 2 < T && !wait_k(j + 2)) break;
        // O_w += P_w V_j once group w has written P_w for tile j.
        if (!mbar_wait_bounded(&p_full[w], (uint32_t)(j >> 1) & 1u, args.err, DEV_ERR_WAIT_FULL)) break;
        tc_fence_after();
        const uint32_t b_lo = v_lo + (uint32_t)sl * (kKVBytes >> 4);
        const uint32_t tP = tmem + (uint32_t)(w * kKT);
        const uint32_t tO = tmem + kOCol + (uint32_t)(w * kD);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)  // keys [16kk, 16kk + 16): P where the softmax placed them
          umma_tmem_a(tO, tP + kPCol[kk >> 1] + (uint32_t)(8 * (kk & 1)),
                      desc(b_lo + (uint32_t)(kk * (2048 >> 4)), desc_hi(1024)), kIdPV, (j >= 2 || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[sl]);
        umma_commit(&o_done[w]);
        if (j + 2 < T) issue_qk(j + 2);  // after this group's output MMA, in issue order
      }
    }
  } else if (warp == kAuxWarp) {
    // ---------------- aux warp: this split's share of the in-block rows ----------------
    if (SPLIT && args.step.enabled) {
      int r0, r1;
      split_rows(rows_valid, plan.splits, split, r0, r1);
      inblock_rows_to_ws<bf16, kD>(d, q, k_blk, v_blk, b, kvh, row0, r0, r1, args.inblock + unit * RT * (kD + 4),
                                   0, 1, lane, smem + kAuxOff);
    }
  } else {
    // ---------------- softmax warpgroups: one query row per thread ----------------
    const int w = (warp - 2) >> 2;  // 0 = group a (even key tiles), 1 = group b (odd)
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const bool real = quarter < kRealWarps;  // warp-uniform: lanes past the row tile are padding
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + (uint32_t)(w * kKT) + lane_addr;
    const uint32_t tO = tmem + kOCol + (uint32_t)(w * kD) + lane_addr;
    const float sl2 = d.scale * 1.4426950408889634f;
    const int ntiles = (real && T > w) ? (T - w + 1) / 2 : 0;
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int j = 2 * i + w;
      if (!warp_wait(&s_full[w], (uint32_t)i & 1u, args.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Raw scores; the scale (> 0) is applied in the exponent.  Keys past the end
      // of the range (only in its last tile) are masked.  The max reads all of S_w
      // and keeps the last 32-key chunk in registers; the exponentials take it first,
      // writing its P over columns already read, then read the other chunks again,
      // each P chunk going to columns whose scores are consumed: P of keys [96, 128)
      // in columns [96, 112), [0, 32) in [112, 128), [32, 64) in [0, 16) and
      // [64, 96) in [16, 32).  The output MMA reads P in that placement (pcol).
      const long long kleft = key_end - key_begin - (long long)j * kKT;
      auto mask32 = [&](float (&v)[32], int c) {
        if (kleft < kKT) {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = c * 32 + t < kleft ? v[t] : -CUDART_INF_F;
        }
      };
      float mx[8];  // eight independent max chains, then a tree
      float va[32], vb[32];
      tmem_ld32(tS, va);
      tmem_ld32(tS + 32, vb);
      tmem_wait_ld();
      mask32(va, 0);
      mask32(vb, 1);
#pragma unroll
      for (int t = 0; t < 8; ++t) mx[t] = fmaxf(va[t], vb[t]);
#pragma unroll
      for (int t = 8; t < 32; ++t) mx[t & 7] = fmax3(mx[t & 7], va[t], vb[t]);
      tmem_ld32(tS + 64, va);
      tmem_ld32(tS + 96, vb);
      tmem_wait_ld();
      mask32(va, 2);
      mask32(vb, 3);
#pragma unroll
      for (int t = 0; t < 32; ++t) mx[t & 7] = fmax3(mx[t & 7], va[t], vb[t]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                       sl2;
      // The output MMA of this group's previous tile is complete: it was issued before
      // the score MMA of this tile, and s_full[w] completes only once every MMA issued
      // before its commit has.  So O_w may be rescaled and P_w overwritten here.
      if (mt != -CUDART_INF_F && (m_used == -CUDART_INF_F || mt > m_used + 8.f)) {
        const float alpha = m_used == -CUDART_INF_F ? 0.f : ex2_approx(m_used - mt);
        l *= alpha;
        if (i > 0) {
#pragma unroll
          for (int c = 0; c < kD / 32; ++c) {
            float v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] *= alpha;
            tmem_st32(tO + c * 32, v);
          }
          tmem_wait_st();
        }
        m_used = mt;
      }
      const float nbase = m_used == -CUDART_INF_F ? 0.f : -m_used;
      uint64_t ps[4] = {0, 0, 0, 0};  // pairs of partial row sums (+0.f bits)
      const uint64_t SL2 = f2_pack(sl2, sl2), NB = f2_pack(nbase, nbase);
      // One 32-key chunk: exponentials, row-sum pairs, P as bf16 pairs into 16 columns.
      auto exp_chunk = [&](const float (&x)[32], uint32_t col) {
        uint32_t u[16];
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          float x0, x1, p0, p1;
          f2_unpack(f2_fma(f2_pack(x[t], x[t + 1]), SL2, NB), x0, x1);
          if (kPolyPair(t)) {
            exp2_fma2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          ps[(t >> 1) & 3] = f2_add(ps[(t >> 1) & 3], f2_pack(p0, p1));
          u[t >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + col, u);
      };
      tmem_ld32(tS, va);  // chunk 0 again, under chunk 3
      exp_chunk(vb, kPCol[3]);
      tmem_wait_ld();
      tmem_ld32(tS + 32, vb);  // chunk 1, under chunk 0
      mask32(va, 0);
      exp_chunk(va, kPCol[0]);
      tmem_wait_ld();
      tmem_ld32(tS + 64, va);  // chunk 2, under chunk 1
      mask32(vb, 1);
      exp_chunk(vb, kPCol[1]);
      tmem_wait_ld();
      mask32(va, 2);
      exp_chunk(va, kPCol[2]);
      {
        float s0, s1;
        f2_unpack(f2_add(f2_add(ps[0], ps[1]), f2_add(ps[2], ps[3])), s0, s1);
        l += s0 + s1;
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
    }
    if (ok && ntiles > 0) {
      ok = warp_wait(&o_done[w], (uint32_t)(ntiles - 1) & 1u, args.err);
      tc_fence_after();
    }
    const bool has = ok && ntiles > 0;  // warp-uniform
    if (w == 1 && real) {
      s_mb[r] = has ? m_used : -CUDART_INF_F;
      s_lb[r] = has ? l : 0.f;
    }
    named_barrier_sync(kBarSoftmax, 256);
    if (w == 0 && real) {
      // Merge the two groups' partial results row by row (the FlashBlock merge).
      const float ma = has ? m_used : -CUDART_INF_F, la = has ? l : 0.f;
      const float mb = s_mb[r], lb = s_lb[r];
      const bool has_b = T > 1;  // group b's O holds data (warp-uniform)
      const float M = fmaxf(ma, mb);
      const float wa = (M == -CUDART_INF_F || ma == -CUDART_INF_F) ? 0.f : ex2_approx(ma - M);
      const float wb = (M == -CUDART_INF_F || mb == -CUDART_INF_F) ? 0.f : ex2_approx(mb - M);
      const float lt = wa * la + wb * lb;
      const bool row_has = lt > 0.f;
      const float inv = row_has ? 1.f / lt : 0.f;
      const float L = row_has ? (M + __log2f(lt)) * 0.6931471805599453f : -CUDART_INF_F;
      // SPLIT: this CTA's partial row (A normalised, L natural) into the workspace,
      // for every row of the tile; otherwise the epilogue for recomputed rows.
      float* prow = SPLIT ? args.partials + ((unit * plan.splits + split) * RT + r) * (size_t)(kD + 4) : nullptr;
      const bool mine = SPLIT ? true : (r < rows_valid && s_flags[r]);
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        float va[32], vb[32];
        if (has) tmem_ld32(tO + c * 32, va);
        if (has_b) tmem_ld32(tmem + kOCol + kD + lane_addr + c * 32, vb);
        if (has || has_b) tmem_wait_ld();
        if (!mine) continue;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row_has) {
            const float fa = wa * inv, fb2 = wb * inv;
            A.x = (has ? fa * va[t] : 0.f) + (has_b ? fb2 * vb[t] : 0.f);
            A.y = (has ? fa * va[t + 1] : 0.f) + (has_b ? fb2 * vb[t + 1] : 0.f);
            A.z = (has ? fa * va[t + 2] : 0.f) + (has_b ? fb2 * vb[t + 2] : 0.f);
            A.w = (has ? fa * va[t + 3] : 0.f) + (has_b ? fb2 * vb[t + 3] : 0.f);
          }
          if (SPLIT)
            *reinterpret_cast<float4*>(prow + c * 32 + t) = A;
          else
            epilogue4(args.ep, kD, grow0 + r, (c * 32 + t) / 4, A, L);
        }
      }
      if (SPLIT) prow[kD] = L;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  if constexpr (SPLIT) {
    // Every split CTA combines its share of the tile's rows once all splits have
    // arrived (cooperative launch); the shared memory is idle now.
    int r0, r1;
    split_rows(rows_valid, plan.splits, split, r0, r1);
    const Epilogue sep = step_epilogue(args);
    const size_t nunits = (size_t)d.b * d.hkv * plan.n_row_tiles;
    uint32_t fin_phase = 0;
    coop_finish_rows<kD, kThreads>(args.partials + unit * plan.splits * RT * (kD + 4), plan.splits, RT, r0, r1,
                                   args.step.enabled ? args.inblock + unit * RT * (kD + 4) : nullptr, s_flags,
                                   grow0, args.ep, args.step.enabled ? &sep : nullptr, smem, kBufBytes, &fin_bar,
                                   &fin_phase, args.counters + unit, args.counters + nunits + unit, args.err, tid,
                                   kBarFinish);
    if (args.step.enabled && split == 0)
      record_decisions(args.gate, d, b, kvh, row0, rows_valid, s_flags, s_M, args.step.dec_M, args.step.dec_reuse,
                       kvh == 0 && rt == 0, tid, kThreads);
  }
}

template <int RT, bool SPLIT>
cudaError_t launch_tc(const PassArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      cudaStream_t s) {
  auto kern = pass_tc_kernel<RT, SPLIT>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = SPLIT ? dim3(a.plan.splits, a.plan.n_row_tiles, a.d.b * a.d.hkv)
                      : dim3(a.plan.n_row_tiles, a.d.b * a.d.hkv);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the split CTAs of a tile wait for one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (SPLIT && a.plan.splits > 1) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, a);
}

// The pass's pairwise form on pairs (x[2i], x[2i + 1]); an odd last element alone.
__global__ void exp2_fma_kernel(const float* x, float* y, long long n) {
  const long long pairs = n / 2;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += (long long)gridDim.x * blockDim.x) {
    float y0, y1;
    exp2_fma2(x[2 * i], x[2 * i + 1], y0, y1);
    y[2 * i] = y0;
    y[2 * i + 1] = y1;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && (n & 1)) y[n - 1] = exp2_fma(x[n - 1]);
}

}  // namespace

cudaError_t launch_exp2_fma(const float* x, float* y, long long n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const long long blocks = std::min<long long>((n + 255) / 256, 148 * 8);
  exp2_fma_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_pass_tc(const PassArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           cudaStream_t s) {
  if (a.plan.tc == 2) return a.plan.row_tile == kM ? launch_tc<kM, false>(a, tq, tk, tv, s) : cudaErrorInvalidValue;
  switch (a.plan.row_tile) {
    case 32: return launch_tc<32, true>(a, tq, tk, tv, s);
    case 64: return launch_tc<64, true>(a, tq, tk, tv, s);
    case 128: return launch_tc<128, true>(a, tq, tk, tv, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fb
