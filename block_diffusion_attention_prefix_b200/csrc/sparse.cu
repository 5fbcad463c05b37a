// sparse.cu -- page-sparse attention with a cached residual (sm_100a).
//
// FlashBlock technical summary (gist.science 2602.05305), "Adaptive reuse
// strategies / compatibility with sparse attention": the keys a sparse selector
// leaves out are treated as the out-of-block set and their attention is cached as
// a residual; the selected keys are attended fresh every step.  The selector is a
// per-query top-k of 16-token pages ranked by a channel-wise min/max bound (the
// LoSA page, gist.science 2604.12056, names QUEST as its selector):
//     e_p = sum_d max(q_d kmin_{p,d}, q_d kmax_{p,d}),
// summed in float64 in ascending d (each bf16 x bf16 product is exact in
// float64, so any implementation summing in that order gets the same bits), top
// k = ceil(density * pages) by (e desc, page asc).
//
// Kernels:
//  * page_minmax_kernel: kmin / kmax [b*H_kv][D][page capacity] (channel-major
//    so that the estimate reads coalesce; the page stride is what the K cache's
//    row capacity holds, so a growing prefix keeps its layout), exact bf16; pages
//    [p_first, P), so a block transition refreshes only the pages it touched.
//  * page_estimate_kernel: e for every (row, page) of recomputing batch
//    elements; one thread per page runs the 16 rows' float64 DFMA chains
//    (max(q kmin, q kmax) is the product picked by the sign of q, exactly).
//  * topk_kernel: one CTA per row: radix select of the k-th key on an
//    order-preserving 64-bit key, tie ranks and compaction in page order ->
//    sorted page list, row bitmap, union bitmap of the KV group (atomicOr).
//  * sparse_pass_kernel: the TMA + mma.sync split pipeline of the dense pass
//    with page-granular loads (four consecutive pages as one 64-key box, other
//    pages as 16-key boxes).  Recompute step: every page, both online softmaxes
//    per row from one score tile (selected pages -> fresh part, other pages ->
//    residual; one exponential per score).  Reuse step: only the union pages of
//    the KV group, selected part only (rows mask the union pages they did not
//    select).  Cooperative launch: once all splits of a tile have arrived, each
//    split CTA combines its own rows of both parts, writes the residual cache
//    (recompute) and A_full = merge(merge(A_sel, A_res), A_in) with the in-block
//    rows its aux warp computed.
#include <cuda.h>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "fb_device.cuh"
#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kPage = 16;
constexpr int kTilePages = 4;  // 64 keys per pipeline tile
constexpr int kBitsWords = 4096;  // shared words for the tile rows' selection bitmaps (16 KB)

__device__ __forceinline__ bool sparse_recompute(const GateParams& g, int b, int B, int* s_red) {
  if (!g.enabled) return true;
  const int M = block_updated_count(g.mask + (size_t)b * B, B, s_red);
  return !tau_reuse(g, M);
}

// ------------------------------------------------------------------ LoSA locality score

// One CTA per (token i, batch element b), one thread per query head: the head's
// sum over d of (q - q_prev)^2 in float64, ascending d, each term a rounded product
// then a rounded sum (no fused multiply-add: the products are not exact); thread 0
// adds the heads in ascending order and divides by H_q * D.  Reading L1 of the LoSA
// page ("2. Methodology": MSE between the queries of steps t and t - 1).
// Sum over d (ascending) of (q - q_prev)^2 for one (batch element, head, token) row of D
// channels, in float64, each term a rounded product then a rounded sum.
__device__ __forceinline__ double head_sq_diff(const bf16* q, const bf16* qp, size_t off, int D) {
  const uint4* qv = reinterpret_cast<const uint4*>(q + off);
  const uint4* pv = reinterpret_cast<const uint4*>(qp + off);
  double acc = 0.0;
  for (int c0 = 0; c0 < D / 8; c0 += 8) {  // 64 channels' loads in flight, then their terms in order
    uint4 xa[8], xb[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      xa[c] = c0 + c < D / 8 ? __ldg(qv + c0 + c) : make_uint4(0, 0, 0, 0);
      xb[c] = c0 + c < D / 8 ? __ldg(pv + c0 + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c0 + c >= D / 8) break;
      const bf16* ea = reinterpret_cast<const bf16*>(&xa[c]);
      const bf16* eb = reinterpret_cast<const bf16*>(&xb[c]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const double diff = __dsub_rn((double)__bfloat162float(ea[e]), (double)__bfloat162float(eb[e]));
        acc = __dadd_rn(acc, __dmul_rn(diff, diff));
      }
    }
  }
  return acc;
}

// The token's score from its heads' sums (ascending h), divided by H_q * D.
__device__ __forceinline__ float token_score(const double* head_sums, int hq, int D) {
  double tot = 0.0;
  for (int h = 0; h < hq; ++h) tot = __dadd_rn(tot, head_sums[h]);
  return (float)__ddiv_rn(tot, (double)hq * D);
}

__global__ void token_mse_kernel(const Dims d, const bf16* q, const bf16* qp, float delta, float* mse,
                                 uint8_t* active) {
  extern __shared__ double s_head[];
  const int i = blockIdx.x, b = blockIdx.y;
  for (int h = threadIdx.x; h < d.hq; h += blockDim.x)
    s_head[h] = head_sq_diff(q, qp, (((size_t)b * d.hq + h) * d.B + i) * d.D, d.D);
  __syncthreads();
  if (threadIdx.x == 0) {
    const float m = token_score(s_head, d.hq, d.D);
    if (mse) mse[(size_t)b * d.B + i] = m;
    active[(size_t)b * d.B + i] = m > delta ? 1 : 0;
  }
}

// Largest number of (token, head) sums the page estimate keeps to score the tokens itself.
constexpr int kEstScoreMax = 2048;

// ------------------------------------------------------------------ page bounds

template <int D>
__global__ void __launch_bounds__(32 * (D / 16)) page_minmax_kernel(const SparseArgs a) {
  const int lane = threadIdx.x & 31, chunk = threadIdx.x >> 5;  // 16 channels per warp
  const int bg = blockIdx.y;
  const int p = a.p_first + blockIdx.x * 32 + lane;
  if (p >= a.P) return;
  const bf16* kp = static_cast<const bf16*>(a.k) + (size_t)bg * a.d.head_stride +
                   (size_t)p * kPage * a.d.row_stride + chunk * 16;
  const long long kend = min((long long)kPage, a.d.N - (long long)p * kPage);
  float mn[16], mx[16];
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    mn[t] = CUDART_INF_F;
    mx[t] = -CUDART_INF_F;
  }
  for (int j = 0; j < kend; ++j) {
    const uint4* src = reinterpret_cast<const uint4*>(kp + (size_t)j * a.d.row_stride);
    const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
      mn[2 * t] = fminf(mn[2 * t], f.x);
      mx[2 * t] = fmaxf(mx[2 * t], f.x);
      mn[2 * t + 1] = fminf(mn[2 * t + 1], f.y);
      mx[2 * t + 1] = fmaxf(mx[2 * t + 1], f.y);
    }
  }
  bf16* omn = a.kmin_out + (size_t)bg * D * a.Pcap + (size_t)(chunk * 16) * a.Pcap + p;
  bf16* omx = a.kmax_out + (size_t)bg * D * a.Pcap + (size_t)(chunk * 16) * a.Pcap + p;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    omn[(size_t)t * a.Pcap] = __float2bfloat16_rn(mn[t]);  // exact: the inputs are bf16
    omx[(size_t)t * a.Pcap] = __float2bfloat16_rn(mx[t]);
  }
}

// ------------------------------------------------------------------ page estimates

constexpr int kEstVec = 2;      // consecutive pages per thread: one 4-byte load per bound row
constexpr int kEstRows = 8;     // rows per thread
constexpr int kEstAhead = 16;   // channels of bound loads in flight (a shared-memory ring per thread)
constexpr int kEstThreads = 128;
constexpr int kEstPages = kEstThreads * kEstVec;  // pages per CTA
constexpr bool kEstSplitSign = true;  // q as (max(q, 0), min(q, 0)) pairs instead of a select

// The rows to estimate (rows[0 .. n)) of KV group bg as float64 pairs
// (max(q, 0), min(q, 0)), channel-major: sq2[2 (c Rp + k) + {0, 1}] for the k-th row;
// rows n .. Rp are zero.  Every thread issues all its 16-byte loads (R <= 32 rows)
// before it stores any of them, so their latencies overlap.
template <int D, int NT>
__device__ void load_group_q2(const SparseArgs& a, int bg, double* sq2, int Rp, const int* rows, int n, int tid) {
  constexpr int kChunks = D / 8;                          // 16-byte chunks per row
  constexpr int kPer = (32 * kChunks + NT - 1) / NT;      // chunks per thread at most
  const Dims& d = a.d;
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const bf16* qg = static_cast<const bf16*>(a.q) + (size_t)(b * d.hq + kvh * d.G) * d.B * D;
  uint4 v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = tid + j * NT;
    v[j] = i < n * kChunks ? __ldg(reinterpret_cast<const uint4*>(qg + (size_t)rows[i / kChunks] * D) + i % kChunks)
                           : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = tid + j * NT;
    if (i >= n * kChunks) break;
    const int k = i / kChunks, c0 = (i % kChunks) * 8;
    const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double q = (double)__uint_as_float(e & 1 ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
      double* dst = sq2 + 2 * ((size_t)(c0 + e) * Rp + k);
      dst[0] = kEstSplitSign ? fmax(q, 0.0) : q;
      dst[1] = kEstSplitSign ? fmin(q, 0.0) : q;
    }
  }
  for (int i = tid; i < (Rp - n) * D; i += NT) {  // padding rows
    const int k = n + i / D, c = i % D;
    sq2[2 * ((size_t)c * Rp + k)] = 0.0;
    sq2[2 * ((size_t)c * Rp + k) + 1] = 0.0;
  }
}

// e for every (row, page) of recomputing batch elements: the bound of each channel
// picked by the sign of q (max(q kmin, q kmax), exactly), summed in float64 in
// ascending d.  With kEstSplitSign the pick is written without a select: q kmax is
// added with max(q, 0) and q kmin with min(q, 0), one of which is a zero -- adding
// q * 0 = +-0 leaves a sum unchanged (it is never -0: it starts at +0, and a rounded
// sum is -0 only when both terms are), so every (row, page) chain rounds exactly as
// the ordered sum of the picked products.  A thread owns 2 consecutive pages (one
// 4-byte load per bound per channel, kEstAhead channels in flight) and 8 rows: 16
// independent float64 chains, each bound widened to float64 once for 8 rows.
// Grid: (page blocks, b * H_kv, chunks of 8 rows); a chunk past the rows to
// estimate returns at once.
template <int D>
__global__ void __launch_bounds__(kEstThreads) page_estimate_kernel(const SparseArgs a) {
  extern __shared__ double sq2[];  // [D][rows rounded up to 8][2], then the bounds ring
  __shared__ int s_red[32];
  __shared__ int s_rows[32];
  __shared__ int s_nrows;
  const Dims& d = a.d;
  const int bg = blockIdx.y, b = bg / d.hkv, kvh = bg - b * d.hkv;
  if (!sparse_recompute(a.gate, b, d.B, s_red)) return;
  const int p0 = blockIdx.x * kEstPages;
  // The union of the group is rebuilt by the top-k: clear this chunk's words.
  if (blockIdx.z == 0 && threadIdx.x < kEstPages / 32) {
    const int w = p0 / 32 + threadIdx.x;
    if (w < a.words) a.union_bits[(size_t)bg * a.words + w] = 0u;
  }
  // LoSA with the score taken here: every CTA scores its batch element's B tokens
  // (the same float64 arithmetic as token_mse_kernel, so every CTA agrees), and one
  // CTA per batch element writes the scores and activity for the launches after it.
  __shared__ uint8_t s_act[kSmallBlockMax];
  __shared__ double s_hsum[kEstScoreMax];
  const bool own_score = a.q_prev != nullptr;
  if (own_score) {
    const bf16* q = static_cast<const bf16*>(a.q);
    const bf16* qp = static_cast<const bf16*>(a.q_prev);
    for (int t = threadIdx.x; t < d.B * d.hq; t += kEstThreads) {
      const int i = t / d.hq, h = t - i * d.hq;
      s_hsum[t] = head_sq_diff(q, qp, (((size_t)b * d.hq + h) * d.B + i) * d.D, d.D);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < d.B; i += kEstThreads) {
      const float m = token_score(s_hsum + (size_t)i * d.hq, d.hq, d.D);
      s_act[i] = m > a.delta ? 1 : 0;
      if (blockIdx.x == 0 && kvh == 0 && blockIdx.z == 0) {
        if (a.mse) a.mse[(size_t)b * d.B + i] = m;
        a.active_out[(size_t)b * d.B + i] = s_act[i];
      }
    }
    __syncthreads();
  }
  // The group rows to estimate: all, or (LoSA) the rows of active tokens (R <= 32).
  if (threadIdx.x == 0) {
    int n = 0;
    for (int r = 0; r < d.R; ++r)
      if (own_score ? s_act[r % d.B] != 0 : (!a.active || a.active[(size_t)b * d.B + r % d.B])) s_rows[n++] = r;
    s_nrows = n;
  }
  __syncthreads();
  const int n = s_nrows;
  if (n == 0) return;
  const int Rp = (n + kEstRows - 1) / kEstRows * kEstRows;
  load_group_q2<D, kEstThreads>(a, bg, sq2, Rp, s_rows, n, threadIdx.x);
  __syncthreads();
  const int pg = p0 + threadIdx.x * kEstVec;  // first of this thread's pages
  if (pg >= a.P) return;
  // Pcap is a multiple of 8 and pg of 2: 4-byte aligned, inside the allocation.
  const uint32_t* mn = reinterpret_cast<const uint32_t*>(a.kmin + (size_t)bg * D * a.Pcap + pg);
  const uint32_t* mx = reinterpret_cast<const uint32_t*>(a.kmax + (size_t)bg * D * a.Pcap + pg);
  const size_t cstride = (size_t)a.Pcap / 2;  // words per channel row
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B;
  auto widen = [](uint32_t u, double (&o)[kEstVec]) {
    o[0] = (double)__uint_as_float(u << 16);
    o[1] = (double)__uint_as_float(u & 0xFFFF0000u);
  };
  {
    const int rc = blockIdx.z;  // this CTA's chunk of 8 rows
    if (rc * kEstRows >= n) return;
    double acc[kEstRows][kEstVec];
#pragma unroll
    for (int k = 0; k < kEstRows; ++k)
#pragma unroll
      for (int p = 0; p < kEstVec; ++p) acc[k][p] = 0.0;
    // Bounds of the next kEstAhead channels in flight through cp.async into this
    // thread's slots of the ring (a DRAM latency covers ~16 channels of work); a
    // slot is refilled right after the thread has read it.
    uint32_t* ring = reinterpret_cast<uint32_t*>(sq2 + 2 * (size_t)Rp * D);  // [kEstAhead][2][kEstThreads]
    auto slot = [&](int c, int bound) { return ring + ((size_t)(c % kEstAhead) * 2 + bound) * kEstThreads + threadIdx.x; };
#pragma unroll
    for (int t = 0; t < kEstAhead; ++t) {
      if (t < D) {
        cp_async4(slot(t, 0), mn + t * cstride);
        cp_async4(slot(t, 1), mx + t * cstride);
      }
      cp_async_commit();
    }
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      cp_async_wait_group<kEstAhead - 1>();  // channel c has landed
      const uint32_t ln = *slot(c, 0), lx = *slot(c, 1);
      double kn[kEstVec], kx[kEstVec];
      widen(ln, kn);
      widen(lx, kx);
      if (c + kEstAhead < D) {
        cp_async4(slot(c, 0), mn + (c + kEstAhead) * cstride);
        cp_async4(slot(c, 1), mx + (c + kEstAhead) * cstride);
      }
      cp_async_commit();
      const double2* qq = reinterpret_cast<const double2*>(sq2 + 2 * ((size_t)c * Rp + rc * kEstRows));
      double2 q[kEstRows];
#pragma unroll
      for (int k = 0; k < kEstRows; ++k) q[k] = qq[k];
      if (kEstSplitSign) {  // all the max(q, 0) terms, then all the min(q, 0) terms: independent FMAs apiece
#pragma unroll
        for (int k = 0; k < kEstRows; ++k)
#pragma unroll
          for (int p = 0; p < kEstVec; ++p) acc[k][p] = fma(q[k].x, kx[p], acc[k][p]);
#pragma unroll
        for (int k = 0; k < kEstRows; ++k)
#pragma unroll
          for (int p = 0; p < kEstVec; ++p) acc[k][p] = fma(q[k].y, kn[p], acc[k][p]);
      } else {
#pragma unroll
        for (int k = 0; k < kEstRows; ++k)
#pragma unroll
          for (int p = 0; p < kEstVec; ++p) acc[k][p] = fma(q[k].x, q[k].x >= 0.0 ? kx[p] : kn[p], acc[k][p]);
      }
    }
    cp_async_wait_all();
#pragma unroll
    for (int k = 0; k < kEstRows; ++k) {
      if (rc * kEstRows + k >= n) break;
      double* e = a.est + (grow0 + s_rows[rc * kEstRows + k]) * (size_t)a.P + pg;
#pragma unroll
      for (int p = 0; p < kEstVec; ++p)
        if (pg + p < a.P) e[p] = acc[k][p];
    }
  }
}

// ------------------------------------------------------------------ top-k pages

constexpr int kTopkThreads = 512;

// Order-preserving key: ascending key <=> descending estimate (estimates are never -0).
__device__ __forceinline__ unsigned long long desc_key(double e) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(e);
  const unsigned long long asc = (u >> 63) ? ~u : (u | (1ull << 63));
  return ~asc;
}

// Exclusive scan of one int per thread over the block (kTopkThreads threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) s_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kTopkThreads / 32 ? s_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kTopkThreads / 32) s_tmp[lane] = t;
  }
  __syncthreads();
  const int before = warp > 0 ? s_tmp[warp - 1] : 0;
  return before + x - v;
}

// KEYS_IN_REGS: each thread holds its (at most 8) keys in registers; otherwise they
// are recomputed from the estimates in global memory at every pass.
template <int REG>
struct KeyCache {
  unsigned long long k[REG > 0 ? REG : 1];
  __device__ __forceinline__ void load(const double* est, int pb, int n) {
#pragma unroll
    for (int t = 0; t < (REG > 0 ? REG : 1); ++t) k[t] = (REG > 0 && t < n) ? desc_key(est[pb + t]) : ~0ull;
  }
};

template <int REG>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const SparseArgs a) {
  extern __shared__ uint32_t s_bits[];  // [words] row bitmap
  __shared__ unsigned hist[256];
  __shared__ int s_tmp[32];
  __shared__ unsigned long long s_prefix, s_key;
  __shared__ unsigned long long s_kand[kTopkThreads / 32], s_kor[kTopkThreads / 32];
  __shared__ int s_kk, s_unique;
  const Dims& d = a.d;
  const int row = blockIdx.x;
  const int b = row / (d.hq * d.B);
  const int h = (row / d.B) % d.hq;
  const int kvh = h / d.G;
  if (!sparse_recompute(a.gate, b, d.B, s_tmp)) return;
  if (a.active && !a.active[(size_t)b * d.B + row % d.B]) return;  // LoSA: stable tokens keep their cache
  const int P = a.P, tid = threadIdx.x;
  if (a.k_sel <= 0 || P <= 0) return;
  const int per = (P + kTopkThreads - 1) / kTopkThreads;
  const int pb = min(P, tid * per), pe = min(P, pb + per);
  const int n = pe - pb;
  const double* est = a.est + (size_t)row * P;
  KeyCache<REG> kc;
  kc.load(est, pb, n);
  // key of the t-th page of this thread (t < n)
#define FB_KEY(t) (REG > 0 ? kc.k[(t)] : desc_key(est[pb + (t)]))
#define FB_FOR_MINE(t) _Pragma("unroll") for (int t = 0; t < (REG > 0 ? REG : 1); ++t) if (REG > 0 ? (t < n) : false)

  // Radix select (up to 8 passes of 8 bits, most significant first) of the k-th
  // smallest key; it stops early once the chosen bin holds a single key, which is
  // then the k-th smallest itself.
  unsigned long long prefix = 0, mask = 0;
  int kk = a.k_sel;
  int first_pass = 0;
  if (REG > 0) {
    // Whole leading bytes that every key shares (the estimates mostly share sign and
    // exponent) would each cost a pass whose histogram has one bin: start past them.
    unsigned long long kand = ~0ull, kor = 0ull;
    FB_FOR_MINE(t) {
      kand &= FB_KEY(t);
      kor |= FB_KEY(t);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kand &= __shfl_xor_sync(0xffffffffu, kand, o);
      kor |= __shfl_xor_sync(0xffffffffu, kor, o);
    }
    if ((tid & 31) == 0) {
      s_kand[tid >> 5] = kand;
      s_kor[tid >> 5] = kor;
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long ba = ~0ull, bo = 0ull;
      for (int w = 0; w < kTopkThreads / 32; ++w) {
        ba &= s_kand[w];
        bo |= s_kor[w];
      }
      s_kand[0] = ba;
      s_kor[0] = bo;
    }
    __syncthreads();
    const unsigned long long diff = s_kand[0] ^ s_kor[0];
    first_pass = diff ? __clzll((long long)diff) / 8 : 8;
    if (first_pass > 0) {
      mask = first_pass >= 8 ? ~0ull : ~0ull << (64 - 8 * first_pass);
      prefix = s_kand[0] & mask;
    }
  }
  for (int pass = first_pass; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    if (tid < 256) hist[tid] = 0u;
    if (tid == 0) s_unique = 0;
    __syncthreads();
    if (REG > 0) {
      // When every lane's key of a warp falls in one bin (the leading bits of the
      // estimates are nearly all equal), one atomic adds the warp's 32.
      const int lane = tid & 31;
#pragma unroll
      for (int t = 0; t < (REG > 0 ? REG : 1); ++t) {
        const unsigned long long key = kc.k[t];
        const bool part = t < n && (key & mask) == prefix;
        const unsigned bin = (unsigned)(key >> shift) & 255u;
        const unsigned bin0 = __shfl_sync(0xffffffffu, bin, 0);
        if (__all_sync(0xffffffffu, part && bin == bin0)) {
          if (lane == 0) atomicAdd(&hist[bin], 32u);
        } else if (part) {
          atomicAdd(&hist[bin], 1u);
        }
      }
    } else {
      for (int t = 0; t < n; ++t) {
        const unsigned long long key = FB_KEY(t);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (tid < 32) {
      unsigned c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[tid * 8 + j];
        sum += c[j];
      }
      unsigned incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const unsigned excl = incl - sum;
      const unsigned long long hit = __ballot_sync(0xffffffffu, excl < (unsigned)kk && (unsigned)kk <= incl);
      const int owner = __ffsll((long long)hit) - 1;
      if (tid == owner) {
        unsigned run = excl, cnt = 0;
        int bin = 0;
        for (int j = 0; j < 8; ++j) {
          if ((unsigned)kk <= run + c[j]) {
            bin = tid * 8 + j;
            cnt = c[j];
            break;
          }
          run += c[j];
        }
        s_prefix = prefix | ((unsigned long long)bin << shift);
        s_kk = kk - (int)run;
        s_unique = cnt == 1u;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    kk = s_kk;
    mask |= 0xFFull << shift;
    const bool unique = s_unique != 0;
    if (unique) {  // the one key under this prefix is the k-th smallest (kk == 1)
      if (REG > 0) {
        FB_FOR_MINE(t) {
          const unsigned long long key = FB_KEY(t);
          if ((key & mask) == prefix) s_key = key;
        }
      } else {
        for (int t = 0; t < n; ++t) {
          const unsigned long long key = FB_KEY(t);
          if ((key & mask) == prefix) s_key = key;
        }
      }
    }
    __syncthreads();
    if (unique) {
      prefix = s_key;
      break;
    }
  }
  const unsigned long long T = prefix;  // the k-th smallest key; take `kk` of the keys equal to it

  // Ties to T go to the lowest pages: rank them in page order, then compact.
  int my_eq = 0;
  if (REG > 0) {
    FB_FOR_MINE(t) my_eq += FB_KEY(t) == T;
  } else {
    for (int t = 0; t < n; ++t) my_eq += FB_KEY(t) == T;
  }
  const int eq_rank = block_exclusive_scan(my_eq, s_tmp);
  int my_take = 0;
  {
    int r = eq_rank;
    if (REG > 0) {
      FB_FOR_MINE(t) {
        const unsigned long long key = FB_KEY(t);
        const bool eq = key == T;
        my_take += (key < T) || (eq && r < kk);
        r += eq;
      }
    } else {
      for (int t = 0; t < n; ++t) {
        const unsigned long long key = FB_KEY(t);
        const bool eq = key == T;
        my_take += (key < T) || (eq && r < kk);
        r += eq;
      }
    }
  }
  int pos = block_exclusive_scan(my_take, s_tmp);
  for (int w = tid; w < a.words; w += kTopkThreads) s_bits[w] = 0u;
  __syncthreads();
  {
    int r = eq_rank;
    int32_t* out = a.sel_idx + (size_t)row * a.k_sel;
    auto take = [&](int t, unsigned long long key) {
      const int p = pb + t;
      const bool eq = key == T;
      if ((key < T) || (eq && r < kk)) {
        out[pos++] = p;
        atomicOr(&s_bits[p >> 5], 1u << (p & 31));
      }
      r += eq;
    };
    if (REG > 0) {
      FB_FOR_MINE(t) take(t, FB_KEY(t));
    } else {
      for (int t = 0; t < n; ++t) take(t, FB_KEY(t));
    }
  }
#undef FB_KEY
#undef FB_FOR_MINE
  __syncthreads();
  uint32_t* rb = a.sel_bits + (size_t)row * a.words;
  uint32_t* ub = a.union_bits + (size_t)(b * d.hkv + kvh) * a.words;
  for (int w = tid; w < a.words; w += kTopkThreads) {
    const uint32_t v = s_bits[w];
    rb[w] = v;
    if (v) atomicOr(ub + w, v);
  }
}

// ------------------------------------------------------------------ sparse pass

template <int D, int WARPS_M, int WARPS_N, int STAGES>
struct SCfg {
  static constexpr int kConsumerWarps = WARPS_M * WARPS_N;
  static constexpr int kProducerWarp = kConsumerWarps;
  static constexpr int kAuxWarp = kConsumerWarps + 1;
  static constexpr int kThreads = 32 * (kConsumerWarps + 2);
  static constexpr int kFinishThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kRowTile = 16 * WARPS_M;
  static constexpr int KW = 64 / WARPS_N;
  static constexpr int kPageBytes = kPage * D * 2;         // one page of K (or V)
  static constexpr int kTileBytes = kTilePages * kPageBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;       // K then V
  static constexpr int kScratchBytes = kConsumerWarps * 16 * (D + 2) * 4 * 2;  // sel and res
  static constexpr int kRingBytes = STAGES * kStageBytes;
  // the aux warp's in-block tile memory, past the ring (which is busy while it works)
  static constexpr int kAuxOff = kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes;
  static constexpr int kSmemBytes = kAuxOff + TileSmem<D>::kOperandBytes + 1024;
  static_assert(KW % 16 == 0, "whole k16 steps per warp");
  // The split combine stages rows x (2 splits + 1) partial rows (rows <= ceil(RT / splits)):
  // at most 2 (2 RT + 149) + RT rows for up to 148 splits (it reads the workspace otherwise).
  static_assert(kRingBytes >= 3 * kRowTile * (D + 4) * 4, "combine staging");
};

// Byte offset of (key in tile, d) for a tile of 4 pages (64 keys) stored as D/64
// boxes of [64 keys x 64 d] with the 128-byte swizzle (chunk c of row r at c ^ (r % 8)).
// Page j of the tile is keys [16 j, 16 j + 16): a 16-row box at offset 2048 j of each
// 64-column half has the same swizzle phase as rows of one 64-row box, so four
// consecutive pages can arrive as one box per half and single pages as small boxes.
__device__ __forceinline__ uint32_t pswz(int key, int d, int D) {
  (void)D;
  return (uint32_t)((d >> 6) * (kTilePages * kPage * 128) + key * 128 + ((((d & 63) >> 3) ^ (key & 7)) << 4) +
                    (d & 7) * 2);
}

// Online-softmax state of one 16-row fragment set (two rows per thread).
template <int D>
struct Acc {
  float o[D / 8][4];
  float m0, m1, l0, l1;
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m0 = m1 = -CUDART_INF_F;
    l0 = l1 = 0.f;
  }
};

// Online softmax update + P V for one tile: `sc` holds base-2 scores (masked to
// -inf where the key is not in this set).
template <int D, int KW>
__device__ __forceinline__ void softmax_pv(Acc<D>& A, float (&sc)[KW / 8][4], uint32_t sV, int wn, int lane) {
  float mx0 = A.m0, mx1 = A.m1;
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
    mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
    mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float base0 = (mx0 == -CUDART_INF_F) ? 0.f : mx0;
  const float base1 = (mx1 == -CUDART_INF_F) ? 0.f : mx1;
  const float al0 = ex2_approx(A.m0 - base0), al1 = ex2_approx(A.m1 - base1);
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
  A.l0 = A.l0 * al0 + ps0;
  A.l1 = A.l1 * al1 + ps1;
  A.m0 = mx0;
  A.m1 = mx1;
#pragma unroll
  for (int dn = 0; dn < D / 8; ++dn) {
    A.o[dn][0] *= al0;
    A.o[dn][1] *= al0;
    A.o[dn][2] *= al1;
    A.o[dn][3] *= al1;
  }
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
      ldsm_x4_t(sV + pswz(key, dd, D), b0, b1, b2, b3);
      mma_bf16_16816(A.o[dn], pa, b0, b1);
      mma_bf16_16816(A.o[dn + 1], pa, b2, b3);
    }
  }
}

// Recompute steps: both online softmaxes -- the selected and the residual key sets
// of each row -- from one score tile.  `sc` holds base-2 scores (-inf where the key
// is past the end), `sel` says which set each score belongs to; one exponential per
// score (against its own set's running max) and two P V products that share every
// V fragment.
template <int D, int KW>
__device__ __forceinline__ void softmax_pv_dual(Acc<D>& As, Acc<D>& Ar, float (&sc)[KW / 8][4],
                                                const bool (&sel)[KW / 8][4], uint32_t sV, int wn, int lane) {
  float ms0 = As.m0, ms1 = As.m1, mr0 = Ar.m0, mr1 = Ar.m1;
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v = sc[n][j];
      if (j < 2) {
        if (sel[n][j]) ms0 = fmaxf(ms0, v); else mr0 = fmaxf(mr0, v);
      } else {
        if (sel[n][j]) ms1 = fmaxf(ms1, v); else mr1 = fmaxf(mr1, v);
      }
    }
  }
#pragma unroll
  for (int x = 1; x <= 2; x <<= 1) {
    ms0 = fmaxf(ms0, __shfl_xor_sync(0xffffffffu, ms0, x));
    ms1 = fmaxf(ms1, __shfl_xor_sync(0xffffffffu, ms1, x));
    mr0 = fmaxf(mr0, __shfl_xor_sync(0xffffffffu, mr0, x));
    mr1 = fmaxf(mr1, __shfl_xor_sync(0xffffffffu, mr1, x));
  }
  const float bs0 = (ms0 == -CUDART_INF_F) ? 0.f : ms0, bs1 = (ms1 == -CUDART_INF_F) ? 0.f : ms1;
  const float br0 = (mr0 == -CUDART_INF_F) ? 0.f : mr0, br1 = (mr1 == -CUDART_INF_F) ? 0.f : mr1;
  const float as0 = ex2_approx(As.m0 - bs0), as1 = ex2_approx(As.m1 - bs1);
  const float ar0 = ex2_approx(Ar.m0 - br0), ar1 = ex2_approx(Ar.m1 - br1);
  float pss0 = 0.f, pss1 = 0.f, psr0 = 0.f, psr1 = 0.f;
  float ps[KW / 8][4], pr[KW / 8][4];
#pragma unroll
  for (int n = 0; n < KW / 8; ++n) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool s_ = sel[n][j];
      const float base = j < 2 ? (s_ ? bs0 : br0) : (s_ ? bs1 : br1);
      const float p = ex2_approx(sc[n][j] - base);
      ps[n][j] = s_ ? p : 0.f;
      pr[n][j] = s_ ? 0.f : p;
    }
    pss0 += ps[n][0] + ps[n][1];
    pss1 += ps[n][2] + ps[n][3];
    psr0 += pr[n][0] + pr[n][1];
    psr1 += pr[n][2] + pr[n][3];
  }
  As.l0 = As.l0 * as0 + pss0;
  As.l1 = As.l1 * as1 + pss1;
  Ar.l0 = Ar.l0 * ar0 + psr0;
  Ar.l1 = Ar.l1 * ar1 + psr1;
  As.m0 = ms0;
  As.m1 = ms1;
  Ar.m0 = mr0;
  Ar.m1 = mr1;
#pragma unroll
  for (int dn = 0; dn < D / 8; ++dn) {
    As.o[dn][0] *= as0;
    As.o[dn][1] *= as0;
    As.o[dn][2] *= as1;
    As.o[dn][3] *= as1;
    Ar.o[dn][0] *= ar0;
    Ar.o[dn][1] *= ar0;
    Ar.o[dn][2] *= ar1;
    Ar.o[dn][3] *= ar1;
  }
#pragma unroll
  for (int k2 = 0; k2 < KW / 16; ++k2) {
    uint32_t pa[4], pb[4];
    pa[0] = pack_bf16x2(ps[2 * k2][0], ps[2 * k2][1]);
    pa[1] = pack_bf16x2(ps[2 * k2][2], ps[2 * k2][3]);
    pa[2] = pack_bf16x2(ps[2 * k2 + 1][0], ps[2 * k2 + 1][1]);
    pa[3] = pack_bf16x2(ps[2 * k2 + 1][2], ps[2 * k2 + 1][3]);
    pb[0] = pack_bf16x2(pr[2 * k2][0], pr[2 * k2][1]);
    pb[1] = pack_bf16x2(pr[2 * k2][2], pr[2 * k2][3]);
    pb[2] = pack_bf16x2(pr[2 * k2 + 1][0], pr[2 * k2 + 1][1]);
    pb[3] = pack_bf16x2(pr[2 * k2 + 1][2], pr[2 * k2 + 1][3]);
#pragma unroll
    for (int dn = 0; dn < D / 8; dn += 2) {
      const int key = wn * KW + k2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int dd = dn * 8 + (lane >> 4) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sV + pswz(key, dd, D), b0, b1, b2, b3);
      mma_bf16_16816(As.o[dn], pa, b0, b1);
      mma_bf16_16816(As.o[dn + 1], pa, b2, b3);
      mma_bf16_16816(Ar.o[dn], pb, b0, b1);
      mma_bf16_16816(Ar.o[dn + 1], pb, b2, b3);
    }
  }
}

// Merge the WARPS_N key slices of each row (scratch in smem) into this CTA's
// partial [RT][D + 4] (A normalised, natural-log L) in global memory.
template <int D, int WARPS_M, int WARPS_N>
__device__ void write_partial(const float* scr, float* mypart, int tid) {
  constexpr int RT = 16 * WARPS_M, NCW = WARPS_M * WARPS_N;
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
        const float s = ex2_approx(w[D] - M);
        den += s * w[D + 1];
        A.x += s * w[d4 * 4 + 0];
        A.y += s * w[d4 * 4 + 1];
        A.z += s * w[d4 * 4 + 2];
        A.w += s * w[d4 * 4 + 3];
      }
      if (den > 0.f) {
        const float inv = 1.f / den;
        A = make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
        L = (M + __log2f(den)) * 0.6931471805599453f;
      } else {
        A = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    *reinterpret_cast<float4*>(mypart + (size_t)r * (D + 4) + d4 * 4) = A;
    if (d4 == 0) mypart[(size_t)r * (D + 4) + D] = L;
  }
}

template <int D>
__device__ __forceinline__ void stash(float* scr, int warp, int lane, const Acc<D>& A) {
  float* w = scr + (size_t)warp * 16 * (D + 2);
  const int c = lane & 3, q0 = lane >> 2, q1 = q0 + 8;
#pragma unroll
  for (int dn = 0; dn < D / 8; ++dn) {
    w[q0 * (D + 2) + dn * 8 + 2 * c] = A.o[dn][0];
    w[q0 * (D + 2) + dn * 8 + 2 * c + 1] = A.o[dn][1];
    w[q1 * (D + 2) + dn * 8 + 2 * c] = A.o[dn][2];
    w[q1 * (D + 2) + dn * 8 + 2 * c + 1] = A.o[dn][3];
  }
  if (c == 0) {
    w[q0 * (D + 2) + D] = A.m0;
    w[q0 * (D + 2) + D + 1] = A.l0;
    w[q1 * (D + 2) + D] = A.m1;
    w[q1 * (D + 2) + D + 1] = A.l1;
  }
}

constexpr int kBarConsumers = 1;
constexpr int kBarFinish = 2;

// Split combine of the sparse pass, spread over the split CTAs of one (b, KV head,
// row tile) `unit` (the launch is cooperative: all CTAs resident).  Called by the
// threads [0, NT) of every split CTA once its partials (selected set; residual set
// on recompute steps) and its in-block rows are in the workspace.  Each CTA waits
// (bounded) for the other splits, pulls rows [r0, r1) of every split's partials and
// its in-block rows into shared memory (one bulk copy per split and set), and then:
//   A_sel, L_sel (and A_res, L_res on recompute) over all splits -- the FlashBlock
//   merge equation with the split weights e_s = e^{L_s - M}, a fixed warp-tree sum;
//   recompute: the residual cache is written; reuse: it is read;
//   A_full = merge(merge(A_sel, A_res), A_in).
template <int D, int NT>
__device__ void sparse_coop_rows(const SparseArgs& args, size_t unit, int RT, int r0, int r1, size_t grow0,
                                 bool recompute, uint8_t* sbuf, int sbuf_bytes, uint64_t* mbar, int tid,
                                 int bar_id) {
  constexpr int RS = D + 4;
  constexpr int D4 = D / 4;
  constexpr int NW = NT / 32;
  const int splits = args.plan.splits;
  const int n = r1 - r0 > 0 ? r1 - r0 : 0;
  const int nsets = recompute ? 2 : 1;
  const float* part[2] = {args.part_sel + unit * splits * RT * RS, args.part_res + unit * splits * RT * RS};
  const float* pin = args.inblock + unit * RT * RS;
  const size_t nd = (size_t)splits * n * RS;  // floats of one set's staged rows
  float* sA = reinterpret_cast<float*>(sbuf);  // [nsets][splits][n][RS]
  float* sIn = sA + nsets * nd;                 // [n][RS]
  float* sE = sIn + (size_t)n * RS;             // [nsets][n][splits]
  float* sL = sE + (size_t)nsets * n * splits;  // [2][n] combined L per set
  float* sInv = sL + 2 * n;                     // [2][n]
  float* sW = sInv + 2 * n;                     // [n][6]: merge weights pre (3), full (3)
  const bool staged = (nsets * nd + (size_t)n * RS + (size_t)nsets * n * splits + 10 * (size_t)n) * 4 <=
                      (size_t)sbuf_bytes;
  unsigned int* arrive = args.counters + unit;
  unsigned int* depart = args.counters + (size_t)args.d.b * args.d.hkv * args.plan.n_row_tiles + unit;
  fence_proxy_async_smem();
  named_barrier_sync(bar_id, NT);  // this CTA's partials and in-block rows are written
  bool ok = true;
  unsigned int dep = 0;
  if (tid == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
    ok = wait_count_bounded(arrive, (unsigned)splits, args.err, DEV_ERR_WAIT_PEERS);
    dep = atomicAdd(depart, 1u);  // result checked at the end
    if (ok && staged && n > 0) {
      fence_proxy_async_global();
      const uint32_t row_bytes = (uint32_t)n * RS * 4;
      mbar_arrive_expect_tx(mbar, row_bytes * (uint32_t)(nsets * splits + 1));
      for (int st = 0; st < nsets; ++st)
        for (int sp = 0; sp < splits; ++sp)
          bulk_load(sA + st * nd + (size_t)sp * n * RS, part[st] + ((size_t)sp * RT + r0) * RS, row_bytes, mbar);
      bulk_load(sIn, pin + (size_t)r0 * RS, row_bytes, mbar);
    }
  }
  ok = named_barrier_and(bar_id, NT, ok);
  if (ok && n > 0) {
    if (staged) ok = mbar_wait_bounded(mbar, 0u, args.err, DEV_ERR_WAIT_COMBINE);
    ok = named_barrier_and(bar_id, NT, ok);
  }
  if (ok && n > 0) {
    auto ld1 = [&](int st, int sp, int rr) -> float {
      return staged ? sA[st * nd + ((size_t)sp * n + rr) * RS + D]
                    : __ldcg(part[st] + ((size_t)sp * RT + r0 + rr) * RS + D);
    };
    auto ld4 = [&](int st, int sp, int rr, int d4) -> float4 {
      return staged ? reinterpret_cast<const float4*>(sA + st * nd + ((size_t)sp * n + rr) * RS)[d4]
                    : __ldcg(reinterpret_cast<const float4*>(part[st] + ((size_t)sp * RT + r0 + rr) * RS) + d4);
    };
    auto in1 = [&](int rr) -> float {
      return staged ? sIn[(size_t)rr * RS + D] : __ldcg(pin + (size_t)(r0 + rr) * RS + D);
    };
    auto in4 = [&](int rr, int d4) -> float4 {
      return staged ? reinterpret_cast<const float4*>(sIn + (size_t)rr * RS)[d4]
                    : __ldcg(reinterpret_cast<const float4*>(pin + (size_t)(r0 + rr) * RS) + d4);
    };
    const int warp = tid >> 5, lane = tid & 31;
    // split weights, one warp per (set, row)
    for (int pr = warp; pr < nsets * n; pr += NW) {
      const int st = pr / n, rr = pr - st * n;
      float M = -CUDART_INF_F;
      for (int sp = lane; sp < splits; sp += 32) M = fmaxf(M, ld1(st, sp, rr));
      M = warp_max(M);
      float den = 0.f;
      for (int sp = lane; sp < splits; sp += 32) {
        const float e = M == -CUDART_INF_F ? 0.f : expf(ld1(st, sp, rr) - M);
        sE[((size_t)st * n + rr) * splits + sp] = e;
        den += e;
      }
      den = warp_sum(den);
      if (lane == 0) {
        sL[st * n + rr] = den > 0.f ? M + logf(den) : -CUDART_INF_F;
        sInv[st * n + rr] = den > 0.f ? 1.f / den : 0.f;
      }
    }
    named_barrier_sync(bar_id, NT);
    // per row: pre = merge(sel, res), full = merge(pre, in)
    const bool losa = args.active != nullptr;
    for (int rr = tid; rr < n; rr += NT) {
      const size_t grow = grow0 + r0 + rr;
      const float ls = sL[rr];
      if (losa) {  // active rows: the fresh sparse result is the new cache; stable rows read it
        const bool act = args.active[(size_t)(grow / ((size_t)args.d.hq * args.d.B)) * args.d.B + grow % args.d.B] != 0;
        const float lc = act ? ls : __ldcg(args.l_res + grow);
        const MergeRow wf = merge_row(lc, in1(rr));
        float* w = sW + (size_t)rr * 6;
        w[0] = act ? 1.f : 0.f;
        w[3] = wf.w1;
        w[4] = wf.w2;
        w[5] = wf.rden;
        if (act) args.l_res[grow] = ls;
        if (args.l_sel) args.l_sel[grow] = ls;
        if (args.step.l_full) args.step.l_full[grow] = wf.l;
        continue;
      }
      const float lr = recompute ? sL[n + rr] : __ldcg(args.l_res + grow);
      const MergeRow wp = merge_row(ls, lr);
      const MergeRow wf = merge_row(wp.l, in1(rr));
      float* w = sW + (size_t)rr * 6;
      w[0] = wp.w1;
      w[1] = wp.w2;
      w[2] = wp.rden;
      w[3] = wf.w1;
      w[4] = wf.w2;
      w[5] = wf.rden;
      if (recompute) args.l_res[grow] = lr;
      if (args.l_sel) args.l_sel[grow] = ls;
      if (args.step.l_full) args.step.l_full[grow] = wf.l;
    }
    named_barrier_sync(bar_id, NT);
    for (int idx = tid; idx < n * D4; idx += NT) {
      const int rr = idx / D4, d4 = idx - rr * D4;
      const size_t off = (grow0 + r0 + rr) * D + (size_t)d4 * 4;
      float4 acc[2];
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        acc[st] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (st >= nsets) continue;
        const float* er = sE + ((size_t)st * n + rr) * splits;
        for (int sp = 0; sp < splits; ++sp) {
          const float e = er[sp];
          const float4 x = ld4(st, sp, rr, d4);
          acc[st].x = fmaf(e, x.x, acc[st].x);
          acc[st].y = fmaf(e, x.y, acc[st].y);
          acc[st].z = fmaf(e, x.z, acc[st].z);
          acc[st].w = fmaf(e, x.w, acc[st].w);
        }
        const float sc = sInv[st * n + rr];
        acc[st] = make_float4(acc[st].x * sc, acc[st].y * sc, acc[st].z * sc, acc[st].w * sc);
      }
      const float4 as = acc[0];
      if (losa) {
        const float* w = sW + (size_t)rr * 6;
        const bool act = w[0] != 0.f;
        const float4 ac = act ? as : __ldcg(reinterpret_cast<const float4*>(args.a_res + off));
        if (act) *reinterpret_cast<float4*>(args.a_res + off) = as;
        if (args.a_sel) *reinterpret_cast<float4*>(args.a_sel + off) = as;
        MergeRow wf;
        wf.w1 = w[3];
        wf.w2 = w[4];
        wf.rden = w[5];
        const float4 ai = in4(rr, d4);
        store4(args.step.a_full, off,
               make_float4(merge_val(wf, ac.x, ai.x), merge_val(wf, ac.y, ai.y), merge_val(wf, ac.z, ai.z),
                           merge_val(wf, ac.w, ai.w)),
               1);
        continue;
      }
      const float4 ar = recompute ? acc[1] : __ldcg(reinterpret_cast<const float4*>(args.a_res + off));
      if (recompute) *reinterpret_cast<float4*>(args.a_res + off) = ar;
      if (args.a_sel) *reinterpret_cast<float4*>(args.a_sel + off) = as;
      const float* w = sW + (size_t)rr * 6;
      MergeRow wp, wf;
      wp.w1 = w[0];
      wp.w2 = w[1];
      wp.rden = w[2];
      wf.w1 = w[3];
      wf.w2 = w[4];
      wf.rden = w[5];
      const float4 ai = in4(rr, d4);
      const float4 pre = make_float4(merge_val(wp, as.x, ar.x), merge_val(wp, as.y, ar.y), merge_val(wp, as.z, ar.z),
                                     merge_val(wp, as.w, ar.w));
      store4(args.step.a_full, off,
             make_float4(merge_val(wf, pre.x, ai.x), merge_val(wf, pre.y, ai.y), merge_val(wf, pre.z, ai.z),
                         merge_val(wf, pre.w, ai.w)),
             1);
    }
  }
  if (tid == 0 && dep == (unsigned)splits - 1u) {  // every split has seen the full count
    *arrive = 0u;
    *depart = 0u;
  }
}



template <int D, int WARPS_M, int WARPS_N, int STAGES>
__global__ void __launch_bounds__(SCfg<D, WARPS_M, WARPS_N, STAGES>::kThreads, 1)
    sparse_pass_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmK4, const __grid_constant__ CUtensorMap tmV4,
                       const SparseArgs args) {
  using C = SCfg<D, WARPS_M, WARPS_N, STAGES>;
  constexpr int NCW = C::kConsumerWarps;
  constexpr int KW = C::KW;
  constexpr int RT = C::kRowTile;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t comb_bar;
  __shared__ int s_pages[STAGES][kTilePages];
  __shared__ uint32_t s_bits[kBitsWords];
  __shared__ int s_flags[RT];
  __shared__ int s_red[32];
  __shared__ int s_M;
  __shared__ int s_recompute;
  __shared__ int s_union_total;

  const Dims& d = args.d;
  const SplitPlan& plan = args.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, rt = blockIdx.y, bg = blockIdx.z;
  const int b = bg / d.hkv, kvh = bg - b * d.hkv;
  const int row0 = rt * RT;
  const int rows_valid = min(RT, d.R - row0);
  const size_t unit = (size_t)bg * plan.n_row_tiles + rt;
  const size_t grow0 = (size_t)(b * d.hq + kvh * d.G) * d.B + row0;
  const bf16* q = static_cast<const bf16*>(args.q);

  // Gate (tau only): every row of the batch element decides alike.
  {
    int M = 0;
    bool rec = true;
    if (args.gate.enabled) {
      M = block_updated_count(args.gate.mask + (size_t)b * d.B, d.B, s_red);
      rec = !tau_reuse(args.gate, M);
    }
    if (args.active) rec = false;  // LoSA: stream the active rows' union pages, no residual
    if (tid == 0) {
      s_M = M;
      s_recompute = rec ? 1 : 0;
    }
    for (int r = tid; r < RT; r += blockDim.x) s_flags[r] = (r < rows_valid && rec) ? 1 : 0;
  }
  // Reuse: this split's share of the union pages of the group.
  if (tid < 32) {
    const uint32_t* ub = args.union_bits + (size_t)bg * args.words;
    int tot = 0;
    for (int w = lane; w < args.words; w += 32) tot += __popc(ub[w]);
    tot = warp_sum_int(tot);
    if (lane == 0) s_union_total = tot;
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], NCW);
    }
    mbar_init(&comb_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool recompute = s_recompute != 0;
  // Work in pages: recompute = all pages; reuse = the union pages, in page order.
  const int total_pages = recompute ? args.P : s_union_total;
  const int total_tiles = (total_pages + kTilePages - 1) / kTilePages;
  const int tps = (total_tiles + plan.splits - 1) / plan.splits;
  const int t_begin = min(total_tiles, split * tps), t_end = min(total_tiles, t_begin + tps);
  const int ntiles = t_end - t_begin;

  if (warp == C::kProducerWarp) {
    // ---------------- producer: page loads into the ring ----------------
    const uint32_t* ub = args.union_bits + (size_t)bg * args.words;
    int wcur = 0, seen = 0;  // reuse: the word holding this split's first union page, pages before it
    if (!recompute && ntiles > 0) {
      // The whole warp locates the (t_begin * 4)-th union page: popcounts of 32 words
      // at a time, an inclusive warp scan, and the first word whose running count
      // passes the target.
      const int target = t_begin * kTilePages;
      int base = 0;
      bool found = false;
      for (int w0 = 0; w0 < args.words && !found; w0 += 32) {
        const int c = (w0 + lane < args.words) ? __popc(__ldg(ub + w0 + lane)) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, base + incl > target);
        if (hit) {
          const int L = __ffs(hit) - 1;
          wcur = w0 + L;
          seen = base + __shfl_sync(0xffffffffu, incl - c, L);
          found = true;
        } else {
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      if (!found) {
        wcur = args.words;
        seen = base;
      }
    }
    if (lane == 0 && ntiles > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmK4);
      prefetch_tmap(&tmV4);
      int cur = t_begin * kTilePages;  // index among the pages of the work list
      int wbits = 0;                   // union enumeration cursor (word wcur)
      if (!recompute) {
        wbits = wcur < args.words ? (int)__ldg(ub + wcur) : 0;
        for (int skip = cur - seen; skip > 0; --skip) wbits &= wbits - 1;
      }
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, args.err, DEV_ERR_WAIT_EMPTY)) break;
        int pg[kTilePages];
        int nvalid = 0;
#pragma unroll
        for (int j = 0; j < kTilePages; ++j) {
          int page = -1;
          if (cur < total_pages) {
            if (recompute) {
              page = cur;
            } else {
              while (wbits == 0 && wcur + 1 < args.words) wbits = (int)__ldg(ub + (++wcur));
              page = wcur * 32 + (__ffs(wbits) - 1);
              wbits &= wbits - 1;
            }
            ++cur;
            ++nvalid;
          }
          pg[j] = page;
          s_pages[s][j] = page;
        }
        // Every slot is loaded: an empty slot reads page P, entirely past the last key,
        // which the TMA fills with zeros (its scores are masked; P V must not see
        // stale shared memory).
        (void)nvalid;
        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)kTilePages * 2u * C::kPageBytes);
        uint8_t* st = smem + s * C::kStageBytes;
        bool run = pg[0] >= 0;  // four consecutive pages: one 64-row box per half
#pragma unroll
        for (int j = 1; j < kTilePages; ++j) run = run && pg[j] == pg[0] + j;
        if (run) {
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            tma_load_3d(st + h * (kTilePages * kPage * 128), &tmK4, &full_bar[s], h * 64, pg[0] * kPage, bg);
            tma_load_3d(st + C::kTileBytes + h * (kTilePages * kPage * 128), &tmV4, &full_bar[s], h * 64,
                        pg[0] * kPage, bg);
          }
        } else {
#pragma unroll
          for (int j = 0; j < kTilePages; ++j) {
            const int row = (pg[j] >= 0 ? pg[j] : args.P) * kPage;
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
              const int off = h * (kTilePages * kPage * 128) + j * (kPage * 128);
              tma_load_3d(st + off, &tmK, &full_bar[s], h * 64, row, bg);
              tma_load_3d(st + C::kTileBytes + off, &tmV, &full_bar[s], h * 64, row, bg);
            }
          }
        }
        ++issued;
      }
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_wait_bounded(&full_bar[i % STAGES], (uint32_t)(i / STAGES) & 1u, args.err, DEV_ERR_WAIT_FULL);
    }
    return;
  }

  const size_t rs = (size_t)D + 4;
  if (warp == C::kAuxWarp) {
    // this split's share of the tile's in-block rows, parked in the workspace
    const int per = (rows_valid + plan.splits - 1) / plan.splits;
    const int r0 = min(rows_valid, split * per), r1 = min(rows_valid, r0 + per);
    inblock_rows_to_ws<bf16, D>(d, q, static_cast<const bf16*>(args.step.k_blk),
                                static_cast<const bf16*>(args.step.v_blk), b, kvh, row0, r0, r1,
                                args.inblock + unit * RT * rs, 0, 1, lane, smem + C::kAuxOff);
  } else {
    // ---------------------------- consumers ----------------------------
    const int wm = warp / WARPS_N, wn = warp - (warp / WARPS_N) * WARPS_N;
    const int c = lane & 3;
    const int r0 = wm * 16 + (lane >> 2), r1 = r0 + 8;
    // LoSA: rows of stable tokens take no key (their scores are all masked)
    auto row_active = [&](int r) -> bool {
      if (!args.active) return true;
      const size_t grow = grow0 + min(r, rows_valid - 1);
      return args.active[(size_t)b * d.B + grow % d.B] != 0;
    };
    const bool act0 = row_active(r0), act1 = row_active(r1);
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
    // The tile rows' selection bitmaps, in shared memory when they fit.
    const bool bits_smem = RT * args.words <= kBitsWords;
    if (bits_smem) {
      for (int i = tid; i < RT * args.words; i += NCW * 32) {
        const int r = i / args.words, wd = i - r * args.words;
        s_bits[i] = __ldg(args.sel_bits + (grow0 + min(r, rows_valid - 1)) * (size_t)args.words + wd);
      }
      named_barrier_sync(kBarConsumers, NCW * 32);
    }
    auto row_sel = [&](int r, int page) -> bool {
      const int rr = min(r, rows_valid - 1);
      const uint32_t w = bits_smem ? s_bits[rr * args.words + (page >> 5)]
                                   : __ldg(args.sel_bits + (grow0 + rr) * (size_t)args.words + (page >> 5));
      return (w >> (page & 31)) & 1u;
    };
    Acc<D> As, Ar;
    As.init();
    Ar.init();
    const float sl2 = d.scale * 1.4426950408889634f;
    // The tile loop, compiled twice: reuse steps keep only the selected set's state
    // live, recompute steps both sets.
    auto tile_loop = [&](auto dual_tag) {
      constexpr bool kDual = decltype(dual_tag)::value;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait_bounded(&full_bar[s], (uint32_t)(i / STAGES) & 1u, args.err, DEV_ERR_WAIT_FULL)) break;
        const uint32_t sK = smem_u32(smem + s * C::kStageBytes);
        const uint32_t sV = sK + C::kTileBytes;
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
            ldsm_x4(sK + pswz(key, dd, D), b0, b1, b2, b3);
            mma_bf16_16816(sc[n], qf[kk], b0, b1);
            mma_bf16_16816(sc[n + 1], qf[kk], b2, b3);
          }
        }
        // Route each score to the selected or the residual set of its row.
        bool sm[KW / 8][4];
#pragma unroll
        for (int n = 0; n < KW / 8; ++n) {
          const int colb = wn * KW + n * 8;
          const int page = s_pages[s][colb >> 4];
          const bool sel0 = page >= 0 && act0 && row_sel(r0, page);
          const bool sel1 = page >= 0 && act1 && row_sel(r1, page);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const long long key = (long long)page * kPage + (colb & 15) + 2 * c + (j & 1);
            const bool valid = page >= 0 && key < d.N;
            const bool sel = j < 2 ? sel0 : sel1;
            sm[n][j] = sel;
            // reuse steps: the selected set only; recompute: every valid key in one of the two
            sc[n][j] = (valid && (sel || kDual)) ? sc[n][j] * sl2 : -CUDART_INF_F;
          }
        }
        if constexpr (kDual)
          softmax_pv_dual<D, KW>(As, Ar, sc, sm, sV, wn, lane);
        else
          softmax_pv<D, KW>(As, sc, sV, wn, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
      }
    };
    if (recompute)
      tile_loop(std::true_type{});
    else
      tile_loop(std::false_type{});
    As.l0 += __shfl_xor_sync(0xffffffffu, As.l0, 1);
    As.l0 += __shfl_xor_sync(0xffffffffu, As.l0, 2);
    As.l1 += __shfl_xor_sync(0xffffffffu, As.l1, 1);
    As.l1 += __shfl_xor_sync(0xffffffffu, As.l1, 2);
    Ar.l0 += __shfl_xor_sync(0xffffffffu, Ar.l0, 1);
    Ar.l0 += __shfl_xor_sync(0xffffffffu, Ar.l0, 2);
    Ar.l1 += __shfl_xor_sync(0xffffffffu, Ar.l1, 1);
    Ar.l1 += __shfl_xor_sync(0xffffffffu, Ar.l1, 2);
    named_barrier_sync(kBarConsumers, NCW * 32);
    float* scr_s = reinterpret_cast<float*>(smem);
    float* scr_r = scr_s + (size_t)NCW * 16 * (D + 2);
    stash<D>(scr_s, warp, lane, As);
    stash<D>(scr_r, warp, lane, Ar);
    named_barrier_sync(kBarConsumers, NCW * 32);
    write_partial<D, WARPS_M, WARPS_N>(scr_s, args.part_sel + (unit * plan.splits + split) * RT * rs, tid);
    if (recompute)
      write_partial<D, WARPS_M, WARPS_N>(scr_r, args.part_res + (unit * plan.splits + split) * RT * rs, tid);
  }

  // ---- consumers + aux: once every split has arrived, combine this CTA's rows ----
  const int ftid = warp < NCW ? tid : NCW * 32 + lane;
  {
    int r0, r1;
    split_rows(rows_valid, plan.splits, split, r0, r1);
    sparse_coop_rows<D, C::kFinishThreads>(args, unit, RT, r0, r1, grow0, recompute, smem, C::kRingBytes, &comb_bar,
                                           ftid, kBarFinish);
  }
  if (args.gate.enabled && !args.active && split == 0) {
    for (int r = ftid; r < rows_valid; r += C::kFinishThreads) {
      const int gr = row0 + r;
      if ((r == 0 || gr % d.B == 0) && args.step.dec_reuse)
        args.step.dec_reuse[(size_t)b * d.hq + kvh * d.G + gr / d.B] = recompute ? 0 : 1;
    }
    if (ftid == 0 && kvh == 0 && rt == 0 && args.step.dec_M) args.step.dec_M[b] = s_M;
  }
}

template <int D, int WM, int WN, int STAGES>
cudaError_t launch_sparse_cfg(const SparseArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& tk4, const CUtensorMap& tv4, cudaStream_t s) {
  using C = SCfg<D, WM, WN, STAGES>;
  auto kern = sparse_pass_kernel<D, WM, WN, STAGES>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.plan.splits, a.plan.n_row_tiles, a.d.b * a.d.hkv);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the split CTAs of a tile wait for one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.plan.splits > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, tk4, tv4, a);
}

}  // namespace

bool losa_score_in_estimate(const Dims& d) { return d.B * d.hq <= kEstScoreMax && d.B <= kSmallBlockMax; }

int sparse_supported(int D, int row_tile) { return (D == 64 || D == 128) && (row_tile == 16 || row_tile == 32); }

cudaError_t launch_token_mse(const Dims& d, const void* q, const void* q_prev, float delta, float* mse,
                             uint8_t* active, cudaStream_t s) {
  const int threads = d.hq < 32 ? 32 : (d.hq > 256 ? 256 : (d.hq + 31) / 32 * 32);
  token_mse_kernel<<<dim3(d.B, d.b), threads, (size_t)d.hq * sizeof(double), s>>>(
      d, static_cast<const bf16*>(q), static_cast<const bf16*>(q_prev), delta, mse, active);
  return cudaGetLastError();
}

cudaError_t launch_page_minmax(const SparseArgs& a, cudaStream_t s) {
  if (a.P <= a.p_first) return cudaSuccess;
  dim3 grid((a.P - a.p_first + 31) / 32, a.d.b * a.d.hkv);
  if (a.d.D == 128)
    page_minmax_kernel<128><<<grid, 32 * 8, 0, s>>>(a);
  else if (a.d.D == 64)
    page_minmax_kernel<64><<<grid, 32 * 4, 0, s>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_sparse_select(const SparseArgs& a, cudaStream_t s) {
  const size_t est_smem = (size_t)((a.d.R + kEstRows - 1) / kEstRows * kEstRows) * a.d.D * 2 * sizeof(double) +
                          (size_t)kEstAhead * 2 * kEstThreads * sizeof(uint32_t);
  dim3 g1((a.P + kEstPages - 1) / kEstPages, a.d.b * a.d.hkv, (a.d.R + kEstRows - 1) / kEstRows);
  cudaError_t e;
  if (a.d.D == 128) {
    e = cudaFuncSetAttribute(page_estimate_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)est_smem);
    if (e != cudaSuccess) return e;
    page_estimate_kernel<128><<<g1, kEstThreads, est_smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(page_estimate_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)est_smem);
    if (e != cudaSuccess) return e;
    page_estimate_kernel<64><<<g1, kEstThreads, est_smem, s>>>(a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t bits_smem = (size_t)a.words * sizeof(uint32_t);
  const bool regs = a.P <= 8 * kTopkThreads;
  auto kern = regs ? topk_kernel<8> : topk_kernel<0>;
  if (bits_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bits_smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<a.d.b * a.d.hq * a.d.B, kTopkThreads, bits_smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_pass(const SparseArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tk4, const CUtensorMap& tv4, cudaStream_t s) {
  const int D = a.d.D, rt = a.plan.row_tile;
  if (D == 128) {
    if (rt == 16) return launch_sparse_cfg<128, 1, 4, 6>(a, tk, tv, tk4, tv4, s);
    if (rt == 32) return launch_sparse_cfg<128, 2, 2, 6>(a, tk, tv, tk4, tv4, s);
  } else if (D == 64) {
    if (rt == 16) return launch_sparse_cfg<64, 1, 4, 6>(a, tk, tv, tk4, tv4, s);
    if (rt == 32) return launch_sparse_cfg<64, 2, 2, 6>(a, tk, tv, tk4, tv4, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fb
