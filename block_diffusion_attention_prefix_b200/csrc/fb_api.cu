// fb_api.cu -- the C-ABI of libfb (declared in include/fb.h): argument
// validation, split-KV planning, TMA descriptor encoding and kernel dispatch.
//
// Every entry point validates on the host and returns a negative fb_status
// before launching anything.  No entry point allocates device memory or
// synchronises the stream (fb_device_error excepted).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fb.h"
#include "fb_internal.h"

namespace fb {

__device__ uint32_t g_device_error;  // bounded-wait timeouts (see fb_ptx.cuh)

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
uint32_t* g_err_ptr[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

int device_sms(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

uint32_t* device_err(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_err_ptr[dev];
}

bool get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Small cache of encoded tensor maps: a step re-encodes the same K/V maps every
// call otherwise.  Keyed by every input of the encoding.
struct MapKey {
  const void* base;
  long long keys, row_stride, head_stride;
  int D, bh, box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && keys == o.keys && row_stride == o.row_stride && head_stride == o.head_stride &&
           D == o.D && bh == o.bh && box_rows == o.box_rows;
  }
};
constexpr int kMapCache = 16;
MapKey g_map_keys[kMapCache];
CUtensorMap g_map_vals[kMapCache];
int g_map_used = 0, g_map_next = 0;

int encode_kv_map_uncached(CUtensorMap* m, const void* base, int D, long long keys, long long row_stride,
                           long long head_stride, int bh, int box_rows);

// 3-D map over a bf16 KV tensor: (D, keys, b*H_kv), box (64, box_rows, 1), 128-B swizzle.
int encode_kv_map(CUtensorMap* m, const void* base, int D, long long keys, long long row_stride,
                  long long head_stride, int bh, int box_rows = 64) {
  std::memset(m, 0, sizeof(*m));
  if (keys == 0) return FB_OK;  // never loaded
  const MapKey key{base, keys, row_stride, head_stride, D, bh, box_rows};
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_map_used; ++i)
      if (g_map_keys[i] == key) {
        *m = g_map_vals[i];
        return FB_OK;
      }
  }
  const int st = encode_kv_map_uncached(m, base, D, keys, row_stride, head_stride, bh, box_rows);
  if (st != FB_OK) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  const int slot = g_map_used < kMapCache ? g_map_used++ : (g_map_next++ % kMapCache);
  g_map_keys[slot] = key;
  g_map_vals[slot] = *m;
  return FB_OK;
}

int encode_kv_map_uncached(CUtensorMap* m, const void* base, int D, long long keys, long long row_stride,
                           long long head_stride, int bh, int box_rows) {
  if (!get_encoder()) return FB_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)keys, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)head_stride * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FB_OK : FB_ERR_CUDA;
}

int resolve(const fb_shape* s, Dims* d) {
  if (!s) return FB_ERR_NULL;
  if (s->dtype != FB_F32 && s->dtype != FB_BF16) return FB_ERR_DTYPE;
  if (s->batch < 1 || s->h_q < 1 || s->h_kv < 1 || s->block < 1 || s->n_prefix < 0) return FB_ERR_SHAPE;
  if (s->h_q % s->h_kv) return FB_ERR_SHAPE;
  if (s->dtype == FB_BF16) {
    if (s->head_dim != 64 && s->head_dim != 128) return FB_ERR_UNSUPPORTED;
  } else {
    if (s->head_dim < 32 || s->head_dim > 128 || s->head_dim % 32) return FB_ERR_UNSUPPORTED;
  }
  if ((long long)s->batch * s->h_kv > 65535) return FB_ERR_SHAPE;
  if ((long long)s->block * (s->h_q / s->h_kv) > (1LL << 24)) return FB_ERR_SHAPE;
  if (s->n_prefix > (1LL << 31) - 64) return FB_ERR_SHAPE;
  const long long rs = s->kv_row_stride ? s->kv_row_stride : s->head_dim;
  if (rs < s->head_dim) return FB_ERR_SHAPE;
  const long long hs = s->kv_head_stride ? s->kv_head_stride : s->n_prefix * rs;
  if (s->n_prefix > 0 && hs < (s->n_prefix - 1) * rs + s->head_dim) return FB_ERR_SHAPE;
  const int eb = s->dtype == FB_BF16 ? 2 : 4;
  if ((rs * eb) % 16 || (hs * eb) % 16) return FB_ERR_ALIGN;
  if (!(s->scale >= 0.f) || std::isinf(s->scale)) return FB_ERR_ARG;
  d->b = s->batch;
  d->hq = s->h_q;
  d->hkv = s->h_kv;
  d->G = s->h_q / s->h_kv;
  d->D = s->head_dim;
  d->B = s->block;
  d->N = s->n_prefix;
  d->row_stride = rs;
  d->head_stride = hs;
  d->scale = s->scale > 0.f ? s->scale : 1.f / std::sqrt((float)s->head_dim);
  d->dtype = s->dtype;
  d->R = d->G * d->B;
  return FB_OK;
}

int check_ptr(const void* p) {
  if (!p) return FB_ERR_NULL;
  return aligned16(p) ? FB_OK : FB_ERR_ALIGN;
}

int gate_params(const fb_gate* g, const Dims& d, GateParams* gp) {
  std::memset(gp, 0, sizeof(*gp));
  if (!g) return FB_OK;
  if (!g->updated_mask) return FB_ERR_NULL;
  if (g->head_sim && !aligned16(g->head_sim)) return FB_ERR_ALIGN;
  if (!std::isfinite(g->gamma) && g->head_sim) return FB_ERR_ARG;
  gp->mask = g->updated_mask;
  gp->sim = g->head_sim;
  gp->enabled = 1;
  gp->first = g->first_step ? 1 : 0;
  gp->tau = g->tau;
  gp->gamma = g->gamma;
  (void)d;
  return FB_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? FB_OK : FB_ERR_CUDA; }

#define FB_TRY(x)            \
  do {                       \
    const int _st = (x);     \
    if (_st != FB_OK) return _st; \
  } while (0)

// One split-KV attention pass over `keys` keys (prefix or large in-block).
int run_pass(const Dims& d0, long long keys, const void* q, const void* k, const void* v, long long row_stride,
             long long head_stride, const GateParams& gp, const Epilogue& ep, void* ws, size_t ws_bytes,
             cudaStream_t stream, const StepArgs* step = nullptr) {
  if (!ws) return FB_ERR_WORKSPACE;
  if (!aligned16(ws)) return FB_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return FB_ERR_CUDA;
  const int sms = device_sms(dev);
  uint32_t* err = device_err(dev);
  if (!sms || !err) return FB_ERR_CUDA;
  Dims d = d0;
  d.N = keys;
  d.row_stride = row_stride;
  d.head_stride = head_stride;
  PassArgs a;
  a.d = d;
  const bool fused = step != nullptr && step->enabled;
  a.plan = plan_split(d.R, d.D, keys, d.b, d.hkv, d.dtype, sms, fused, true, fused);
  if (a.plan.n_row_tiles > 65535) return FB_ERR_SHAPE;
  if (ws_bytes < a.plan.total()) return FB_ERR_WORKSPACE;
  a.q = q;
  a.k = k;
  a.v = v;
  a.gate = gp;
  a.ep = ep;
  if (step)
    a.step = *step;
  else
    std::memset(&a.step, 0, sizeof(a.step));
  a.counters = static_cast<unsigned int*>(ws);
  a.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + a.plan.counter_bytes);
  a.inblock = a.plan.inblock_bytes
                  ? reinterpret_cast<float*>(static_cast<char*>(ws) + a.plan.counter_bytes + a.plan.partial_bytes)
                  : nullptr;
  a.err = err;
  if (a.plan.reuse_rows) {
    // Batched fused step: every reusing row (and the decision record) first, in the
    // light kernel; the pass then only touches tiles with a row that recomputes.
    if (!reuse_rows_supported(d.dtype, d.D)) return FB_ERR_UNSUPPORTED;
    a.step.reuse_done = 1;
    FB_TRY(cuda_status(launch_reuse_rows(a, stream)));
  }
  if (a.plan.tc) {
    // Dense contraction (more than 16 query rows per KV head): tcgen05 + TMEM.
    CUtensorMap tq, tk, tv;
    const long long qrows = (long long)d.b * d.hq * d.B;
    FB_TRY(encode_kv_map(&tq, q, d.D, qrows, d.D, qrows * d.D, 1, 128));
    FB_TRY(encode_kv_map(&tk, k, d.D, keys, row_stride, head_stride, d.b * d.hkv, a.plan.key_tile));
    FB_TRY(encode_kv_map(&tv, v, d.D, keys, row_stride, head_stride, d.b * d.hkv, a.plan.key_tile));
    return cuda_status(launch_pass_tc(a, tq, tk, tv, stream));
  }
  if (d.dtype == FB_BF16) {
    if (!bf16_pass_supported(d.D, a.plan.row_tile)) return FB_ERR_UNSUPPORTED;
    CUtensorMap tk, tv;
    FB_TRY(encode_kv_map(&tk, k, d.D, keys, row_stride, head_stride, d.b * d.hkv));
    FB_TRY(encode_kv_map(&tv, v, d.D, keys, row_stride, head_stride, d.b * d.hkv));
    return cuda_status(launch_pass_bf16(a, tk, tv, stream));
  }
  return cuda_status(launch_pass_f32(a, stream));
}

size_t pass_bytes(const Dims& d, long long keys, bool with_inblock = false) {
  const int dev = current_device();
  const int sms = dev >= 0 ? device_sms(dev) : 0;
  return plan_split(d.R, d.D, keys, d.b, d.hkv, d.dtype, sms > 0 ? sms : 148, with_inblock, true, with_inblock)
      .total();
}

}  // namespace

SplitPlan plan_split(int R, int D, long long N, int b, int hkv, int dtype, int num_sms, bool with_inblock,
                     bool allow_tc, bool batch_reuse) {
  SplitPlan p;
  std::memset(&p, 0, sizeof(p));
  if (batch_reuse && with_inblock) {
    // Batched fused step: when the units (on the mma.sync / fp32 row tiles) fill two
    // waves or more, every tile is one split, the reuse-rows kernel writes the
    // reusing rows, and bf16 runs persistent CTAs that skip tiles whose rows all reuse.
    const int rt = dtype == FB_BF16 ? (R <= 16 ? 16 : (R <= 32 ? 32 : 64)) : 16;
    const long long n_rt = (R + rt - 1) / rt;
    const long long units = (long long)b * hkv * n_rt;
    const long long wave = (long long)num_sms * (dtype == FB_BF16 ? 1 : 4);
    if (units >= 2 * wave) {
      p.row_tile = rt;
      p.n_row_tiles = (int)n_rt;
      p.key_tile = dtype == FB_BF16 ? 64 : 32;
      p.splits = 1;
      p.tiles_per_split = (int)((N + p.key_tile - 1) / p.key_tile);
      p.reuse_rows = 1;
      if (dtype == FB_BF16) {
        p.persistent = 1;
        const long long min_grid = (units + kMaxUnitsPerCta - 1) / kMaxUnitsPerCta;
        p.grid = (int)std::max<long long>(std::min<long long>(units, num_sms), min_grid);
      }
      p.counter_bytes = ((size_t)units * 2 * 4 + 255) / 256 * 256;
      p.partial_bytes = (size_t)units * p.row_tile * (D + 4) * sizeof(float);
      p.inblock_bytes = (size_t)units * p.row_tile * (D + 4) * sizeof(float);
      return p;
    }
  }
  if (dtype == FB_BF16) {
    // More than 16 packed query rows per KV head make the tiles a real dense
    // contraction: tcgen05 (M = 128, rows past the tile padded); otherwise mma.sync.
    p.tc = (allow_tc && D == 128 && R > 16) ? 1 : 0;
    p.row_tile = p.tc ? (R <= 32 ? 32 : (R <= 64 ? 64 : 128)) : (R <= 16 ? 16 : (R <= 32 ? 32 : 64));
    p.key_tile = p.tc ? 128 : 64;
  } else {
    p.row_tile = 16;
    p.key_tile = 32;
  }
  const int ctas_per_sm = dtype == FB_BF16 ? 1 : 4;
  p.n_row_tiles = (R + p.row_tile - 1) / p.row_tile;
  const long long units = (long long)b * hkv * p.n_row_tiles;
  const long long total_tiles = (N + p.key_tile - 1) / p.key_tile;
  long long target = (long long)num_sms * ctas_per_sm;
  if (p.tc && p.row_tile == 128 && !with_inblock && units >= target) {
    // Enough row tiles to fill the GPU: one CTA per row tile over all keys, no combine.
    p.tc = 2;
    p.splits = 1;
    p.tiles_per_split = (int)total_tiles;
    p.counter_bytes = 256;  // unused; keeps the workspace non-empty
    return p;
  }
  long long splits = units > 0 ? target / units : 1;
  if (splits < 1) splits = 1;
  if (total_tiles > 0 && splits > total_tiles) splits = total_tiles;
  if (total_tiles > 0) {
    p.tiles_per_split = (int)((total_tiles + splits - 1) / splits);
    p.splits = (int)((total_tiles + p.tiles_per_split - 1) / p.tiles_per_split);
  } else {
    p.tiles_per_split = 0;
    p.splits = 1;
  }
  p.counter_bytes = ((size_t)units * 2 * 4 + 255) / 256 * 256;
  p.partial_bytes = (size_t)units * p.splits * p.row_tile * (D + 4) * sizeof(float);
  p.inblock_bytes = with_inblock ? (size_t)units * p.row_tile * (D + 4) * sizeof(float) : 0;
  return p;
}

}  // namespace fb

using namespace fb;

extern "C" {

int fb_version(void) { return 100; }

const char* fb_status_string(int status) {
  switch (status) {
    case FB_OK: return "ok";
    case FB_ERR_NULL: return "required pointer is NULL";
    case FB_ERR_SHAPE: return "sizes out of range or inconsistent";
    case FB_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case FB_ERR_DTYPE: return "dtype not supported";
    case FB_ERR_WORKSPACE: return "workspace missing or too small";
    case FB_ERR_CUDA: return "CUDA call failed";
    case FB_ERR_UNSUPPORTED: return "configuration not implemented";
    case FB_ERR_ARG: return "invalid argument";
    default: return "unknown status";
  }
}

int fb_device_error(int32_t* code) {
  if (!code) return FB_ERR_NULL;
  const int dev = current_device();
  if (dev < 0) return FB_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return FB_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FB_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FB_ERR_CUDA;
  *code = (int32_t)v;
  return FB_OK;
}

size_t fb_workspace_bytes(const fb_shape* shape) {
  Dims d;
  if (resolve(shape, &d) != FB_OK) return 0;
  size_t n = pass_bytes(d, d.N, d.B <= kSmallBlockMax);
  if (d.B > kSmallBlockMax) {
    const size_t nb = pass_bytes(d, d.B);
    if (nb > n) n = nb;
  }
  return n;
}

int fb_workspace_init(void* ws, size_t ws_bytes, fb_stream_t stream) {
  if (!ws) return FB_ERR_NULL;
  return cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}

int fb_gate_eval(const fb_shape* shape, const fb_gate* gate, int32_t* dec_M, uint8_t* dec_reuse,
                 fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  if (!gate || (!dec_M && !dec_reuse)) return FB_ERR_NULL;
  GateParams gp;
  FB_TRY(gate_params(gate, d, &gp));
  return cuda_status(launch_gate_eval(d, gp, dec_M, dec_reuse, (cudaStream_t)stream));
}

int fb_prefix_attn(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache,
                   const fb_gate* gate, float* a_out, float* l_out, void* ws, size_t ws_bytes,
                   fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(a_out));
  FB_TRY(check_ptr(l_out));
  if (d.N > 0) {
    FB_TRY(check_ptr(k_cache));
    FB_TRY(check_ptr(v_cache));
  }
  GateParams gp;
  FB_TRY(gate_params(gate, d, &gp));
  Epilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 0;
  ep.a_dst = a_out;
  ep.l_dst = l_out;
  return run_pass(d, d.N, q, k_cache, v_cache, d.row_stride, d.head_stride, gp, ep, ws, ws_bytes,
                  (cudaStream_t)stream);
}

int fb_block_attn(const fb_shape* shape, const void* q, const void* k_blk, const void* v_blk, float* a_in,
                  float* l_in, void* ws, size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  FB_TRY(check_ptr(a_in));
  FB_TRY(check_ptr(l_in));
  Epilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 0;
  ep.a_dst = a_in;
  ep.l_dst = l_in;
  GateParams none;
  std::memset(&none, 0, sizeof(none));
  if (d.B <= kSmallBlockMax) {
    SmallBlockArgs a;
    a.d = d;
    a.q = q;
    a.k_blk = k_blk;
    a.v_blk = v_blk;
    a.gate = none;
    a.ep = ep;
    a.dec_M = nullptr;
    a.dec_reuse = nullptr;
    return cuda_status(launch_small_block(a, (cudaStream_t)stream));
  }
  return run_pass(d, d.B, q, k_blk, v_blk, d.D, (long long)d.B * d.D, none, ep, ws, ws_bytes,
                  (cudaStream_t)stream);
}

int fb_merge(const fb_shape* shape, const float* a1, const float* l1, const float* a2, const float* l2,
             void* a_full, float* l_full, fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(a1));
  FB_TRY(check_ptr(a2));
  FB_TRY(check_ptr(a_full));
  if (!l1 || !l2) return FB_ERR_NULL;
  return cuda_status(launch_merge(d, a1, l1, a2, l2, a_full, l_full, (cudaStream_t)stream));
}

int fb_exp2_fma(const float* x, float* y, int64_t n, fb_stream_t stream) {
  if (n == 0) return FB_OK;
  if (!x || !y) return FB_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u)) return FB_ERR_ALIGN;
  if (n < 0 || n >= (int64_t(1) << 31)) return FB_ERR_SHAPE;
  if (current_device() < 0) return FB_ERR_CUDA;
  return cuda_status(launch_exp2_fma(x, y, n, (cudaStream_t)stream));
}

int fb_merge_partials(const fb_shape* shape, const float* a_parts, int64_t a_part_stride, const float* l_parts,
                      int64_t l_part_stride, int n_parts, const fb_gate* gate, float* a_out, float* l_out,
                      fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(a_parts));
  FB_TRY(check_ptr(a_out));
  if (!l_parts || !l_out) return FB_ERR_NULL;
  if (n_parts < 1) return FB_ERR_ARG;
  const long long rows = (long long)d.b * d.hq * d.B;
  if (n_parts > 1 && (a_part_stride < rows * d.D || l_part_stride < rows)) return FB_ERR_SHAPE;
  if (a_part_stride % 4) return FB_ERR_ALIGN;  // every partial's A starts 16-byte aligned
  GateParams gp;
  FB_TRY(gate_params(gate, d, &gp));
  return cuda_status(launch_merge_parts(d, gp, a_parts, a_part_stride, l_parts, l_part_stride, n_parts, a_out,
                                        l_out, (cudaStream_t)stream));
}

int fb_block_merge(const fb_shape* shape, const void* q, const void* k_blk, const void* v_blk,
                   const fb_gate* gate, const float* a_out, const float* l_out, void* a_full, float* l_full,
                   int32_t* dec_M, uint8_t* dec_reuse, void* ws, size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  FB_TRY(check_ptr(a_out));
  FB_TRY(check_ptr(a_full));
  if (!l_out) return FB_ERR_NULL;
  GateParams gp;
  FB_TRY(gate_params(gate, d, &gp));
  if (!gp.enabled && (dec_M || dec_reuse)) return FB_ERR_NULL;
  Epilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 1;
  ep.a_prev = a_out;
  ep.l_prev = l_out;
  ep.a_full = a_full;
  ep.l_full = l_full;
  ep.out_bf16 = d.dtype == FB_BF16;
  if (d.B <= kSmallBlockMax) {
    SmallBlockArgs a;
    a.d = d;
    a.q = q;
    a.k_blk = k_blk;
    a.v_blk = v_blk;
    a.gate = gp;
    a.ep = ep;
    a.dec_M = dec_M;
    a.dec_reuse = dec_reuse;
    return cuda_status(launch_small_block(a, (cudaStream_t)stream));
  }
  if (gp.enabled && (dec_M || dec_reuse))
    FB_TRY(cuda_status(launch_gate_eval(d, gp, dec_M, dec_reuse, (cudaStream_t)stream)));
  GateParams none;
  std::memset(&none, 0, sizeof(none));
  return run_pass(d, d.B, q, k_blk, v_blk, d.D, (long long)d.B * d.D, none, ep, ws, ws_bytes,
                  (cudaStream_t)stream);
}

int fb_step(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache, const void* k_blk,
            const void* v_blk, const fb_gate* gate, float* a_out, float* l_out, void* a_full, float* l_full,
            int32_t* dec_M, uint8_t* dec_reuse, void* ws, size_t ws_bytes, fb_stream_t stream) {
  if (!gate) return FB_ERR_NULL;
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  FB_TRY(check_ptr(a_full));
  if (ws_bytes < fb_workspace_bytes(shape)) return FB_ERR_WORKSPACE;
  if (d.B <= kSmallBlockMax) {
    // One launch: the prefix pass (gated) whose finishing CTAs also run the
    // in-block pass, the merge and the decision record.
    FB_TRY(check_ptr(q));
    FB_TRY(check_ptr(a_out));
    FB_TRY(check_ptr(l_out));
    if (d.N > 0) {
      FB_TRY(check_ptr(k_cache));
      FB_TRY(check_ptr(v_cache));
    }
    GateParams gp;
    FB_TRY(gate_params(gate, d, &gp));
    Epilogue ep;
    std::memset(&ep, 0, sizeof(ep));
    ep.mode = 0;
    ep.a_dst = a_out;
    ep.l_dst = l_out;
    StepArgs st;
    std::memset(&st, 0, sizeof(st));
    st.enabled = 1;
    st.k_blk = k_blk;
    st.v_blk = v_blk;
    st.a_full = a_full;
    st.l_full = l_full;
    st.dec_M = dec_M;
    st.dec_reuse = dec_reuse;
    return run_pass(d, d.N, q, k_cache, v_cache, d.row_stride, d.head_stride, gp, ep, ws, ws_bytes,
                    (cudaStream_t)stream, &st);
  }
  FB_TRY(fb_prefix_attn(shape, q, k_cache, v_cache, gate, a_out, l_out, ws, ws_bytes, stream));
  return fb_block_merge(shape, q, k_blk, v_blk, gate, a_out, l_out, a_full, l_full, dec_M, dec_reuse, ws,
                        ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Sparse attention with a cached residual.
namespace fb {
namespace {

constexpr int kSparsePage = 16;

struct SparseLayout {
  SplitPlan plan;
  int P, words;
  size_t counters, part_sel, part_res, inblock, est, total;
};

int sparse_layout(const Dims& d, int sms, SparseLayout* L) {
  L->plan = plan_split(d.R, d.D, d.N, d.b, d.hkv, FB_BF16, sms, true, false);
  L->P = (int)((d.N + kSparsePage - 1) / kSparsePage);
  L->words = (L->P + 31) / 32;
  const size_t units = (size_t)d.b * d.hkv * L->plan.n_row_tiles;
  const size_t part = units * L->plan.splits * L->plan.row_tile * (d.D + 4) * sizeof(float);
  L->counters = 0;
  L->part_sel = L->plan.counter_bytes;
  L->part_res = L->part_sel + part;
  L->inblock = L->part_res + part;
  L->est = L->inblock + (units * L->plan.row_tile * (d.D + 4) * sizeof(float) + 255) / 256 * 256;
  L->total = L->est + (size_t)d.b * d.hq * d.B * L->P * sizeof(double);
  return FB_OK;
}

// Pages the K cache's row capacity holds (rows r with r * row_stride + D <=
// head_stride, at least N), rounded up to a multiple of 8: the page stride of the
// bounds layout, so that every channel row of the bounds starts on 16 bytes.
int page_capacity(const Dims& d) {
  long long rows = d.row_stride > 0 ? (d.head_stride - d.D) / d.row_stride + 1 : d.N;
  if (rows < d.N) rows = d.N;
  const long long pages = (rows + kSparsePage - 1) / kSparsePage;
  return (int)((pages + 7) / 8 * 8);
}

int sparse_check(const fb_shape* shape, const fb_gate* gate, const fb_sparse* sp, Dims* d, GateParams* gp) {
  FB_TRY(resolve(shape, d));
  if (!sp) return FB_ERR_NULL;
  if (d->dtype != FB_BF16) return FB_ERR_DTYPE;
  if (sp->page_size != kSparsePage) return FB_ERR_ARG;
  if (d->N < 1 || d->B > kSmallBlockMax || d->R > 32) return FB_ERR_UNSUPPORTED;
  const long long P = (d->N + kSparsePage - 1) / kSparsePage;
  if (sp->n_select < 1 || sp->n_select > P) return FB_ERR_ARG;
  if ((P + 31) / 32 > 12288) return FB_ERR_UNSUPPORTED;  // row bitmap must fit in shared memory
  if (gate && gate->head_sim) return FB_ERR_UNSUPPORTED;  // tau gate only
  FB_TRY(check_ptr(sp->kmin));
  FB_TRY(check_ptr(sp->kmax));
  FB_TRY(check_ptr(sp->sel_idx));
  FB_TRY(check_ptr(sp->sel_bits));
  FB_TRY(check_ptr(sp->union_bits));
  FB_TRY(check_ptr(sp->a_res));
  FB_TRY(check_ptr(sp->l_res));
  if (sp->a_sel) FB_TRY(check_ptr(sp->a_sel));
  return gate_params(gate, *d, gp);
}

int sparse_args(const Dims& d, const GateParams& gp, const fb_sparse* sp, const void* q, void* ws,
                size_t ws_bytes, SparseArgs* a) {
  if (!ws) return FB_ERR_WORKSPACE;
  if (!aligned16(ws)) return FB_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return FB_ERR_CUDA;
  const int sms = device_sms(dev);
  uint32_t* err = device_err(dev);
  if (!sms || !err) return FB_ERR_CUDA;
  SparseLayout L;
  sparse_layout(d, sms, &L);
  if (ws_bytes < L.total) return FB_ERR_WORKSPACE;
  if (!sparse_supported(d.D, L.plan.row_tile)) return FB_ERR_UNSUPPORTED;
  std::memset(a, 0, sizeof(*a));
  a->d = d;
  a->plan = L.plan;
  a->P = L.P;
  a->Pcap = page_capacity(d);
  a->k_sel = sp->n_select;
  a->words = L.words;
  a->q = q;
  a->kmin = static_cast<const __nv_bfloat16*>(sp->kmin);
  a->kmax = static_cast<const __nv_bfloat16*>(sp->kmax);
  char* w = static_cast<char*>(ws);
  a->counters = reinterpret_cast<unsigned int*>(w + L.counters);
  a->part_sel = reinterpret_cast<float*>(w + L.part_sel);
  a->part_res = reinterpret_cast<float*>(w + L.part_res);
  a->inblock = reinterpret_cast<float*>(w + L.inblock);
  a->est = reinterpret_cast<double*>(w + L.est);
  a->sel_idx = sp->sel_idx;
  a->sel_bits = sp->sel_bits;
  a->union_bits = sp->union_bits;
  a->gate = gp;
  a->a_res = sp->a_res;
  a->l_res = sp->l_res;
  a->a_sel = sp->a_sel;
  a->l_sel = sp->l_sel;
  a->err = err;
  return FB_OK;
}

}  // namespace
}  // namespace fb

extern "C" int fb_page_cap(const fb_shape* shape, int page_size) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  if (page_size != kSparsePage) return FB_ERR_ARG;
  if (d.N < 1) return FB_ERR_UNSUPPORTED;
  return page_capacity(d);
}

extern "C" int fb_page_minmax(const fb_shape* shape, const void* k_cache, int page_size, void* kmin, void* kmax,
                              fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  if (d.dtype != FB_BF16) return FB_ERR_DTYPE;
  if (page_size != kSparsePage) return FB_ERR_ARG;
  if (d.N < 1) return FB_ERR_UNSUPPORTED;
  FB_TRY(check_ptr(k_cache));
  FB_TRY(check_ptr(kmin));
  FB_TRY(check_ptr(kmax));
  SparseArgs a;
  std::memset(&a, 0, sizeof(a));
  a.d = d;
  a.P = (int)((d.N + kSparsePage - 1) / kSparsePage);
  a.Pcap = page_capacity(d);
  a.p_first = 0;
  a.k = k_cache;
  a.kmin_out = static_cast<__nv_bfloat16*>(kmin);
  a.kmax_out = static_cast<__nv_bfloat16*>(kmax);
  return cuda_status(launch_page_minmax(a, (cudaStream_t)stream));
}

extern "C" int fb_losa_step(const fb_shape* shape, const void* q, const void* q_prev, const void* k_cache,
                            const void* v_cache, const void* k_blk, const void* v_blk, float delta,
                            const fb_sparse* sp, void* a_full, float* l_full, float* mse, uint8_t* dec_active,
                            void* ws, size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  GateParams gp;
  FB_TRY(sparse_check(shape, nullptr, sp, &d, &gp));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(q_prev));
  FB_TRY(check_ptr(k_cache));
  FB_TRY(check_ptr(v_cache));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  if (!a_full || !dec_active) return FB_ERR_NULL;
  if (!(delta == delta)) return FB_ERR_ARG;  // NaN threshold
  SparseArgs a;
  FB_TRY(sparse_args(d, gp, sp, q, ws, ws_bytes, &a));
  a.active = dec_active;
  a.step.enabled = 1;
  a.step.k_blk = k_blk;
  a.step.v_blk = v_blk;
  a.step.a_full = a_full;
  a.step.l_full = l_full;
  a.step.dec_M = nullptr;
  a.step.dec_reuse = nullptr;
  CUtensorMap tk, tv, tk4, tv4;
  FB_TRY(encode_kv_map(&tk, k_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, kSparsePage));
  FB_TRY(encode_kv_map(&tv, v_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, kSparsePage));
  FB_TRY(encode_kv_map(&tk4, k_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, 4 * kSparsePage));
  FB_TRY(encode_kv_map(&tv4, v_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, 4 * kSparsePage));
  if (losa_score_in_estimate(d)) {
    // the page estimate scores the tokens itself (one launch fewer)
    a.q_prev = q_prev;
    a.delta = delta;
    a.mse = mse;
    a.active_out = dec_active;
  } else {
    FB_TRY(cuda_status(launch_token_mse(d, q, q_prev, delta, mse, dec_active, (cudaStream_t)stream)));
  }
  FB_TRY(cuda_status(launch_sparse_select(a, (cudaStream_t)stream)));
  return cuda_status(launch_sparse_pass(a, tk, tv, tk4, tv4, (cudaStream_t)stream));
}

extern "C" size_t fb_similarity_workspace_bytes(const fb_shape* shape) {
  Dims d;
  if (resolve(shape, &d) != FB_OK) return 0;
  return similarity_bytes(d);
}

extern "C" int fb_head_similarity(const fb_shape* shape, const void* q, const void* q_ref, float* sim, void* ws,
                                  size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(q_ref));
  if (!sim) return FB_ERR_NULL;
  if (!ws) return FB_ERR_WORKSPACE;
  if (!aligned16(ws)) return FB_ERR_ALIGN;
  if (ws_bytes < similarity_bytes(d)) return FB_ERR_WORKSPACE;
  return cuda_status(launch_similarity(d, q, q_ref, sim, ws, (cudaStream_t)stream));
}

extern "C" int fb_refresh_reference(const fb_shape* shape, const void* q, void* q_ref, const uint8_t* dec_reuse,
                                    fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(q_ref));
  if (!dec_reuse) return FB_ERR_NULL;
  return cuda_status(launch_refresh(d, q, q_ref, dec_reuse, (cudaStream_t)stream));
}

extern "C" int fb_append_block(const fb_shape* shape, void* k_cache, void* v_cache, const void* k_blk,
                               const void* v_blk, int page_size, void* kmin, void* kmax, fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  if (!shape->kv_head_stride) return FB_ERR_SHAPE;  // a contiguous cache has no room to grow
  // Row capacity per head: rows r with r * row_stride + D <= head_stride.
  const long long cap = (d.head_stride - d.D) / d.row_stride + 1;
  if (d.N + d.B > cap || d.N + d.B > (1LL << 31) - 64) return FB_ERR_SHAPE;
  FB_TRY(check_ptr(k_cache));
  FB_TRY(check_ptr(v_cache));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  const bool bounds = kmin || kmax;
  if (bounds) {
    if (d.dtype != FB_BF16) return FB_ERR_DTYPE;
    if (page_size != kSparsePage) return FB_ERR_ARG;
    FB_TRY(check_ptr(kmin));
    FB_TRY(check_ptr(kmax));
  }
  FB_TRY(cuda_status(launch_append_block(d, k_cache, v_cache, k_blk, v_blk, (cudaStream_t)stream)));
  if (!bounds) return FB_OK;
  // Page bounds of the grown prefix: only the pages the new rows fall in change
  // (the first may be a partial page that already holds old rows).
  SparseArgs a;
  std::memset(&a, 0, sizeof(a));
  a.d = d;
  a.d.N = d.N + d.B;
  a.P = (int)((a.d.N + kSparsePage - 1) / kSparsePage);
  a.Pcap = page_capacity(a.d);
  a.p_first = (int)(d.N / kSparsePage);
  a.k = k_cache;
  a.kmin_out = static_cast<__nv_bfloat16*>(kmin);
  a.kmax_out = static_cast<__nv_bfloat16*>(kmax);
  return cuda_status(launch_page_minmax(a, (cudaStream_t)stream));
}

extern "C" size_t fb_sparse_workspace_bytes(const fb_shape* shape, int page_size) {
  Dims d;
  if (resolve(shape, &d) != FB_OK || page_size != kSparsePage) return 0;
  const int dev = current_device();
  const int sms = dev >= 0 ? device_sms(dev) : 0;
  SparseLayout L;
  sparse_layout(d, sms > 0 ? sms : 148, &L);
  return L.total;
}

extern "C" int fb_sparse_select(const fb_shape* shape, const void* q, const fb_gate* gate, const fb_sparse* sp,
                                void* ws, size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  GateParams gp;
  FB_TRY(sparse_check(shape, gate, sp, &d, &gp));
  FB_TRY(check_ptr(q));
  SparseArgs a;
  FB_TRY(sparse_args(d, gp, sp, q, ws, ws_bytes, &a));
  return cuda_status(launch_sparse_select(a, (cudaStream_t)stream));
}

extern "C" int fb_sparse_step(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache,
                              const void* k_blk, const void* v_blk, const fb_gate* gate, const fb_sparse* sp,
                              void* a_full, float* l_full, int32_t* dec_M, uint8_t* dec_reuse, void* ws,
                              size_t ws_bytes, fb_stream_t stream) {
  Dims d;
  GateParams gp;
  FB_TRY(sparse_check(shape, gate, sp, &d, &gp));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(k_cache));
  FB_TRY(check_ptr(v_cache));
  FB_TRY(check_ptr(k_blk));
  FB_TRY(check_ptr(v_blk));
  FB_TRY(check_ptr(a_full));
  SparseArgs a;
  FB_TRY(sparse_args(d, gp, sp, q, ws, ws_bytes, &a));
  a.step.enabled = 1;
  a.step.k_blk = k_blk;
  a.step.v_blk = v_blk;
  a.step.a_full = a_full;
  a.step.l_full = l_full;
  a.step.dec_M = dec_M;
  a.step.dec_reuse = dec_reuse;
  CUtensorMap tk, tv;
  FB_TRY(encode_kv_map(&tk, k_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, kSparsePage));
  FB_TRY(encode_kv_map(&tv, v_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, kSparsePage));
  CUtensorMap tk4, tv4;
  FB_TRY(encode_kv_map(&tk4, k_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, 4 * kSparsePage));
  FB_TRY(encode_kv_map(&tv4, v_cache, d.D, d.N, d.row_stride, d.head_stride, d.b * d.hkv, 4 * kSparsePage));
  FB_TRY(cuda_status(launch_sparse_select(a, (cudaStream_t)stream)));
  return cuda_status(launch_sparse_pass(a, tk, tv, tk4, tv4, (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------
// fb_prefix_attn_noalloc: the prefix pass with its split-KV workspace in a
// library-owned static device array, for callers that cannot allocate.
namespace fb {
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[FB_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a stand-in, so the address is looked up on every call (a
// host-side query; nothing is cached that a device reset could leave stale).
int static_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess || !p) return FB_ERR_CUDA;
  *out = p;
  return FB_OK;
}

}  // namespace
}  // namespace fb

extern "C" int fb_prefix_attn_noalloc(const fb_shape* shape, const void* q, const void* k_cache,
                                      const void* v_cache, const fb_gate* gate, float* a_out, float* l_out,
                                      fb_stream_t stream) {
  Dims d;
  FB_TRY(resolve(shape, &d));
  FB_TRY(check_ptr(q));
  FB_TRY(check_ptr(a_out));
  FB_TRY(check_ptr(l_out));
  if (d.N > 0) {
    FB_TRY(check_ptr(k_cache));
    FB_TRY(check_ptr(v_cache));
  }
  GateParams gp;
  FB_TRY(gate_params(gate, d, &gp));
  const int dev = current_device();
  if (dev < 0) return FB_ERR_CUDA;
  const int sms = device_sms(dev);
  if (!sms) return FB_ERR_CUDA;
  const SplitPlan plan = plan_split(d.R, d.D, d.N, d.b, d.hkv, d.dtype, sms);
  if (plan.total() > (size_t)FB_STATIC_SCRATCH_BYTES) return FB_ERR_WORKSPACE;
  void* ws = nullptr;
  FB_TRY(static_scratch(&ws));
  // The array keeps the previous call's contents: the arrival counters must start at zero.
  if (cudaMemsetAsync(ws, 0, plan.counter_bytes, (cudaStream_t)stream) != cudaSuccess) return FB_ERR_CUDA;
  Epilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 0;
  ep.a_dst = a_out;
  ep.l_dst = l_out;
  return run_pass(d, d.N, q, k_cache, v_cache, d.row_stride, d.head_stride, gp, ep, ws,
                  (size_t)FB_STATIC_SCRATCH_BYTES, (cudaStream_t)stream);
}
