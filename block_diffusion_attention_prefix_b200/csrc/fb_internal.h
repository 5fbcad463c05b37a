// fb_internal.h -- declarations shared by the translation units of libfb.
//
// Plain structs passed by value to kernels, the split-KV workspace plan, and the
// launch functions each kernel file provides to the C-ABI layer (fb_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace fb {

// Largest block handled by the fused small-block code (scores on CUDA cores).
constexpr int kSmallBlockMax = 64;

// Largest number of row tiles a persistent pass CTA walks (its list of tiles that
// recompute lives in shared memory).
constexpr int kMaxUnitsPerCta = 1024;

// Gate of one denoising step, as device-readable arguments.  enabled == 0 means
// "recompute every row" (no gate).  See fb_gate in include/fb.h.
struct GateParams {
  const uint8_t* mask;  // [b, B]
  const float* sim;     // [b, H_q] or nullptr
  int enabled;
  int first;
  int tau;
  float gamma;
};

// Resolved problem sizes (strides in elements).
struct Dims {
  int b, hq, hkv, G, D, B;
  long long N;            // keys of the pass (prefix N, or B for an in-block pass)
  long long row_stride;   // elements between keys
  long long head_stride;  // elements between KV heads
  float scale;            // softmax temperature (natural units)
  int dtype;              // 0 = fp32, 1 = bf16
  int R;                  // query rows per KV head = G * B
};

// Split-KV plan of one attention pass over N keys for R rows per KV head.
struct SplitPlan {
  int row_tile;         // rows per CTA
  int n_row_tiles;      // ceil(R / row_tile)
  int key_tile;         // keys per pipeline tile
  int splits;           // CTAs along the key axis per (b, kv head, row tile)
  int tiles_per_split;  // key tiles per split
  int tc;               // 0: mma.sync / CUDA-core pass; 1: tcgen05 split pass; 2: tcgen05, one CTA per row tile
  int persistent;       // bf16 mma.sync pass, one split: a grid of `grid` CTAs that each walk their row tiles
  int grid;             // persistent: CTAs of the launch
  int reuse_rows;       // batched fused step: the reuse-rows kernel runs first (see plan_split)
  size_t counter_bytes; // arrival then departure counters, one each per (b, kv head, row tile), 256-B padded
  size_t partial_bytes; // [b*hkv][n_row_tiles][splits][row_tile][D + 4] fp32
  size_t inblock_bytes; // fused step only: [b*hkv][n_row_tiles][row_tile][D + 4] fp32 (A_in, L_in)
  size_t total() const { return counter_bytes + partial_bytes + inblock_bytes; }
};

// What the split combine of a (b, kv head, row tile) does with the combined rows.
struct Epilogue {
  int mode;               // 0: write (A, L) fp32 to a_dst / l_dst; 1: merge with (a_prev, l_prev)
  float* a_dst;           // mode 0, [b, H_q, B, D]
  float* l_dst;           // mode 0, [b, H_q, B]
  const float* a_prev;    // mode 1: cached (A_out, L_out)
  const float* l_prev;
  void* a_full;           // mode 1: output in the shape dtype
  float* l_full;          // mode 1: nullable
  int out_bf16;
};

// Fused-step extension of a prefix pass (blocks of at most kSmallBlockMax tokens):
// the CTA that finishes a (b, kv head, row tile) -- the last to arrive, or split
// 0 when every row of the tile reuses -- also computes the in-block attention of
// its rows, merges it with the cache into A_full / L_full and records the gate's
// decisions.  One launch is then one whole denoising step.
struct StepArgs {
  int enabled;
  const void* k_blk;      // [b, H_kv, B, D]
  const void* v_blk;
  void* a_full;           // [b, H_q, B, D] in the shape dtype
  float* l_full;          // nullable
  int32_t* dec_M;         // nullable
  uint8_t* dec_reuse;     // nullable
  int reuse_done;         // the reuse-rows kernel already wrote the reusing rows and the decisions
};

// Arguments of a split-KV attention pass (prefix, or in-block for large B).
struct PassArgs {
  Dims d;
  SplitPlan plan;
  const void* q;          // [b, H_q, B, D] in d.dtype
  const void* k;          // keys base (fp32 path reads through pointers; bf16 path uses TMA maps)
  const void* v;
  GateParams gate;
  Epilogue ep;
  StepArgs step;
  unsigned int* counters; // workspace
  float* partials;        // workspace
  float* inblock;         // workspace, fused step only
  uint32_t* err;          // device error word
};

// Page-sparse attention with a cached residual (sparse.cu).
struct SparseArgs {
  Dims d;                 // N = prefix tokens
  SplitPlan plan;         // splits over 64-key (4-page) tiles
  int P;                  // pages (16 tokens each)
  int Pcap;               // page stride of the bounds layout: pages the K cache's capacity holds
  int p_first;            // page_minmax: first page to (re)compute
  int k_sel;              // pages selected per query row
  int words;              // ceil(P / 32)
  const void* q;
  const void* k;          // prefix K (page bounds only)
  const __nv_bfloat16* kmin;   // [b*H_kv][D][Pcap], pages [0, P) valid
  const __nv_bfloat16* kmax;
  __nv_bfloat16* kmin_out;     // page bounds output
  __nv_bfloat16* kmax_out;
  double* est;            // workspace [b*H_q*B][P]
  int32_t* sel_idx;       // [b*H_q*B][k_sel] ascending
  uint32_t* sel_bits;     // [b*H_q*B][words]
  uint32_t* union_bits;   // [b*H_kv][words]
  GateParams gate;        // tau only
  const uint8_t* active;  // LoSA mode: token activity [b, B] (NULL otherwise)
  // LoSA mode with the locality score taken inside the page estimate (q_prev != NULL):
  // each estimate CTA scores its batch element's tokens, one CTA writes mse / active.
  const void* q_prev;     // [b, H_q, B, D] bf16, the previous step's queries
  float delta;            // activity threshold
  float* mse;             // optional output [b, B]
  uint8_t* active_out;    // output [b, B] (the same buffer as `active`)
  float* a_res;           // residual cache [b, H_q, B, D] / [b, H_q, B]
  float* l_res;
  float* a_sel;           // optional
  float* l_sel;
  StepArgs step;          // in-block, A_full, L_full, decisions
  unsigned int* counters; // workspace
  float* part_sel;
  float* part_res;
  float* inblock;
  uint32_t* err;
};
int sparse_supported(int D, int row_tile);
cudaError_t launch_page_minmax(const SparseArgs& a, cudaStream_t s);
// LoSA: per-token locality score (float32 [b, B], nullable) and activity (score > delta).
bool losa_score_in_estimate(const Dims& d);  // the page estimate can score the LoSA tokens itself
cudaError_t launch_token_mse(const Dims& d, const void* q, const void* q_prev, float delta, float* mse,
                             uint8_t* active, cudaStream_t s);
cudaError_t launch_sparse_select(const SparseArgs& a, cudaStream_t s);
// tk / tv: 16-row boxes (one page); tk4 / tv4: 64-row boxes (four consecutive pages).
cudaError_t launch_sparse_pass(const SparseArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tk4, const CUtensorMap& tv4, cudaStream_t s);

// batch_reuse: a fused step (fb_step) may take the batched plan -- when the (b, KV
// head, row tile) units fill two waves or more, the reuse-rows kernel writes every
// reusing row first and the pass (one split per tile, persistent CTAs for bf16)
// walks only the tiles that recompute.
SplitPlan plan_split(int R, int D, long long N, int b, int hkv, int dtype, int num_sms,
                     bool with_inblock = false, bool allow_tc = true, bool batch_reuse = false);

// Launchers (return cudaError_t of the launch).
cudaError_t launch_pass_f32(const PassArgs& a, cudaStream_t s);
cudaError_t launch_pass_bf16(const PassArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                             cudaStream_t s);
int bf16_pass_supported(int D, int row_tile);
// tcgen05 pass (flash_tc.cu): bf16, D = 128, more than 16 query rows per KV head.
cudaError_t launch_pass_tc(const PassArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           cudaStream_t s);

// Reusing rows of a step for many (b, KV head) groups at once (reuse.cu): the gate,
// the decisions, and A_full = merge(cache row, in-block row) for every row whose
// head reuses; one CTA per group, a warp per row.
cudaError_t launch_reuse_rows(const PassArgs& a, cudaStream_t s);
int reuse_rows_supported(int dtype, int D);

// Small in-block pass fused with gate and merge (B <= kSmallBlockMax).
struct SmallBlockArgs {
  Dims d;
  const void* q;
  const void* k_blk;
  const void* v_blk;
  GateParams gate;
  Epilogue ep;            // mode 0: write (A_in, L_in); mode 1: merge with the cache
  int32_t* dec_M;         // nullable
  uint8_t* dec_reuse;     // nullable
};
cudaError_t launch_small_block(const SmallBlockArgs& a, cudaStream_t s);
cudaError_t launch_gate_eval(const Dims& d, const GateParams& g, int32_t* dec_M, uint8_t* dec_reuse,
                             cudaStream_t s);
// Context-parallel combine: cache rows of recomputing heads = merge of P partials.
cudaError_t launch_exp2_fma(const float* x, float* y, long long n, cudaStream_t s);
cudaError_t launch_merge_parts(const Dims& d, const GateParams& g, const float* a_parts, long long a_stride,
                               const float* l_parts, long long l_stride, int P, float* a_out, float* l_out,
                               cudaStream_t s);
cudaError_t launch_merge(const Dims& d, const float* a1, const float* l1, const float* a2,
                         const float* l2, void* a_full, float* l_full, cudaStream_t s);
// Per-head similarity estimate (similarity.cu): workspace bytes, sim = cosine of
// Q and the reference queries; refresh of the reference for recomputed heads.
size_t similarity_bytes(const Dims& d);
cudaError_t launch_similarity(const Dims& d, const void* q, const void* q_ref, float* sim, void* ws, cudaStream_t s);
cudaError_t launch_refresh(const Dims& d, const void* q, void* q_ref, const uint8_t* dec_reuse, cudaStream_t s);
// Block transition: copy the block's K/V ([b, H_kv, B, D]) into cache rows [N, N + B).
cudaError_t launch_append_block(const Dims& d, void* k_cache, void* v_cache, const void* k_blk, const void* v_blk,
                                cudaStream_t s);

}  // namespace fb
