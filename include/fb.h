/*
 * fb.h -- C-ABI of libfb: cached block-diffusion attention (FlashBlock) on B200.
 *
 * What it computes.  "Technical summary: FlashBlock" (gist.science, paper
 * 2602.05305), section "2. Methodology / Core mechanism": for each query of the
 * current block, attention splits into an out-of-block part over the prefix KV
 * cache (J_out) and an in-block part over the block's own keys (J_in).  The
 * out-of-block output A_out and its log-normaliser L_out = log Z_out are cached
 * and reused by later denoising steps, and each step recombines them with the
 * fresh in-block (A_in, L_in) in log space:
 *     m = max(L_out, L_in)
 *     A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}).
 * Section "Adaptive reuse strategies" gates the reuse: by a threshold tau on the
 * number of updated tokens M^{s+1} (reuse iff M < tau), by a per-head similarity
 * threshold gamma in the video setting (only heads whose similarity is above
 * gamma reuse), and optionally by caching the attention over the keys a sparse
 * selector leaves out (fb_sparse_* below).
 *
 * Conventions shared by every entry point.
 *  - Pointers named q, k_*, v_*, a_*, l_*, dec_*, ws, mask, sim are DEVICE
 *    pointers owned by the caller; the library never allocates, frees or keeps
 *    them.  `fb_shape` and `fb_gate` structs are HOST memory, read during the call.
 *  - Layouts (row-major, innermost last; b = batch, H_q query heads, H_kv KV heads,
 *    G = H_q / H_kv, B = block size, N = prefix length, D = head_dim):
 *        Q, A_full            [b, H_q, B, D]       dtype of the shape (fp32 or bf16)
 *        prefix K, V          [b, H_kv, N, D]      dtype; row stride kv_row_stride,
 *                                                  head stride kv_head_stride (elements)
 *        in-block K, V        [b, H_kv, B, D]      dtype, contiguous
 *        A_out, A_in (cache)  [b, H_q, B, D]       fp32
 *        L_out, L_in, L_full  [b, H_q, B]          fp32, natural log
 *        updated mask         [b, B]               uint8, nonzero = updated this step
 *        head similarity      [b, H_q]             fp32
 *        dec_M                [b]                  int32, M^{s+1}
 *        dec_reuse            [b, H_q]             uint8, 1 = cache reused
 *    Query head h reads KV head h / G.  Q, A and the in-block tensors are
 *    contiguous.  All device pointers must be 16-byte aligned.
 *  - An empty key set has L = -inf and A = 0.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Arguments are validated on the host first: a negative fb_status is
 *    returned and nothing is launched.  FB_ERR_CUDA means a launch failed
 *    (cudaGetLastError); kernels report a bounded-wait timeout through
 *    fb_device_error().  NaN or Inf inputs give undefined (but memory-safe) results.
 *  - Calls that write the same outputs must not overlap on the GPU.
 */
#ifndef FB_H_
#define FB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fb_stream_t; /* identical to cudaStream_t */

typedef enum fb_status {
  FB_OK = 0,
  FB_ERR_NULL = -1,        /* a required pointer is NULL */
  FB_ERR_SHAPE = -2,       /* sizes out of range or inconsistent */
  FB_ERR_ALIGN = -3,       /* pointer or stride not 16-byte aligned */
  FB_ERR_DTYPE = -4,       /* dtype not supported for this call */
  FB_ERR_WORKSPACE = -5,   /* workspace missing or smaller than fb_workspace_bytes() */
  FB_ERR_CUDA = -6,        /* a CUDA runtime/driver call failed */
  FB_ERR_UNSUPPORTED = -7, /* valid request the library does not implement */
  FB_ERR_ARG = -8          /* other invalid argument (e.g. page size, k) */
} fb_status;

typedef enum fb_dtype { FB_F32 = 0, FB_BF16 = 1 } fb_dtype;

/* Problem sizes of one attention layer.  head_dim must be 64 or 128 for bf16 and
 * a multiple of 32 up to 128 for fp32.  kv_row_stride / kv_head_stride of 0 mean
 * "contiguous" (head_dim and n_prefix * kv_row_stride).  scale of 0 means
 * 1/sqrt(head_dim) (the pages leave the temperature open; this is the standard one). */
typedef struct fb_shape {
  int32_t batch;
  int32_t h_q;
  int32_t h_kv;
  int32_t head_dim;
  int32_t block;          /* B: queries per step and in-block keys */
  int32_t dtype;          /* fb_dtype of Q, K, V and A_full */
  int64_t n_prefix;       /* N: prefix tokens (J_out), may be 0 */
  int64_t kv_row_stride;  /* elements between consecutive prefix tokens */
  int64_t kv_head_stride; /* elements between consecutive KV heads; batch stride is h_kv times it */
  float scale;            /* softmax temperature */
} fb_shape;

/* Reuse gate of one denoising step (FlashBlock, "Adaptive reuse strategies").
 *   M[b]        = number of nonzero entries of updated_mask[b, 0..B-1]
 *   reuse[b, h] = !first_step && M[b] < tau && (head_sim == NULL || head_sim[b, h] > gamma)
 * Step 0 of a block always recomputes (there is no cache yet).  tau <= 0 disables
 * reuse; tau > B disables the threshold.  head_sim == NULL disables the per-head
 * gate.  The comparisons are strict, and gamma is compared in fp32. */
typedef struct fb_gate {
  const uint8_t* updated_mask; /* device [b, B], required */
  const float* head_sim;       /* device [b, H_q] or NULL */
  int32_t first_step;
  int32_t tau;
  float gamma;
} fb_gate;

/* Library version (major*10000 + minor*100 + patch) and status strings. */
int fb_version(void);
const char* fb_status_string(int status);

/* Reads and clears the device error word of the current device: 0 if no kernel
 * hit a wait bound since the last call, else a nonzero code: 1 a tile load did not
 * arrive, 2 the producer found no free stage, 3 the bulk copy of split partials did
 * not arrive, 4 the split CTAs of a tile (or the grid) did not all arrive.  Each wait
 * gives up after 2 s.  Synchronises the current device.  After a nonzero code the
 * outputs of the failed calls are undefined and workspaces should be re-initialised
 * (fb_workspace_init). */
int fb_device_error(int32_t* code);

/* Workspace (device bytes) needed by fb_prefix_attn / fb_step / fb_block_merge for
 * this shape: split-KV partials plus arrival counters.  The counters must be zero
 * before the first use of a workspace (fb_workspace_init does it); every call
 * leaves them zero again, so a workspace is reusable across calls on one stream. */
size_t fb_workspace_bytes(const fb_shape* shape);
int fb_workspace_init(void* ws, size_t ws_bytes, fb_stream_t stream);

/* Gate only (the updated-token count, the tau gate and the per-head gamma gate):
 * writes dec_M [b] and dec_reuse [b, H_q]. */
int fb_gate_eval(const fb_shape* shape, const fb_gate* gate, int32_t* dec_M, uint8_t* dec_reuse,
                 fb_stream_t stream);

/* Out-of-block attention (split-KV pass, split combine, cache write).  Passage:
 * FlashBlock technical summary, "2. Methodology / Core mechanism" -- A_out and
 * L_out = log Z_out over J_out (the tokens outside the current block), computed
 * once and cached.  (A_out, L_out) of every query row over the whole prefix J_out,
 * computed split-KV and reduced in log space.  With gate == NULL every row is
 * recomputed; otherwise only rows of heads whose decision is
 * "recompute" are written, and rows of reusing heads are left bit-for-bit
 * untouched (the decision is taken on the device; no host synchronisation).
 * ws: fb_workspace_bytes(shape) bytes. */
int fb_prefix_attn(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache,
                   const fb_gate* gate, float* a_out, float* l_out, void* ws, size_t ws_bytes,
                   fb_stream_t stream);

/* In-block attention.  Passage: FlashBlock technical summary, "2. Methodology /
 * Core mechanism" -- the part over J_in, the tokens of the current block, that
 * every denoising step computes afresh.  (A_in, L_in) of every query row over the
 * B block keys, bidirectional (no mask).  ws may be NULL when block <= 64; larger blocks need
 * fb_workspace_bytes(shape) bytes. */
int fb_block_attn(const fb_shape* shape, const void* q, const void* k_blk, const void* v_blk,
                  float* a_in, float* l_in, void* ws, size_t ws_bytes, fb_stream_t stream);

/* Log-space merge.  Passage: FlashBlock technical summary, "2. Methodology /
 * Core mechanism", the merge equation (also the split-KV reduction: every split is
 * a subset of J_out).  Elementwise over [b, H_q, B] rows:
 * A_full = merge((a1, l1), (a2, l2)) in the shape's dtype; l_full (nullable) gets
 * m + ln(e^{l1-m} + e^{l2-m}).  Two empty inputs give (0, -inf). */
int fb_merge(const fb_shape* shape, const float* a1, const float* l1, const float* a2,
             const float* l2, void* a_full, float* l_full, fb_stream_t stream);

/* Context-parallel combine of the out-of-block part.  Passage: FlashBlock
 * technical summary, "2. Methodology / Core mechanism", the merge equation: the
 * log-space merge of partial results over disjoint key sets is the result over
 * their union, so J_out may be cut into P key ranges -- one per GPU, each GPU
 * holding its range of the prefix K/V -- whose partial (A, L) are computed apart
 * (fb_prefix_attn on the range) and merged here.  Partial p (p = 0 .. n_parts-1)
 * is A_p = a_parts + p * a_part_stride ([b, H_q, B, D] fp32) and L_p = l_parts +
 * p * l_part_stride ([b, H_q, B] fp32, natural log); the caller gathers them into
 * these buffers (e.g. one all-gather).  For every row of a head whose gate decision
 * is "recompute" (every row when gate == NULL):
 *     M = max_p L_p,  e_p = e^{L_p - M},  den = sum_p e_p   (p ascending)
 *     A_out = (sum_p e_p A_p) / den,  L_out = M + ln den
 * written to a_out / l_out (the cache); rows of reusing heads are left untouched.
 * Empty ranges (L = -inf) are allowed; all empty gives (0, -inf).  The merge runs
 * in range order, so the result does not depend on timing.  a_part_stride must be
 * a multiple of 4 (16-byte aligned partials) and, with n_parts > 1, at least
 * b*H_q*B*D; l_part_stride at least b*H_q*B. */
int fb_merge_partials(const fb_shape* shape, const float* a_parts, int64_t a_part_stride,
                      const float* l_parts, int64_t l_part_stride, int n_parts, const fb_gate* gate,
                      float* a_out, float* l_out, fb_stream_t stream);

/* Second half of a step (gate, in-block attention, merge): evaluates the gate, records dec_M /
 * dec_reuse (nullable), computes (A_in, L_in) and merges it with the cache
 * (a_out, l_out) as it is in memory, writing A_full and L_full (nullable).
 * gate may be NULL (then no decision is recorded).  ws as for fb_block_attn. */
int fb_block_merge(const fb_shape* shape, const void* q, const void* k_blk, const void* v_blk,
                   const fb_gate* gate, const float* a_out, const float* l_out, void* a_full,
                   float* l_full, int32_t* dec_M, uint8_t* dec_reuse, void* ws, size_t ws_bytes,
                   fb_stream_t stream);

/* One denoising step of one attention layer.  Passages: FlashBlock technical
 * summary, "2. Methodology / Core mechanism" (cache, in-block part, merge) and
 * "Adaptive reuse strategies" (the tau and gamma gates that decide whether the
 * cache is reused).  fb_prefix_attn(gate) refreshes the
 * cache rows that recompute, then fb_block_merge writes A_full, L_full and the
 * decisions.  On a reuse step the prefix K/V are not read.  gate is required. */
int fb_step(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache,
            const void* k_blk, const void* v_blk, const fb_gate* gate, float* a_out,
            float* l_out, void* a_full, float* l_full, int32_t* dec_M, uint8_t* dec_reuse,
            void* ws, size_t ws_bytes, fb_stream_t stream);

/* ---------------------------------------------------------------------------
 * Sparse attention with a cached residual (FlashBlock, "Adaptive reuse
 * strategies / compatibility with sparse attention"): the keys a sparse selector
 * leaves out are the "out-of-block" set whose attention is cached (the
 * residual); the selected keys are attended fresh every step:
 *     A_full = merge(merge(A_sel, A_res), A_in).
 * Selector (the pages name QUEST as one, without defining it; this is the plain
 * page-bound reading): prefix pages of 16 tokens; per page and channel the
 * min / max of K; for each query row the page estimate
 *     e_p = sum_d max(q_d kmin_{p,d}, q_d kmax_{p,d})   (float64, ascending d)
 * and the top n_select pages by (e desc, page asc).  On a recompute step (first
 * step of the block, or M >= tau) the selection is redone and frozen and the
 * residual is recomputed with the current queries; on a reuse step only the
 * union of the KV group's selected pages is read.  Supported: bf16, head_dim 64
 * or 128, page_size 16, block * (h_q / h_kv) <= 32, block <= 64, n_prefix >= 1,
 * the tau gate only (head_sim must be NULL).  words = ceil(n_pages / 32),
 * n_pages = ceil(n_prefix / 16).  All buffers are caller-owned device memory. */
typedef struct fb_sparse {
  int32_t page_size;      /* 16 */
  int32_t n_select;       /* pages per query row, 1 .. n_pages */
  const void* kmin;       /* [b, H_kv, D, page_cap] bf16 page minima (fb_page_minmax), pages
                             [0, n_pages) valid; page_cap (fb_page_cap) = ceil(cap / page_size)
                             rounded up to a multiple of 8 (16-byte channel rows), with cap
                             the K cache's row capacity per head (rows r with
                             r * kv_row_stride + head_dim <= kv_head_stride; = n_prefix for a
                             contiguous cache), so the layout survives fb_append_block */
  const void* kmax;       /* same layout, page maxima */
  int32_t* sel_idx;       /* state [b, H_q, B, n_select] int32, selected pages ascending */
  uint32_t* sel_bits;     /* state [b, H_q, B, words] bitmap of the same pages */
  uint32_t* union_bits;   /* state [b, H_kv, words] union over the KV group's rows */
  float* a_res;           /* state: residual cache [b, H_q, B, D] fp32 */
  float* l_res;           /* state: [b, H_q, B] fp32, natural log */
  float* a_sel;           /* optional output (fresh part) [b, H_q, B, D] fp32, or NULL */
  float* l_sel;           /* optional output [b, H_q, B], or NULL */
} fb_sparse;

/* The page stride page_cap of the bounds layout (see fb_sparse.kmin) for this
 * shape: > 0 and a multiple of 8, or a negative fb_status (bad shape,
 * page_size != 16, n_prefix < 1).
 * Host only; allocate kmin / kmax as [b, H_kv, D, page_cap] bf16. */
int fb_page_cap(const fb_shape* shape, int page_size);

/* Channel-wise page bounds of the prefix keys (exact bf16 min / max over each
 * page's real tokens; the last page may be partial). */
int fb_page_minmax(const fb_shape* shape, const void* k_cache, int page_size, void* kmin, void* kmax,
                   fb_stream_t stream);

/* LoSA-style step (after a block's first step, which runs fb_step densely with
 * sp->a_res / sp->l_res as its cache A_out / L_out).  "LoSA: Locality Aware Sparse
 * Attention for Block-Wise Diffusion Language Models" (gist.science 2604.12056),
 * "2. Methodology": tokens whose queries moved (active) get sparse attention over
 * the prefix, stable tokens reuse the prefix attention of the previous step, and
 * the KV pages loaded are the union over the active tokens only.
 *   1. score[b, i] = mean over heads and channels of (q - q_prev)^2 (float64, fixed
 *      order: per head ascending d, heads ascending; float32 result) -> `mse`
 *      (nullable); dec_active[b, i] = score > delta;
 *   2. every row (head) of an active token: page estimates and top-k as in
 *      fb_sparse_select (sel_idx / sel_bits rows of stable tokens are not written);
 *      union_bits = union over the active rows of each KV group;
 *   3. one pass over the union pages: active rows get (A, L) over their selected
 *      pages, which overwrites their cache row in sp->a_res / sp->l_res; stable rows
 *      keep theirs; A_full = merge(cache row, in-block row) for every row.
 * q, q_prev [b, H_q, B, D] bf16; the other arguments as in fb_sparse_step (gate
 * none: the score decides).  Workspace: fb_sparse_workspace_bytes. */
int fb_losa_step(const fb_shape* shape, const void* q, const void* q_prev, const void* k_cache,
                 const void* v_cache, const void* k_blk, const void* v_blk, float delta, const fb_sparse* sp,
                 void* a_full, float* l_full, float* mse, uint8_t* dec_active, void* ws, size_t ws_bytes,
                 fb_stream_t stream);

/* Per-head similarity estimate for the gamma gate.  FlashBlock technical summary
 * (gist.science 2602.05305), "Adaptive reuse strategies": in the video setting only
 * heads whose estimated cross-step similarity is above gamma reuse their cache; the
 * pages give no estimator.  This one: sim[b, h] = cosine between the head's block
 * queries q [b, H_q, B, D] and the reference queries q_ref (same layout and dtype:
 * the queries the head's cache was last computed with), i.e.
 * <Q, R> / sqrt(<Q, Q> <R, R>) in float64 rounded to float32 (0 when a norm is 0).
 * The sums run in one plain order -- each row's products in ascending d give the
 * row's dot product, and the row dot products are added one after another in
 * ascending row order -- so the result, and the gate decision sim > gamma taken on
 * it, is reproducible bit for bit.  sim [b, H_q]
 * float32 device memory, then usable as fb_gate.head_sim.  Workspace: at least
 * fb_similarity_workspace_bytes(shape) bytes (arrival counters and 32 bytes per
 * query row), zeroed once (fb_workspace_init); its counters return to zero after
 * each call.  Asynchronous on `stream`. */
size_t fb_similarity_workspace_bytes(const fb_shape* shape);
int fb_head_similarity(const fb_shape* shape, const void* q, const void* q_ref, float* sim, void* ws,
                       size_t ws_bytes, fb_stream_t stream);

/* After a step: heads that recomputed (dec_reuse[b, h] == 0, as written by fb_step)
 * copy their block queries q into q_ref; heads that reused keep their reference. */
int fb_refresh_reference(const fb_shape* shape, const void* q, void* q_ref, const uint8_t* dec_reuse,
                         fb_stream_t stream);

/* Block transition (after the last denoising step of a block): the block's tokens
 * join the prefix.  FlashBlock technical summary (gist.science 2602.05305),
 * "1. Problem definition": attention splits into the current block J_in and the
 * tokens outside it, J_out, which are the earlier blocks -- so when a block is
 * finished its keys and values are appended to the prefix cache and the next
 * block's J_out is one block longer.
 *
 * shape->n_prefix is N before the call; k_blk / v_blk ([b, H_kv, B, D], the block's
 * keys and values as of its last step) are copied into cache rows [N, N + B) of
 * every (b, KV head).  The cache must have room: shape->kv_head_stride must be
 * given (non-zero) and hold at least N + B rows of kv_row_stride (FB_ERR_SHAPE
 * otherwise).  When kmin / kmax are non-NULL (bf16, page_size 16; layout as in
 * fb_sparse, with the page stride of the capacity) the page bounds of the pages
 * the new rows fall in are recomputed over their real tokens; other pages keep
 * theirs.  Afterwards the caller uses n_prefix = N + B.  The cached (A_out,
 * L_out) of the finished block is stale for the next block, whose step 0
 * recomputes it (first_step).  All pointers caller-owned device memory,
 * 16-byte aligned; asynchronous on `stream`. */
int fb_append_block(const fb_shape* shape, void* k_cache, void* v_cache, const void* k_blk, const void* v_blk,
                    int page_size, void* kmin, void* kmax, fb_stream_t stream);

/* Workspace of fb_sparse_select / fb_sparse_step (split partials of both parts,
 * in-block rows, page estimates, counters; same reuse rules as fb_workspace_bytes). */
size_t fb_sparse_workspace_bytes(const fb_shape* shape, int page_size);

/* Selection only: for batch elements whose gate says recompute, page estimates and
 * top-k -> sel_idx, sel_bits, union_bits.  Others keep their state untouched. */
int fb_sparse_select(const fb_shape* shape, const void* q, const fb_gate* gate, const fb_sparse* sp,
                     void* ws, size_t ws_bytes, fb_stream_t stream);

/* One denoising step in sparse mode: fb_sparse_select, then the sparse pass that
 * writes the residual cache (recompute), A_full, L_full (nullable) and the
 * decisions (nullable). */
int fb_sparse_step(const fb_shape* shape, const void* q, const void* k_cache, const void* v_cache,
                   const void* k_blk, const void* v_blk, const fb_gate* gate, const fb_sparse* sp,
                   void* a_full, float* l_full, int32_t* dec_M, uint8_t* dec_reuse, void* ws,
                   size_t ws_bytes, fb_stream_t stream);

/* Out-of-block attention for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is a deployment variant of fb_prefix_attn.
 * Some callers cannot call cudaMalloc (or any allocator) at the point where they
 * run attention -- for example code running under a fixed memory budget whose
 * pools are already carved up, or hosts that forbid allocation on their hot path.
 * They cannot provide the split-KV workspace that fb_prefix_attn takes, so this
 * entry point keeps it in library-owned device memory instead: a file-scope
 * static device array of FB_STATIC_SCRATCH_BYTES, which every GPU that loads the
 * library holds until the process exits.  Nothing is allocated or freed by the
 * call.  The caller still passes q, the KV cache and the outputs, with the same
 * meaning, layout and gate as fb_prefix_attn.
 *
 *  - Shapes whose prefix-pass scratch exceeds FB_STATIC_SCRATCH_BYTES are
 *    rejected with FB_ERR_WORKSPACE before any launch.  The limit applies to the
 *    split-KV scratch of the prefix pass alone -- what fb_prefix_attn itself uses
 *    for the shape -- which can be smaller than fb_workspace_bytes(shape): that
 *    figure also covers the in-block rows of the fused step (fb_step).
 *  - Each call looks up the array's device address with the current device
 *    (a host-side query, so nothing goes stale after a device reset).  The first
 *    call on a device may load the library's device code: make it before any
 *    stream capture.
 *  - All calls on a device share the one array, and it keeps the last call's
 *    contents: each call first clears the arrival counters it needs on `stream`.
 *    Calls that overlap on the GPU (other streams, other threads) race on the
 *    array and give wrong results: serialise them. */
#define FB_STATIC_SCRATCH_BYTES (8u << 20)
int fb_prefix_attn_noalloc(const fb_shape* shape, const void* q, const void* k_cache,
                           const void* v_cache, const fb_gate* gate, float* a_out, float* l_out,
                           fb_stream_t stream);

/* Diagnostics: evaluates on the device, element by element, y[i] = 2^x[i] in the
 * arithmetic the tcgen05 attention pass uses for a quarter of its softmax
 * exponentials (those it keeps off the special-function unit): x = n + f with
 * n = round(x), a cubic in f fitted for the least largest relative error on
 * [-1/2, 1/2] with p(0) = 1, then n added to the exponent.  Relative error at
 * most 1.02e-4 for x in [-125, 2^22); exact at integers; 0 for x < -125 and -inf.
 * x and y are device arrays of n floats (they may alias; NULL when n == 0);
 * n >= 0.  For tests of that error bound.  FB_ERR_NULL, FB_ERR_ALIGN (4-byte alignment), FB_ERR_SHAPE
 * (n < 0 or n >= 2^31). */
int fb_exp2_fma(const float* x, float* y, int64_t n, fb_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FB_H_ */
