/*
 * lowram.h -- C ABI of the LowRAM compressed-KV-cache path for NVIDIA B200 (sm_100a).
 *
 * The method (LowRAM: low-rank keys and amortised values):
 *   - "LowRAM" project page, Figure 3: the keys of a group of adjacent layers are
 *     stored as one shared per-token factor A and a smaller per-layer factor, so
 *     the keys of layer l are A . B_l.
 *   - "Predicting the value cache from keys" explainer, paragraphs 2-4: values are
 *     not stored; a small per-KV-head network rebuilds them from the keys (a
 *     pseudoinverse-initialised linear map plus a GELU branch), and exact residual
 *     corrections are kept for the tokens it predicts worst, ranked by error.
 *   - arXiv 2611.07025 abstract: at each decode step only a selected subset of the
 *     cached pairs needs to be rebuilt (selective reconstruction).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller. The library never
 *     allocates device memory, never frees caller memory and keeps no state between
 *     calls; scratch space is the caller's workspace (`ws`, `ws_bytes`).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) in stream order. No entry point synchronises the host except
 *     lr_get_device_error.
 *   - Floating tensors all use the storage type `dtype` of the cache shape
 *     (LR_BF16 or LR_F32); arithmetic is fp32 with fp32 accumulation.
 *     Index tensors are int32. Every tensor is dense, row-major, with the
 *     dimensions listed (leftmost slowest).
 *   - Data pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - Host-side checks (null pointers, shapes, alignment, workspace size) run
 *     before any launch and return a status without touching device memory.
 *     LR_ERR_CUDA means a launch failed (cudaGetLastError). Device-side data
 *     checks (out-of-range or unsorted indices) skip the offending entry and set
 *     bits in an error word inside the workspace; read it with
 *     lr_get_device_error. No kernel traps or asserts, and every wait inside a
 *     kernel is bounded (on expiry the call's output is invalid and the error
 *     word gets LR_DEVERR_TIMEOUT).
 *   - The last failing host-side check's message is available, per thread, from
 *     lr_last_error().
 *   - Kernel families: decode calls on bf16 caches with hd = 128, H of 128 or 256,
 *     r a multiple of 64 and at most 8 query heads per KV head, and lr_pack_prefill
 *     on bf16 with hd = 128, H of 128 or 256 and r a multiple of 128, run on the
 *     tensor-core kernels; other shapes run on CUDA-core kernels, with the same
 *     results to the stated tolerances. Two
 *     environment variables, read at each call, force the CUDA-core kernels on
 *     shapes the tensor-core kernels would take: LOWRAM_DECODE_PATH=general (decode
 *     entry points) and LOWRAM_PACK_PATH=general (lr_pack_prefill). Any other value,
 *     or none, keeps the default choice. They exist for testing and comparison.
 *
 * Notation: B batch (sequences), T context tokens, L_g layers per group,
 * Hkv KV heads, G = Hq / Hkv query heads per KV head (query head hq reads KV
 * head hq / G), hd head_dim, D = L_g * Hkv * hd, r key rank, H predictor
 * hidden width, k residual rows per (sequence, layer, KV head),
 * nblk = ceil(T / 64) key blocks of 64 tokens.
 */
#ifndef LOWRAM_H
#define LOWRAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LR_ABI_VERSION 2
#define LR_BLOCK_TOKENS 64

typedef void* lr_stream_t; /* cudaStream_t */

typedef enum lr_status {
  LR_OK = 0,
  LR_ERR_INVALID_ARG = 1,  /* a null pointer, bad size, bad alignment or out-of-range argument */
  LR_ERR_UNSUPPORTED = 2,  /* a valid shape this build does not implement */
  LR_ERR_WORKSPACE = 3,    /* ws_bytes below the size the matching *_workspace_bytes returns */
  LR_ERR_CUDA = 4,         /* a CUDA launch or copy failed */
  LR_ERR_DEVICE_CHECK = 5  /* lr_get_device_error found a nonzero device error word */
} lr_status;

typedef enum lr_dtype { LR_F32 = 0, LR_BF16 = 1 } lr_dtype;

/* Bits of the device error word (OR-ed over one call). */
#define LR_DEVERR_BLOCK_RANGE 1 /* a selected block id outside [0, nblk): entry skipped */
#define LR_DEVERR_BLOCK_ORDER 2 /* selected block ids not strictly ascending: entry skipped */
#define LR_DEVERR_RES_RANGE 4   /* a residual index outside its block or [0, T): entry skipped */
#define LR_DEVERR_RES_ORDER 8   /* residual indices not strictly ascending */
#define LR_DEVERR_PTR 16        /* a residual block pointer out of [0, k] or decreasing */
#define LR_DEVERR_TIMEOUT 32    /* a kernel gave up waiting on its own pipeline (its output is invalid) */
#define LR_DEVERR_LAUNCH 64     /* a kernel found its shared memory misaligned and did not run (output invalid) */

typedef struct lr_cache_shape {
  int32_t batch;      /* B >= 0 */
  int32_t T;          /* context tokens per sequence, >= 0 */
  int32_t n_layers;   /* L_g >= 1: layers sharing one key factor A */
  int32_t n_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;   /* hd: multiple of 8, <= 256 */
  int32_t rank;       /* r: multiple of 8, >= 8 */
  int32_t hidden;     /* H: predictor hidden width, multiple of 8, <= 512 */
  lr_dtype dtype;     /* storage type of every floating tensor */
} lr_cache_shape;

/*
 * Value predictor f_theta of every (layer, KV head) of the group ("Predicting
 * the value cache from keys", paragraphs 2-3):
 *     v_hat = k W_lin^T + GELU(k W1^T + b1) W2^T + b2,   GELU(x) = x Phi(x) (erf form),
 * where k is the reconstructed key of one token and one KV head (the tensor-core decode
 * kernels evaluate GELU in a tanh form within 2.7e-4 of the erf form). Weights are in
 * nn.Linear layout (out x in). With per_sequence = 1 every array has a leading
 * batch dimension [B, ...]; with 0 one predictor serves all sequences.
 *     W_lin [(B,) L_g, Hkv, hd, hd]     W1 [(B,) L_g, Hkv, H, hd]     b1 [(B,) L_g, Hkv, H]
 *     W2    [(B,) L_g, Hkv, hd, H]      b2 [(B,) L_g, Hkv, hd] or NULL (= zero)
 */
typedef struct lr_predictor {
  const void* W_lin;
  const void* W1;
  const void* b1;
  const void* W2;
  const void* b2;
  int32_t per_sequence;
} lr_predictor;

/* ------------------------------------------------------------------ prefill packer */

/* Workspace bytes lr_pack_prefill needs for this shape and residual count. */
size_t lr_pack_workspace_bytes(const lr_cache_shape* shape, int32_t k);

/*
 * lr_pack_prefill -- build the compressed cache of one layer group.
 *
 * Steps (project page Figure 3; explainer paragraphs 2-4):
 *   1. A = round(K_group . Bt): project every token's group keys onto the shared
 *      factor (Bt has orthonormal columns: the truncated-SVD basis B transposed).
 *   2. For each layer l and KV head h: k~_t = A[t] . B_l^h, where B_l^h is rows
 *      (l*Hkv + h)*hd .. +hd of Bt;
 *   3. v_hat_t = f_theta(k~_t) with the (l, h) predictor;
 *   4. e_t = sum_j (v_t[j] - v_hat_t[j])^2 (fp32);
 *   5. the k tokens of largest e_t, ties to the lower token index, ascending;
 *   6. res_val = round(v - v_hat) at those tokens, and the block pointers
 *      res_blk_ptr[j] = #{i : res_idx[i] < 64 j}, j = 0 .. nblk.
 *   round() is round-to-nearest-even to the storage type.
 *
 * Inputs:  K_group [B, T, D]; V [B, L_g, T, Hkv, hd]; Bt [B, D, r];
 *          predictor as above; 0 <= k <= T.
 * Outputs: A [B, T, r]; res_idx [B, L_g, Hkv, k] int32; res_val [B, L_g, Hkv, k, hd];
 *          res_blk_ptr [B, L_g, Hkv, nblk + 1] int32 or NULL;
 *          err_out [B, L_g, Hkv, T] fp32 or NULL (the e_t of step 4).
 * res_idx / res_val may be NULL when k == 0.
 */
lr_status lr_pack_prefill(const lr_cache_shape* shape, const void* K_group, const void* V,
                          const void* Bt, const lr_predictor* predictor, int32_t k, void* A,
                          int32_t* res_idx, void* res_val, int32_t* res_blk_ptr, float* err_out,
                          void* ws, size_t ws_bytes, lr_stream_t stream);

/* ------------------------------------------------------------------ decode attention */

/* Workspace bytes lr_decode_attn needs (n_sel = 0 for full reconstruction). The
 * answer depends on the current device's SM count; query it on the device that runs
 * the call. */
size_t lr_decode_workspace_bytes(const lr_cache_shape* shape, int32_t n_q_heads, int32_t n_sel);

/*
 * lr_decode_attn -- one decode step of one layer over the compressed cache.
 *
 * For each sequence b and query head hq (KV head h = hq / G):
 *   S    = all tokens [0, T) when block_list is NULL, else the union of the 64-token
 *          blocks block_list[b, h, 0 .. n_sel) (selective reconstruction, arXiv
 *          abstract); the last block is clipped at T;
 *   k~_t = A[b, t] . B_l^h                         (project page, Figure 3)
 *   v_t  = f_theta(k~_t) + res_val[i]  if t = res_idx[b, l, h, i], else f_theta(k~_t)
 *                                                  (explainer, paragraph 2)
 *   o[b, hq] = sum_{t in S} softmax_t(scale * q[b, hq] . k~_t) v_t
 * An empty S gives o = 0. scale <= 0 selects 1/sqrt(hd).
 *
 * Inputs:  q [B, Hq, hd]; A [B, T, r]; Bt [B, D, r]; predictor of the group;
 *          res_idx [B, L_g, Hkv, k] ascending per row; res_val [B, L_g, Hkv, k, hd];
 *          res_blk_ptr [B, L_g, Hkv, nblk + 1] or NULL (then the kernel searches res_idx);
 *          block_list [B, Hkv, n_sel] strictly ascending block ids, or NULL = all tokens;
 *          0 <= layer < L_g; n_q_heads a multiple of Hkv; 0 <= n_sel <= nblk.
 * Output:  o [B, Hq, hd].
 */
lr_status lr_decode_attn(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads,
                         const void* q, const void* A, const void* Bt,
                         const lr_predictor* predictor, const int32_t* res_idx,
                         const void* res_val, const int32_t* res_blk_ptr, int32_t k,
                         const int32_t* block_list, int32_t n_sel, float scale, void* o,
                         void* ws, size_t ws_bytes, lr_stream_t stream);

/* Largest exact tail lr_decode_attn_tail accepts. */
#define LR_MAX_TAIL 4096

/*
 * lr_decode_attn_tail -- lr_decode_attn with an exact recent-token tail.
 *
 * Tokens generated after the cache was packed are kept exactly until the cache is packed
 * again (explainer, paragraph on prefill and decode costs: newly generated tokens are
 * stored exactly). They join the same softmax with their own keys and values:
 *   o[b, hq] = sum_{t in S + tail} softmax_t(scale * q[b, hq] . key_t) value_t,
 * where a tail token i of KV head h has key tail_K[b, h, i] and value tail_V[b, h, i]
 * (this layer's), and S is the compressed set of lr_decode_attn.
 *
 * Inputs:  those of lr_decode_attn, plus tail_K, tail_V [B, Hkv, n_tail, hd] in the cache
 *          dtype (caller-owned device memory, this layer's slices), 0 <= n_tail <=
 *          LR_MAX_TAIL; tail_K / tail_V may be NULL when n_tail == 0, which makes the call
 *          lr_decode_attn. The tail is attended whatever block_list selects; T may be 0.
 * Output:  o [B, Hq, hd]. Workspace: lr_decode_workspace_bytes, as for lr_decode_attn.
 * Errors:  as lr_decode_attn; n_tail outside [0, LR_MAX_TAIL] or a NULL tail with
 *          n_tail > 0 return LR_ERR_INVALID_ARG before any launch.
 */
lr_status lr_decode_attn_tail(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads,
                              const void* q, const void* A, const void* Bt,
                              const lr_predictor* predictor, const int32_t* res_idx,
                              const void* res_val, const int32_t* res_blk_ptr, int32_t k,
                              const int32_t* block_list, int32_t n_sel, const void* tail_K,
                              const void* tail_V, int32_t n_tail, float scale, void* o,
                              void* ws, size_t ws_bytes, lr_stream_t stream);

/* ------------------------------------------------------------------ test-time fitting */

/* The predictor's parameters as fp32 arrays (the layouts of lr_predictor), updated in place by
 * lr_fit_predictor. b2 may be NULL: then the predictor has no b2 and it is not fitted. */
typedef struct lr_predictor_f32 {
  float* W_lin;
  float* W1;
  float* b1;
  float* W2;
  float* b2;
  int32_t per_sequence;
} lr_predictor_f32;

/* Copies of the fitted parameters in the cache dtype (the lr_predictor layouts), written after
 * the last step; b2 may be NULL. */
typedef struct lr_predictor_out {
  void* W_lin;
  void* W1;
  void* b1;
  void* W2;
  void* b2;
} lr_predictor_out;

/* Workspace bytes lr_fit_predictor needs (0 for a shape it does not support). The answer
 * depends on the current device's SM count. */
size_t lr_fit_workspace_bytes(const lr_cache_shape* shape, int32_t per_sequence);

/*
 * lr_fit_predictor -- test-time fitting of the value predictor to the context's own keys and
 * values (explainer, paragraph on prefill cost: the per-head network is fitted to each context
 * with gradient steps, 150 of them in the paper's quick setting, 300 for a full fit; arXiv
 * abstract: the predictor is fitted at test time). The pages name neither the loss nor the
 * optimiser; the reading taken is n_steps of full-batch gradient descent
 *     theta <- theta - lr * grad L(theta),
 *     L = mean over tokens t and entries j of (v_hat_t[j] - v_t[j])^2,
 * per (layer, KV head) predictor, over the rebuilt keys k~_t = A[t] . B_l^h and the true values
 * of the context (of each sequence with per_sequence = 1; of all sequences with 0). theta is
 * every parameter: W_lin, W1, b1, W2 and b2 when present. GELU is evaluated in the tanh form
 * of the tensor-core kernels (within 2.71e-4 of x Phi(x)) and its derivative in the same form.
 * Run it between the projection and the residual selection: lr_pack_prefill with k = 0 gives A,
 * then this call, then lr_pack_prefill again with the fitted (rounded) predictor.
 *
 * Inputs:  A [B, T, r] (cache dtype); Bt [B, D, r]; V [B, L_g, T, Hkv, hd]; params (fp32,
 *          the starting point: the pseudoinverse initialisation or an earlier fit), updated in
 *          place; n_steps >= 0; lr >= 0.
 * Outputs: params; out (or NULL): the fitted parameters rounded to the cache dtype.
 * Shapes:  bf16 cache, head_dim 128, hidden 128 or 256, rank a multiple of 128
 *          (LR_ERR_UNSUPPORTED otherwise).
 * Errors:  host checks before any launch; LR_ERR_CUDA on a launch failure; the workspace's
 *          error word as for the other calls.
 */
lr_status lr_fit_predictor(const lr_cache_shape* shape, const void* A, const void* Bt, const void* V,
                           const lr_predictor_f32* params, int32_t n_steps, float lr,
                           const lr_predictor_out* out, void* ws, size_t ws_bytes, lr_stream_t stream);

/* ------------------------------------------------------------------ 2-bit residual rows */

/*
 * lr_quantize_residuals -- store residual rows with 2 bits per number (explainer, comparison
 * table: LowRAM combined with quantisation keeps 2-bit residuals). The pages name no
 * quantiser; this one is uniform per row: lo = min, hi = max, step = (hi - lo) / 3, and entry
 * x gets the code c = nearest integer of (x - lo) / step (ties to the even code), clamped to
 * 0..3 (code 0 everywhere when step = 0). Each of hi - lo, the step, x - lo and the quotient
 * is one correctly rounded fp32 operation, so the codes are exact integers of the stored row.
 * A decode step reads lo + c * step in place of the row (lr_decode_attn_q2).
 *
 * Inputs:  res_val [n_rows, hd] in the cache dtype (e.g. the rows lr_pack_prefill wrote,
 *          n_rows = B * L_g * Hkv * k); shape gives hd (a multiple of 4) and the dtype.
 * Outputs: res_codes [n_rows, hd / 4] uint8, entry 4i + s in bits 2s..2s+1 of byte i;
 *          res_lo [n_rows] fp32 row minimum; res_step [n_rows] fp32 level step.
 * Errors:  shape errors and NULL / misaligned pointers on the host; LR_ERR_CUDA on a launch
 *          failure. Needs no workspace.
 */
lr_status lr_quantize_residuals(const lr_cache_shape* shape, int64_t n_rows, const void* res_val,
                                uint8_t* res_codes, float* res_lo, float* res_step, lr_stream_t stream);

/*
 * lr_decode_attn_q2 -- lr_decode_attn over 2-bit residual rows: the residual added to token
 * t = res_idx[b, l, h, i] is res_lo[b, l, h, i] + c_j * res_step[b, l, h, i] for entry j, c_j
 * the code of lr_quantize_residuals. Everything else (inputs, output, workspace, errors) is
 * as lr_decode_attn; res_codes [B, L_g, Hkv, k, hd / 4], res_lo / res_step [B, L_g, Hkv, k]
 * take the place of res_val (they may be NULL when k == 0).
 */
lr_status lr_decode_attn_q2(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads,
                            const void* q, const void* A, const void* Bt,
                            const lr_predictor* predictor, const int32_t* res_idx,
                            const uint8_t* res_codes, const float* res_lo, const float* res_step,
                            const int32_t* res_blk_ptr, int32_t k, const int32_t* block_list,
                            int32_t n_sel, float scale, void* o, void* ws, size_t ws_bytes,
                            lr_stream_t stream);

/* ------------------------------------------------------------------ block selection */

/*
 * lr_block_means -- the mean A row of every 64-token block of the packed cache:
 *   Abar[b, j] = mean_{t in block j} A[b, t],   the last block clipped at T.
 * The rebuilt key is linear in A, so Abar[b, j] . B_l^h is the mean rebuilt key of block j
 * for every layer and KV head of the group. Abar does not depend on the query: compute it
 * once after lr_pack_prefill and pass it to every lr_select_blocks call on that cache.
 * Inputs: A [B, T, r] (cache dtype). Output: Abar [B, nblk, r] fp32 (1/64 of A's rows).
 * Errors: shape errors and NULL / misaligned pointers on the host; LR_ERR_CUDA on a launch
 * failure. Needs no workspace.
 */
lr_status lr_block_means(const lr_cache_shape* shape, const void* A, float* Abar, lr_stream_t stream);

/* Workspace bytes lr_select_blocks needs. */
size_t lr_select_workspace_bytes(const lr_cache_shape* shape, int32_t n_q_heads);

/*
 * lr_select_blocks -- choose the 64-token blocks a decode step rebuilds (selective
 * reconstruction: arXiv abstract; explainer, paragraph on prefill and decode costs, where
 * only the chunks the current query selects are rebuilt). The pages' trained selector is
 * not available; this one scores a block by its mean reconstructed key:
 *   score[b, h, j] = max over the query heads hq = h G .. h G + G - 1 of
 *                    scale * q[b, hq] . mean_{t in block j} k~_t
 *                  = max_hq (scale * B_l^h q[b, hq]) . Abar[b, j],   k~_t = A[b, t] . B_l^h,
 * and returns per (b, h) the n_sel blocks of highest score, ties to the lower block id, in
 * ascending order: the block_list layout of lr_decode_attn. The list is exactly the top
 * n_sel of the returned fp32 scores.
 *
 * Inputs:  q [B, Hq, hd]; Abar [B, nblk, r] fp32 from lr_block_means; Bt [B, D, r];
 *          0 <= layer < L_g; n_q_heads a multiple of Hkv with at most 8 query heads per KV
 *          head; 0 <= n_sel <= nblk; scale <= 0 selects 1/sqrt(hd).
 * Outputs: block_list [B, Hkv, n_sel] int32 (not touched when n_sel == 0);
 *          scores_out [B, Hkv, nblk] fp32 or NULL (the scores the list was taken from).
 * Errors:  argument and shape errors on the host before any launch; LR_ERR_CUDA on a launch
 *          failure. Scores are fp32 (a rank-space dot product accumulated in fp32).
 */
lr_status lr_select_blocks(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads, const void* q,
                           const float* Abar, const void* Bt, int32_t n_sel, float scale, int32_t* block_list,
                           float* scores_out, void* ws, size_t ws_bytes, lr_stream_t stream);

/* ------------------------------------------------------------------ single steps */

/* Workspace bytes lr_topk_tokens needs. */
size_t lr_topk_workspace_bytes(int32_t n_segments, int32_t T, int32_t k);

/*
 * lr_topk_tokens -- step 5 of the packer on its own (explainer, paragraph 4:
 * residuals go to the tokens ranked worst by error).
 * err [n_segments, T] fp32 -> idx_out [n_segments, k] int32: per segment the k
 * tokens of largest error, ties to the lower index, in ascending index order.
 * Errors compare as IEEE values (-0 == +0); NaN ranks below every number.
 * The result is unique, so it is bit-exact by definition.
 */
lr_status lr_topk_tokens(const float* err, int32_t n_segments, int32_t T, int32_t k,
                         int32_t* idx_out, void* ws, size_t ws_bytes, lr_stream_t stream);

/*
 * lr_residual_block_ptr -- the residual block pointers of step 6 on their own.
 * idx [n_segments, k] ascending -> ptr_out [n_segments, nblk + 1] with
 * ptr_out[s, j] = #{i : idx[s, i] < 64 j}. Needs no workspace.
 */
lr_status lr_residual_block_ptr(const int32_t* idx, int32_t n_segments, int32_t k, int32_t T,
                                int32_t* ptr_out, lr_stream_t stream);

/* ------------------------------------------------------------------ allocation-free decode */

/*
 * lr_decode_attn_noalloc -- lr_decode_attn for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment variant of the decode step above.
 *
 * Some callers cannot call cudaMalloc or any allocating routine: code running inside an
 * allocator or memory-pool callback, runtimes that own every device allocation and only
 * hand out fixed buffers, and latency-critical paths where an allocation could block or
 * fail. This entry point takes the same inputs and output as lr_decode_attn (caller-owned
 * device tensors) but no workspace: it runs on a 16 MiB scratch array compiled into the
 * library (a file-scope __device__ array, present on every GPU that loads the library
 * until the process exits).
 *   - Shapes whose lr_decode_workspace_bytes exceeds 16 MiB return LR_ERR_WORKSPACE with
 *     a message in lr_last_error(); nothing is launched.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share the array and each call clears the part that must start
 *     at zero; calls that overlap on the GPU (different streams, or host threads without
 *     ordering) race on it.
 *   - Device-side data checks write the shared array's error word; lr_get_device_error
 *     with ws = NULL reads it (the word of the last call on the current device).
 *   - The array's address is looked up once per device and kept for the life of the
 *     process: do not use this entry point on a device after cudaDeviceReset there.
 * Argument meaning, layouts, ownership and the other error behaviour: as lr_decode_attn.
 */
lr_status lr_decode_attn_noalloc(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads,
                                 const void* q, const void* A, const void* Bt,
                                 const lr_predictor* predictor, const int32_t* res_idx,
                                 const void* res_val, const int32_t* res_blk_ptr, int32_t k,
                                 const int32_t* block_list, int32_t n_sel, float scale, void* o,
                                 lr_stream_t stream);

/* ------------------------------------------------------------------ errors, version */

/* Copies the device error word of the last call that used `ws` into *code and
 * synchronises `stream`. Returns LR_OK when the word is 0, LR_ERR_DEVICE_CHECK when it
 * is not, LR_ERR_CUDA when the copy fails. Every call that takes a workspace clears
 * the word when it starts. ws = NULL reads the word of the last lr_decode_attn_noalloc
 * call on the current device. */
lr_status lr_get_device_error(const void* ws, lr_stream_t stream, int32_t* code);

const char* lr_status_string(lr_status status);
const char* lr_last_error(void);
int32_t lr_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LOWRAM_H */
