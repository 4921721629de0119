// Host side of the C ABI declared in include/lowram.h: argument checks, workspace
// planning and kernel launches. Nothing here allocates device memory or keeps
// state between calls; the only per-thread state is the last error message.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "lowram.h"
#include "lr_common.cuh"
#include "lr_launch.h"
#include "lr_plan.h"

namespace {

thread_local char g_msg[512] = "";

lr_status fail(lr_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

lr_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

#define CHECK_PTR(p, name)                                                          \
  do {                                                                              \
    if (!(p)) return fail(LR_ERR_INVALID_ARG, "%s is NULL", name);                  \
    if (!aligned((p), 16)) return fail(LR_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

#define CHECK_OPT_PTR(p, name)                                                      \
  do {                                                                              \
    if ((p) && !aligned((p), 16)) return fail(LR_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

lr_status check_shape(const lr_cache_shape* s) {
  if (!s) return fail(LR_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 0 || s->T < 0) return fail(LR_ERR_INVALID_ARG, "batch and T must be >= 0");
  if (s->n_layers < 1 || s->n_kv_heads < 1) return fail(LR_ERR_INVALID_ARG, "n_layers and n_kv_heads must be >= 1");
  if (s->head_dim < 1 || s->rank < 1 || s->hidden < 1) return fail(LR_ERR_INVALID_ARG, "head_dim, rank and hidden must be >= 1");
  if (s->dtype != LR_F32 && s->dtype != LR_BF16) return fail(LR_ERR_INVALID_ARG, "unknown dtype %d", (int)s->dtype);
  if (s->head_dim % 8 || s->head_dim > 256) return fail(LR_ERR_UNSUPPORTED, "head_dim must be a multiple of 8 and <= 256");
  if (s->rank % 8) return fail(LR_ERR_UNSUPPORTED, "rank must be a multiple of 8");
  if (s->hidden % 8 || s->hidden > 512) return fail(LR_ERR_UNSUPPORTED, "hidden must be a multiple of 8 and <= 512");
  const long long D = (long long)s->n_layers * s->n_kv_heads * s->head_dim;
  if (D > (1 << 20)) return fail(LR_ERR_UNSUPPORTED, "layer-group key width too large");
  return LR_OK;
}

lr_status check_predictor(const lr_predictor* p) {
  if (!p) return fail(LR_ERR_INVALID_ARG, "predictor is NULL");
  CHECK_PTR(p->W_lin, "predictor.W_lin");
  CHECK_PTR(p->W1, "predictor.W1");
  CHECK_PTR(p->b1, "predictor.b1");
  CHECK_PTR(p->W2, "predictor.W2");
  CHECK_OPT_PTR(p->b2, "predictor.b2");
  if (p->per_sequence != 0 && p->per_sequence != 1) return fail(LR_ERR_INVALID_ARG, "predictor.per_sequence must be 0 or 1");
  return LR_OK;
}

lr_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(LR_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(LR_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  if (ws_bytes < need) return fail(LR_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return LR_OK;
}

int current_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  return n;
}

}  // namespace

namespace lr {
// Records a message for lr_last_error() (used by entry points defined in other files).
void set_last_error(const char* msg) { snprintf(g_msg, sizeof(g_msg), "%s", msg); }
lr_status noalloc_scratch_address(void** out);
}  // namespace lr

extern "C" {

const char* lr_last_error(void) { return g_msg; }

int32_t lr_abi_version(void) { return LR_ABI_VERSION; }

const char* lr_status_string(lr_status s) {
  switch (s) {
    case LR_OK: return "ok";
    case LR_ERR_INVALID_ARG: return "invalid argument";
    case LR_ERR_UNSUPPORTED: return "unsupported shape";
    case LR_ERR_WORKSPACE: return "workspace too small";
    case LR_ERR_CUDA: return "CUDA error";
    case LR_ERR_DEVICE_CHECK: return "device-side data check failed";
  }
  return "unknown status";
}

lr_status lr_get_device_error(const void* ws, lr_stream_t stream, int32_t* code) {
  if (!code) return fail(LR_ERR_INVALID_ARG, "code must not be NULL");
  if (!ws) {  // the scratch array of lr_decode_attn_noalloc on the current device
    void* p = nullptr;
    if (lr::noalloc_scratch_address(&p) != LR_OK) return fail(LR_ERR_CUDA, "locating the allocation-free scratch");
    ws = p;
  }
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *code = v;
  return v ? LR_ERR_DEVICE_CHECK : LR_OK;
}

// ------------------------------------------------------------------ decode

size_t lr_decode_workspace_bytes(const lr_cache_shape* s, int32_t n_q_heads, int32_t n_sel) {
  if (check_shape(s) != LR_OK || n_q_heads < 1) return 0;
  return lr::plan_decode(*s, n_q_heads, n_sel, current_sm_count()).ws_bytes;
}

}  // extern "C"

namespace {
// Residual rows as stored values (res_val) or as 2-bit codes (res_codes, res_lo, res_step).
struct ResRows {
  const void* val;
  const uint8_t* codes;
  const float* lo;
  const float* step;
};

lr_status decode_impl(const lr_cache_shape* s, int32_t layer, int32_t n_q_heads, const void* q, const void* A,
                      const void* Bt, const lr_predictor* pred, const int32_t* res_idx, const ResRows& rr,
                      const int32_t* res_blk_ptr, int32_t k, const int32_t* block_list, int32_t n_sel,
                      const void* tail_K, const void* tail_V, int32_t n_tail, float scale, void* o, void* ws,
                      size_t ws_bytes, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (layer < 0 || layer >= s->n_layers) return fail(LR_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, s->n_layers);
  if (n_q_heads < 1 || n_q_heads % s->n_kv_heads) return fail(LR_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (n_q_heads / s->n_kv_heads > 8) return fail(LR_ERR_UNSUPPORTED, "more than 8 query heads per KV head");
  const int nblk = lr::ceil_div(s->T, LR_BLOCK_TOKENS);
  if (k < 0 || k > s->T) return fail(LR_ERR_INVALID_ARG, "k=%d outside [0, T]", k);
  if (block_list && (n_sel < 0 || n_sel > nblk)) return fail(LR_ERR_INVALID_ARG, "n_sel=%d outside [0, nblk=%d]", n_sel, nblk);
  if (!block_list) n_sel = 0;
  if ((st = check_predictor(pred)) != LR_OK) return st;
  CHECK_PTR(q, "q");
  CHECK_PTR(A, "A");
  CHECK_PTR(Bt, "Bt");
  CHECK_PTR(o, "o");
  if (k > 0) {
    CHECK_PTR(res_idx, "res_idx");
    if (rr.codes) {
      CHECK_PTR(rr.lo, "res_lo");
      CHECK_PTR(rr.step, "res_step");
    } else {
      CHECK_PTR(rr.val, "res_val");
    }
  }
  CHECK_OPT_PTR(res_blk_ptr, "res_blk_ptr");
  CHECK_OPT_PTR(block_list, "block_list");
  if (n_tail < 0 || n_tail > LR_MAX_TAIL) return fail(LR_ERR_INVALID_ARG, "n_tail=%d outside [0, %d]", n_tail, LR_MAX_TAIL);
  if (n_tail > 0) {
    CHECK_PTR(tail_K, "tail_K");
    CHECK_PTR(tail_V, "tail_V");
  }
  const lr::DecodePlan plan = lr::plan_decode(*s, n_q_heads, n_sel, current_sm_count());
  if ((st = check_ws(ws, ws_bytes, plan.ws_bytes)) != LR_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  if (s->batch == 0) return LR_OK;

  lr::DecodeArgs a{};
  a.B = s->batch; a.T = s->T; a.L = s->n_layers; a.Hkv = s->n_kv_heads; a.G = n_q_heads / s->n_kv_heads;
  a.hd = s->head_dim; a.r = s->rank; a.H = s->hidden;
  a.layer = layer; a.k = k; a.n_sel = n_sel; a.nblk = nblk;
  a.pred_per_seq = pred->per_sequence;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)s->head_dim);
  a.q = q; a.A = A; a.Bt = Bt;
  a.W_lin = pred->W_lin; a.W1 = pred->W1; a.b1 = pred->b1; a.W2 = pred->W2; a.b2 = pred->b2;
  a.res_idx = k ? res_idx : nullptr; a.res_val = (k && !rr.codes) ? rr.val : nullptr;
  a.res_codes = k ? rr.codes : nullptr; a.res_lo = k ? rr.lo : nullptr; a.res_step = k ? rr.step : nullptr;
  a.res_ptr = k ? res_blk_ptr : nullptr;
  a.blocks = block_list;
  a.tail_K = n_tail ? tail_K : nullptr;
  a.tail_V = n_tail ? tail_V : nullptr;
  a.n_tail = n_tail;
  a.o = o;
  a.err = (int*)ws;
  a.partials = (float*)((char*)ws + plan.part_off);
  a.n_split = plan.n_split;
  a.part_stride = plan.part_stride;
  if ((e = lr::launch_decode(a, plan, s->dtype, cs)) != cudaSuccess) return cuda_fail(e, "decode launch");
  return LR_OK;
}
}  // namespace

extern "C" {

lr_status lr_decode_attn(const lr_cache_shape* s, int32_t layer, int32_t n_q_heads, const void* q,
                         const void* A, const void* Bt, const lr_predictor* pred,
                         const int32_t* res_idx, const void* res_val, const int32_t* res_blk_ptr,
                         int32_t k, const int32_t* block_list, int32_t n_sel, float scale, void* o,
                         void* ws, size_t ws_bytes, lr_stream_t stream) {
  return decode_impl(s, layer, n_q_heads, q, A, Bt, pred, res_idx, ResRows{res_val, nullptr, nullptr, nullptr},
                     res_blk_ptr, k, block_list, n_sel, nullptr, nullptr, 0, scale, o, ws, ws_bytes, stream);
}

lr_status lr_decode_attn_q2(const lr_cache_shape* s, int32_t layer, int32_t n_q_heads, const void* q,
                            const void* A, const void* Bt, const lr_predictor* pred, const int32_t* res_idx,
                            const uint8_t* res_codes, const float* res_lo, const float* res_step,
                            const int32_t* res_blk_ptr, int32_t k, const int32_t* block_list, int32_t n_sel,
                            float scale, void* o, void* ws, size_t ws_bytes, lr_stream_t stream) {
  if (s && s->head_dim % 4) return fail(LR_ERR_UNSUPPORTED, "2-bit rows need head_dim % 4 == 0");
  if (k > 0) CHECK_PTR(res_codes, "res_codes");
  return decode_impl(s, layer, n_q_heads, q, A, Bt, pred, res_idx, ResRows{nullptr, res_codes, res_lo, res_step},
                     res_blk_ptr, k, block_list, n_sel, nullptr, nullptr, 0, scale, o, ws, ws_bytes, stream);
}

lr_status lr_quantize_residuals(const lr_cache_shape* s, int64_t n_rows, const void* res_val, uint8_t* res_codes,
                                float* res_lo, float* res_step, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (n_rows < 0) return fail(LR_ERR_INVALID_ARG, "n_rows must be >= 0");
  if (n_rows == 0) return LR_OK;
  CHECK_PTR(res_val, "res_val");
  CHECK_PTR(res_codes, "res_codes");
  CHECK_PTR(res_lo, "res_lo");
  CHECK_PTR(res_step, "res_step");
  const cudaError_t e = lr::launch_quantize_rows(res_val, s->dtype, n_rows, s->head_dim, res_codes, res_lo, res_step,
                                                 (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "residual quantisation launch");
  return LR_OK;
}

lr_status lr_decode_attn_tail(const lr_cache_shape* s, int32_t layer, int32_t n_q_heads, const void* q,
                              const void* A, const void* Bt, const lr_predictor* pred,
                              const int32_t* res_idx, const void* res_val, const int32_t* res_blk_ptr,
                              int32_t k, const int32_t* block_list, int32_t n_sel, const void* tail_K,
                              const void* tail_V, int32_t n_tail, float scale, void* o, void* ws,
                              size_t ws_bytes, lr_stream_t stream) {
  return decode_impl(s, layer, n_q_heads, q, A, Bt, pred, res_idx, ResRows{res_val, nullptr, nullptr, nullptr},
                     res_blk_ptr, k, block_list, n_sel, tail_K, tail_V, n_tail, scale, o, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ block selection

size_t lr_select_workspace_bytes(const lr_cache_shape* s, int32_t n_q_heads) {
  if (check_shape(s) != LR_OK || n_q_heads < 1) return 0;
  const size_t nblk = (size_t)lr::ceil_div(s->T, LR_BLOCK_TOKENS);
  const size_t qhat = (size_t)s->batch * n_q_heads * s->rank * sizeof(float);
  const size_t scores = (size_t)s->batch * s->n_kv_heads * nblk * sizeof(float);
  const size_t partial = (size_t)lr::select_rank_splits(s->rank) * s->batch * nblk * n_q_heads * sizeof(float);
  return 256 + ((qhat + 255) & ~(size_t)255) + ((scores + 255) & ~(size_t)255) + ((partial + 255) & ~(size_t)255);
}

lr_status lr_block_means(const lr_cache_shape* s, const void* A, float* Abar, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (s->batch == 0 || s->T == 0) return LR_OK;
  CHECK_PTR(A, "A");
  CHECK_PTR(Abar, "Abar");
  const cudaError_t e = lr::launch_block_means(A, s->batch, s->T, s->rank, s->dtype, Abar, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "block means launch");
  return LR_OK;
}

lr_status lr_select_blocks(const lr_cache_shape* s, int32_t layer, int32_t n_q_heads, const void* q,
                           const float* Abar, const void* Bt, int32_t n_sel, float scale, int32_t* block_list,
                           float* scores_out, void* ws, size_t ws_bytes, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (layer < 0 || layer >= s->n_layers) return fail(LR_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, s->n_layers);
  if (n_q_heads < 1 || n_q_heads % s->n_kv_heads) return fail(LR_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (n_q_heads / s->n_kv_heads > 8) return fail(LR_ERR_UNSUPPORTED, "more than 8 query heads per KV head");
  const int nblk = lr::ceil_div(s->T, LR_BLOCK_TOKENS);
  if (n_sel < 0 || n_sel > nblk) return fail(LR_ERR_INVALID_ARG, "n_sel=%d outside [0, nblk=%d]", n_sel, nblk);
  CHECK_PTR(q, "q");
  CHECK_PTR(Bt, "Bt");
  CHECK_OPT_PTR(scores_out, "scores_out");
  const bool work = (n_sel > 0 || scores_out) && nblk > 0;
  if (work) CHECK_PTR(Abar, "Abar");
  if (n_sel > 0) CHECK_PTR(block_list, "block_list");
  if ((st = check_ws(ws, ws_bytes, lr_select_workspace_bytes(s, n_q_heads))) != LR_OK) return st;
  if (!work || s->batch == 0) return LR_OK;
  lr::SelectArgs a{};
  a.B = s->batch; a.T = s->T; a.L = s->n_layers; a.Hkv = s->n_kv_heads; a.G = n_q_heads / s->n_kv_heads;
  a.hd = s->head_dim; a.r = s->rank; a.layer = layer; a.nblk = nblk; a.n_sel = n_sel;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)s->head_dim);
  a.q = q; a.abar = Abar; a.Bt = Bt;
  const size_t qhat = (size_t)s->batch * n_q_heads * s->rank * sizeof(float);
  a.qhat = (float*)((char*)ws + 256);
  const size_t scores_bytes = (size_t)s->batch * s->n_kv_heads * nblk * sizeof(float);
  a.scores = scores_out ? scores_out : (float*)((char*)ws + 256 + ((qhat + 255) & ~(size_t)255));
  a.partial = (float*)((char*)ws + 256 + ((qhat + 255) & ~(size_t)255) + ((scores_bytes + 255) & ~(size_t)255));
  a.n_split = lr::select_rank_splits(s->rank);
  a.blocks_out = block_list;
  const cudaError_t e = lr::launch_select_blocks(a, s->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "block selection launch");
  return LR_OK;
}

// ------------------------------------------------------------------ pack

size_t lr_pack_workspace_bytes(const lr_cache_shape* s, int32_t k) {
  if (check_shape(s) != LR_OK || k < 0) return 0;
  return lr::plan_pack(*s, k).ws_bytes;
}

lr_status lr_pack_prefill(const lr_cache_shape* s, const void* K_group, const void* V, const void* Bt,
                          const lr_predictor* pred, int32_t k, void* A, int32_t* res_idx,
                          void* res_val, int32_t* res_blk_ptr, float* err_out, void* ws,
                          size_t ws_bytes, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (k < 0 || k > s->T) return fail(LR_ERR_INVALID_ARG, "k=%d outside [0, T]", k);
  if ((st = check_predictor(pred)) != LR_OK) return st;
  CHECK_PTR(K_group, "K_group");
  CHECK_PTR(V, "V");
  CHECK_PTR(Bt, "Bt");
  CHECK_PTR(A, "A");
  if (k > 0) {
    CHECK_PTR(res_idx, "res_idx");
    CHECK_PTR(res_val, "res_val");
  }
  CHECK_OPT_PTR(res_blk_ptr, "res_blk_ptr");
  CHECK_OPT_PTR(err_out, "err_out");
  const lr::PackPlan plan = lr::plan_pack(*s, k);
  if ((st = check_ws(ws, ws_bytes, plan.ws_bytes)) != LR_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  if (s->batch == 0) return LR_OK;

  lr::PackArgs a{};
  a.B = s->batch; a.T = s->T; a.L = s->n_layers; a.Hkv = s->n_kv_heads; a.hd = s->head_dim;
  a.r = s->rank; a.H = s->hidden; a.D = s->n_layers * s->n_kv_heads * s->head_dim; a.k = k;
  a.nblk = lr::ceil_div(s->T, LR_BLOCK_TOKENS);
  a.pred_per_seq = pred->per_sequence;
  a.K = K_group; a.V = V; a.Bt = Bt;
  a.W_lin = pred->W_lin; a.W1 = pred->W1; a.b1 = pred->b1; a.W2 = pred->W2; a.b2 = pred->b2;
  a.A = A;
  a.err = err_out ? err_out : (float*)((char*)ws + plan.err_off);
  a.diff = (char*)ws + plan.diff_off;
  a.res_idx = res_idx; a.res_val = res_val; a.res_ptr = res_blk_ptr;
  a.errword = (int*)ws;
  if ((e = lr::launch_pack(a, plan, s->dtype, cs)) != cudaSuccess) return cuda_fail(e, "pack launch");
  return LR_OK;
}

// ------------------------------------------------------------------ test-time fitting

size_t lr_fit_workspace_bytes(const lr_cache_shape* s, int32_t per_sequence) {
  if (check_shape(s) != LR_OK || !lr::pack_tc_supported(*s)) return 0;
  return lr::plan_fit(*s, per_sequence ? 1 : 0, current_sm_count()).ws_bytes;
}

lr_status lr_fit_predictor(const lr_cache_shape* s, const void* A, const void* Bt, const void* V,
                           const lr_predictor_f32* params, int32_t n_steps, float lr,
                           const lr_predictor_out* out, void* ws, size_t ws_bytes, lr_stream_t stream) {
  lr_status st = check_shape(s);
  if (st != LR_OK) return st;
  if (!lr::pack_tc_supported(*s))
    return fail(LR_ERR_UNSUPPORTED, "fitting needs a bf16 cache with head_dim 128, hidden 128 or 256, rank %% 128 == 0");
  if (!params) return fail(LR_ERR_INVALID_ARG, "params is NULL");
  if (params->per_sequence != 0 && params->per_sequence != 1)
    return fail(LR_ERR_INVALID_ARG, "params.per_sequence must be 0 or 1");
  if (n_steps < 0) return fail(LR_ERR_INVALID_ARG, "n_steps must be >= 0");
  if (!(lr >= 0.f) || lr > 1e30f) return fail(LR_ERR_INVALID_ARG, "lr must be finite and >= 0");
  CHECK_PTR(A, "A");
  CHECK_PTR(Bt, "Bt");
  CHECK_PTR(V, "V");
  CHECK_PTR(params->W_lin, "params.W_lin");
  CHECK_PTR(params->W1, "params.W1");
  CHECK_PTR(params->b1, "params.b1");
  CHECK_PTR(params->W2, "params.W2");
  CHECK_OPT_PTR(params->b2, "params.b2");
  if (out) {
    CHECK_PTR(out->W_lin, "out.W_lin");
    CHECK_PTR(out->W1, "out.W1");
    CHECK_PTR(out->b1, "out.b1");
    CHECK_PTR(out->W2, "out.W2");
    CHECK_OPT_PTR(out->b2, "out.b2");
    if (out->b2 && !params->b2) return fail(LR_ERR_INVALID_ARG, "out.b2 given without params.b2");
  }
  const lr::FitPlan plan = lr::plan_fit(*s, params->per_sequence, current_sm_count());
  if (plan.n_wh > 65535) return fail(LR_ERR_UNSUPPORTED, "more than 65535 predictor heads");
  if ((st = check_ws(ws, ws_bytes, plan.ws_bytes)) != LR_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  if (s->batch == 0) return LR_OK;
  lr::FitCall c{};
  c.A = A; c.Bt = Bt; c.V = V;
  c.W_lin = params->W_lin; c.W1 = params->W1; c.b1 = params->b1; c.W2 = params->W2; c.b2 = params->b2;
  c.per_sequence = params->per_sequence;
  c.n_steps = n_steps;
  c.lr = lr;
  if (out) {
    c.out_Wl = out->W_lin; c.out_W1 = out->W1; c.out_b1 = out->b1; c.out_W2 = out->W2; c.out_b2 = out->b2;
  }
  c.ws = ws;
  if ((e = lr::launch_fit(*s, c, plan, cs)) != cudaSuccess) return cuda_fail(e, "fitting launch");
  return LR_OK;
}

// ------------------------------------------------------------------ single steps

size_t lr_topk_workspace_bytes(int32_t n_segments, int32_t T, int32_t k) {
  (void)n_segments; (void)T; (void)k;
  return 256;
}

lr_status lr_topk_tokens(const float* err, int32_t n_segments, int32_t T, int32_t k, int32_t* idx_out,
                         void* ws, size_t ws_bytes, lr_stream_t stream) {
  if (n_segments < 0 || T < 0) return fail(LR_ERR_INVALID_ARG, "n_segments and T must be >= 0");
  if (k < 0 || k > T) return fail(LR_ERR_INVALID_ARG, "k=%d outside [0, T]", k);
  lr_status st = check_ws(ws, ws_bytes, 256);
  if (st != LR_OK) return st;
  if (n_segments > 0 && k > 0) {
    CHECK_PTR(err, "err");
    CHECK_PTR(idx_out, "idx_out");
  }
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, cs);
  if (e == cudaSuccess) e = lr::launch_topk(err, n_segments, T, k, idx_out, cs);
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  return LR_OK;
}

lr_status lr_residual_block_ptr(const int32_t* idx, int32_t n_segments, int32_t k, int32_t T,
                                int32_t* ptr_out, lr_stream_t stream) {
  if (n_segments < 0 || T < 0) return fail(LR_ERR_INVALID_ARG, "n_segments and T must be >= 0");
  if (k < 0 || k > T) return fail(LR_ERR_INVALID_ARG, "k=%d outside [0, T]", k);
  if (n_segments == 0) return LR_OK;
  if (k > 0) CHECK_PTR(idx, "idx");
  CHECK_PTR(ptr_out, "ptr_out");
  cudaError_t e = lr::launch_block_ptr(idx, n_segments, k, T, ptr_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "block pointer launch");
  return LR_OK;
}

}  // extern "C"
