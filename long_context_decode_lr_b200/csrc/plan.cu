// Workspace layout and kernel choice for lr_decode_attn and lr_pack_prefill.
#include <cuda.h>
#include <stdlib.h>
#include <string.h>

#include "lr_common.cuh"
#include "lr_launch.h"
#include "lr_plan.h"
#include "lr_fit.h"
#include "lr_gemm.h"
#include "lr_tc.h"

namespace lr {

namespace {
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t elem_bytes(lr_dtype d) { return d == LR_BF16 ? 2 : 4; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A 16-bit tensor map with 128-byte swizzle; dims/box innermost first, out-of-range reads give 0.
bool tile_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

bool decode_pair_supported(const lr_cache_shape& s, int n_q_heads) {
  const int G = n_q_heads / s.n_kv_heads;
  return s.dtype == LR_BF16 && s.head_dim == 128 && (s.hidden == 128 || s.hidden == 256) && s.rank % 64 == 0 &&
         G >= 1 && G <= 8 && s.T > 0;
}

namespace {
// Kernel family for the decode call: the CTA-pair tensor-core kernel where the shape allows
// it, else the CUDA-core kernel. LOWRAM_DECODE_PATH=general forces the CUDA-core kernel for
// every shape (a supported option, documented in lowram.h); "pair" or unset keeps the default.
DecodePath choose_path(const lr_cache_shape& s, int n_q_heads) {
  const char* env = getenv("LOWRAM_DECODE_PATH");
  const bool want_pair = !env || strcmp(env, "general") != 0;
  if (want_pair && decode_pair_supported(s, n_q_heads)) return DecodePath::Pair;
  return DecodePath::General;
}
}  // namespace

DecodePlan plan_decode(const lr_cache_shape& s, int n_q_heads, int n_sel, int sm_count) {
  DecodePlan p{};
  const int nblk = ceil_div(s.T, LR_BLOCK_TOKENS);
  const DecodePath path = choose_path(s, n_q_heads);
  if (path == DecodePath::Pair) {
    p.path = DecodePath::Pair;
    int clusters = tc::pair_max_clusters();
    if (clusters <= 0 || clusters > sm_count / 2) clusters = sm_count / 2;
    const int rows = s.batch * s.n_kv_heads;
    const int max_tiles = ceil_div(n_sel > 0 ? n_sel : nblk, 4);
    int n_pairs = rows > 0 ? (clusters + rows / 2) / rows : 1;
    if (n_pairs * rows > clusters) n_pairs = clusters / rows;  // one wave of clusters
    if (n_pairs > max_tiles) n_pairs = max_tiles;
    if (n_pairs < 1) n_pairs = 1;
    p.n_pairs = n_pairs;
    p.n_split = 2 * n_pairs;
    p.part_stride = 4 + 2 * s.head_dim + s.hidden;
    p.part_off = 256;
    const size_t part_bytes = (size_t)s.batch * n_q_heads * p.n_split * p.part_stride * sizeof(float);
    p.sched_off = align256(p.part_off + part_bytes);
    // the schedule region is always reserved: an empty selected-block list still writes a count
    const size_t sched_bytes = (size_t)rows * (1 + (size_t)(n_sel > 0 ? n_sel : 0)) * sizeof(int);
    p.w1h_off = align256(p.sched_off + sched_bytes);
    const size_t w1h_bytes = (size_t)s.batch * s.n_kv_heads * s.hidden * s.head_dim * 2;
    p.qhat_off = align256(p.w1h_off + w1h_bytes);
    const size_t qhat_bytes = (size_t)rows * tc::kPairQRows * s.rank * 2;
    p.ws_bytes = align256(p.qhat_off + qhat_bytes);
    return p;
  }
  p.path = DecodePath::General;
  const int units = n_sel > 0 ? n_sel : nblk;
  const int per_row = s.batch * s.n_kv_heads;
  int n_split = per_row > 0 ? ceil_div(2 * sm_count, per_row) : 1;
  if (n_split > units) n_split = units;
  if (n_split > 1024) n_split = 1024;
  if (n_split < 1) n_split = 1;
  p.n_split = n_split;
  p.part_stride = 4 + 2 * s.head_dim + s.hidden;
  p.part_off = 256;
  const size_t part_bytes = (size_t)s.batch * n_q_heads * n_split * p.part_stride * sizeof(float);
  p.sched_off = align256(p.part_off + part_bytes);
  p.ws_bytes = p.sched_off;
  return p;
}

bool pack_tc_supported(const lr_cache_shape& s) {
  const long long D = (long long)s.n_layers * s.n_kv_heads * s.head_dim;
  return s.dtype == LR_BF16 && s.head_dim == 128 && (s.hidden == 128 || s.hidden == 256) && s.rank % 128 == 0 &&
         D % 128 == 0 && s.T > 0;
}

PackPlan plan_pack(const lr_cache_shape& s, int k) {
  (void)k;
  PackPlan p{};
  const char* env = getenv("LOWRAM_PACK_PATH");
  p.tensor = pack_tc_supported(s) && !(env && !strcmp(env, "general"));
  const size_t rows = (size_t)s.batch * s.n_layers * s.n_kv_heads * s.T;
  p.err_off = 256;
  const size_t after_err = align256(p.err_off + rows * sizeof(float));
  if (!p.tensor) {
    p.diff_off = after_err;
    p.ws_bytes = align256(p.diff_off + rows * s.head_dim * elem_bytes(s.dtype));
    return p;
  }
  const size_t D = (size_t)s.n_layers * s.n_kv_heads * s.head_dim;
  const size_t heads = (size_t)s.batch * s.n_layers * s.n_kv_heads;  // per-sequence predictors at most
  p.kt_off = after_err;
  p.w1h_off = align256(p.kt_off + (size_t)s.batch * s.T * D * 2);
  p.wlh_off = align256(p.w1h_off + heads * s.hidden * 128 * 2);
  p.w2h_off = align256(p.wlh_off + heads * 128 * 128 * 2);
  p.ws_bytes = align256(p.w2h_off + heads * 128 * s.hidden * 2);
  return p;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& plan, lr_dtype dt, cudaStream_t st) {
  cudaError_t e;
  if (plan.path == DecodePath::Pair) {
    tc::PairArgs t{};
    t.B = a.B; t.T = a.T; t.L = a.L; t.Hkv = a.Hkv; t.G = a.G; t.H = a.H; t.r = a.r;
    t.layer = a.layer; t.k = a.k; t.nblk = a.nblk; t.pred_per_seq = a.pred_per_seq;
    t.n_pairs = plan.n_pairs;
    t.scale = a.scale;
    t.q = (const __nv_bfloat16*)a.q;
    t.b1 = (const __nv_bfloat16*)a.b1;
    t.W1 = (const __nv_bfloat16*)a.W1;
    t.Bt = (const __nv_bfloat16*)a.Bt;
    t.qhat = (__nv_bfloat16*)((char*)a.err + plan.qhat_off);
    t.W1h = (__half*)((char*)a.err + plan.w1h_off);
    t.w1_seqs = a.pred_per_seq ? a.B : 1;
    t.res_idx = a.res_idx;
    t.res_val = (const __nv_bfloat16*)a.res_val;
    t.res_codes = a.res_codes;
    t.res_lo = a.res_lo;
    t.res_step = a.res_step;
    t.res_ptr = a.res_ptr;
    t.sched = a.blocks ? (int*)((char*)a.err + plan.sched_off) : nullptr;
    t.sched_stride = 1 + a.n_sel;
    t.partials = a.partials;
    t.part_stride = plan.part_stride;
    t.err = a.err;
    const cuuint64_t D = (cuuint64_t)a.L * a.Hkv * a.hd;
    CUtensorMap mA, mB0, mB1, mQ, mW1;
    const cuuint64_t dQ[2] = {(cuuint64_t)a.r, (cuuint64_t)a.B * a.Hkv * tc::kPairQRows};
    const cuuint64_t sQ[1] = {(cuuint64_t)a.r * 2};
    const cuuint32_t bQ[2] = {64, (cuuint32_t)tc::kPairQRows};
    const cuuint64_t dA[3] = {(cuuint64_t)a.r, (cuuint64_t)a.T, (cuuint64_t)a.B};
    const cuuint64_t sA[2] = {(cuuint64_t)a.r * 2, (cuuint64_t)a.T * a.r * 2};
    const cuuint32_t bA[3] = {64, 64, 1};
    const cuuint64_t dB[3] = {(cuuint64_t)a.r, D, (cuuint64_t)a.B};
    const cuuint64_t sB[2] = {(cuuint64_t)a.r * 2, D * a.r * 2};
    const cuuint32_t bB0[3] = {64, 72, 1};
    const cuuint32_t bB1[3] = {64, 56, 1};
    const cuuint64_t w1_rows = (cuuint64_t)t.w1_seqs * a.Hkv * a.H;
    const cuuint64_t dW[2] = {(cuuint64_t)a.hd, w1_rows};
    const cuuint64_t sW[1] = {(cuuint64_t)a.hd * 2};
    const cuuint32_t bW[2] = {64, 64};
    if (!tile_map(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.A, 3, dA, sA, bA) ||
        !tile_map(&mB0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Bt, 3, dB, sB, bB0) ||
        !tile_map(&mB1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Bt, 3, dB, sB, bB1) ||
        !tile_map(&mQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, t.qhat, 2, dQ, sQ, bQ) ||
        !tile_map(&mW1, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, t.W1h, 2, dW, sW, bW))
      return cudaErrorInvalidValue;
    if ((e = tc::launch_decode_pair(t, mA, mB0, mB1, mQ, mW1, a.blocks, a.n_sel, st)) != cudaSuccess) return e;
    return launch_decode_combine(a, dt, st);
  }
  e = launch_decode_general(a, dt, st);
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, dt, st);
}

namespace {
// The tensor-core pack: projection and key rebuild on the CTA-pair GEMM, the predictor and
// its error on the fused predictor kernel, the exact top-k, then the residual rows of the
// kept tokens recomputed by the same predictor kernel in gather mode.
cudaError_t launch_pack_tc(const PackArgs& a, const PackPlan& plan, cudaStream_t st) {
  char* ws = (char*)a.errword;
  void* Kt = ws + plan.kt_off;
  void* W1h = ws + plan.w1h_off;
  void* Wlh = ws + plan.wlh_off;
  void* W2h = ws + plan.w2h_off;
  const cuuint64_t B = (cuuint64_t)a.B, T = (cuuint64_t)a.T, D = (cuuint64_t)a.D, r = (cuuint64_t)a.r;
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // P1: A = round(K_group . Bt)
  tc::GemmArgs g1{};
  g1.B = a.B; g1.M = a.T; g1.N = a.r; g1.K = a.D; g1.bn = a.r % 256 == 0 ? 256 : 128;
  g1.b_mn_major = true; g1.out_f16 = false; g1.err = a.errword;
  CUtensorMap mA1, mB1, mC1;
  {
    const cuuint64_t dA[3] = {D, T, B}, sA[2] = {D * 2, T * D * 2};
    const cuuint32_t bA[3] = {64, 128, 1};
    const cuuint64_t dB[3] = {r, D, B}, sB[2] = {r * 2, D * r * 2};
    const cuuint32_t bB[3] = {64, 64, 1};
    const cuuint64_t dC[3] = {r, T, B}, sC[2] = {r * 2, T * r * 2};
    const cuuint32_t bC[3] = {64, 32, 1};
    if (!tile_map(&mA1, BF, a.K, 3, dA, sA, bA) || !tile_map(&mB1, BF, a.Bt, 3, dB, sB, bB) ||
        !tile_map(&mC1, BF, a.A, 3, dC, sC, bC))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = tc::launch_gemm_pair(g1, mA1, mB1, mC1, st);
  if (e != cudaSuccess) return e;
  // P2: K~ = A . Bt^T, every (layer, KV head) slice at once, fp16
  tc::GemmArgs g2{};
  g2.B = a.B; g2.M = a.T; g2.N = a.D; g2.K = a.r; g2.bn = a.D % 256 == 0 ? 256 : 128;
  g2.b_mn_major = false; g2.out_f16 = true; g2.err = a.errword;
  CUtensorMap mA2, mB2, mC2;
  {
    const cuuint64_t dA[3] = {r, T, B}, sA[2] = {r * 2, T * r * 2};
    const cuuint32_t bA[3] = {64, 128, 1};
    const cuuint64_t dB[3] = {r, D, B}, sB[2] = {r * 2, D * r * 2};
    const cuuint32_t bB[3] = {64, (cuuint32_t)(g2.bn / 2), 1};
    const cuuint64_t dC[3] = {D, T, B}, sC[2] = {D * 2, T * D * 2};
    const cuuint32_t bC[3] = {64, 32, 1};
    if (!tile_map(&mA2, BF, a.A, 3, dA, sA, bA) || !tile_map(&mB2, BF, a.Bt, 3, dB, sB, bB) ||
        !tile_map(&mC2, F16, Kt, 3, dC, sC, bC))
      return cudaErrorInvalidValue;
  }
  if ((e = tc::launch_gemm_pair(g2, mA2, mB2, mC2, st)) != cudaSuccess) return e;
  // fp16 predictor weights
  const int n_heads = (a.pred_per_seq ? a.B : 1) * a.L * a.Hkv;
  if ((e = tc::launch_weights_f16(a.W1, a.W_lin, a.W2, n_heads, a.H, W1h, Wlh, W2h, st)) != cudaSuccess) return e;
  CUtensorMap mKt, mW1, mWl, mW2;
  {
    const cuuint64_t dK[3] = {D, T, B}, sK[2] = {D * 2, T * D * 2};
    const cuuint32_t bK[3] = {64, 128, 1};
    const cuuint64_t H = (cuuint64_t)a.H, nh = (cuuint64_t)n_heads;
    const cuuint64_t d1[2] = {128, nh * H}, s1[1] = {256};
    const cuuint64_t dl[2] = {128, nh * 128}, sl[1] = {256};
    const cuuint64_t d2[2] = {H, nh * 128}, s2[1] = {H * 2};
    const cuuint32_t bw[2] = {64, 128};
    if (!tile_map(&mKt, F16, Kt, 3, dK, sK, bK) || !tile_map(&mW1, F16, W1h, 2, d1, s1, bw) ||
        !tile_map(&mWl, F16, Wlh, 2, dl, sl, bw) || !tile_map(&mW2, F16, W2h, 2, d2, s2, bw))
      return cudaErrorInvalidValue;
  }
  tc::PredictArgs p{};
  p.B = a.B; p.T = a.T; p.L = a.L; p.Hkv = a.Hkv; p.H = a.H; p.D = a.D; p.k = a.k;
  p.pred_per_seq = a.pred_per_seq;
  p.gather = false;
  p.Kt = Kt; p.V = a.V; p.b1 = a.b1; p.b2 = a.b2; p.err = a.err;
  p.res_idx = a.res_idx; p.res_val = a.res_val; p.errword = a.errword;
  // P3 + P4: predictor and per-token error of every token
  if ((e = tc::launch_pack_predict_tc(p, mKt, mW1, mWl, mW2, nullptr, nullptr, st)) != cudaSuccess) return e;
  // P5: exact top-k per (sequence, layer, KV head)
  const int n_seg = a.B * a.L * a.Hkv;
  if ((e = launch_topk(a.err, n_seg, a.T, a.k, a.res_idx, st)) != cudaSuccess) return e;
  // P6: residual rows of the kept tokens, recomputed; block pointers
  if (a.k > 0) {
    p.gather = true;
    if ((e = tc::launch_pack_predict_tc(p, mKt, mW1, mWl, mW2, nullptr, nullptr, st)) != cudaSuccess) return e;
  }
  if (a.res_ptr) return launch_block_ptr(a.res_idx, n_seg, a.k, a.T, a.res_ptr, st);
  return cudaSuccess;
}
}  // namespace

FitPlan plan_fit(const lr_cache_shape& s, int per_sequence, int sm_count) {
  FitPlan p{};
  const size_t D = (size_t)s.n_layers * s.n_kv_heads * s.head_dim;
  const size_t segs = (size_t)s.batch * s.n_layers * s.n_kv_heads;
  const size_t H = (size_t)s.hidden, T = (size_t)s.T;
  p.n_wh = (per_sequence ? s.batch : 1) * s.n_layers * s.n_kv_heads;
  p.gstride = tc::fit_grad_stride(s.hidden);
  p.grid = sm_count;
  p.kt_off = 256;
  p.r_off = align256(p.kt_off + (size_t)s.batch * T * D * 2);
  p.g_off = align256(p.r_off + segs * T * 128 * 2);
  p.du_off = align256(p.g_off + segs * T * H * 2);
  p.grad_off = align256(p.du_off + segs * T * H * 2);
  p.w1h_off = align256(p.grad_off + (size_t)p.n_wh * p.gstride * 4);
  p.wlh_off = align256(p.w1h_off + (size_t)p.n_wh * H * 128 * 2);
  p.w2h_off = align256(p.wlh_off + (size_t)p.n_wh * 128 * 128 * 2);
  p.ones_off = align256(p.w2h_off + (size_t)p.n_wh * 128 * H * 2);
  p.ws_bytes = align256(p.ones_off + 64 * 64 * 2);
  return p;
}

cudaError_t launch_fit(const lr_cache_shape& s, const FitCall& c, const FitPlan& plan, cudaStream_t st) {
  char* ws = (char*)c.ws;
  int* errword = (int*)ws;
  void* Kt = ws + plan.kt_off;
  const cuuint64_t B = (cuuint64_t)s.batch, T = (cuuint64_t)s.T, r = (cuuint64_t)s.rank;
  const cuuint64_t D = (cuuint64_t)s.n_layers * s.n_kv_heads * s.head_dim, H = (cuuint64_t)s.hidden;
  const cuuint64_t segs = B * s.n_layers * s.n_kv_heads;
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // rebuilt keys of every (layer, KV head): K~ = A . Bt^T (fp16), once for all steps
  tc::GemmArgs g2{};
  g2.B = s.batch; g2.M = s.T; g2.N = (int)D; g2.K = s.rank; g2.bn = D % 256 == 0 ? 256 : 128;
  g2.b_mn_major = false; g2.out_f16 = true; g2.err = errword;
  CUtensorMap mA2, mB2, mC2, mKt, mKt64, mW1, mWl, mW2, mR, mDU, mG, mOnes;
  {
    const cuuint64_t dA[3] = {r, T, B}, sA[2] = {r * 2, T * r * 2};
    const cuuint32_t bA[3] = {64, 128, 1};
    const cuuint64_t dB[3] = {r, D, B}, sB[2] = {r * 2, D * r * 2};
    const cuuint32_t bB[3] = {64, (cuuint32_t)(g2.bn / 2), 1};
    const cuuint64_t dK[3] = {D, T, B}, sK[2] = {D * 2, T * D * 2};
    const cuuint32_t bC[3] = {64, 32, 1}, bK[3] = {64, 128, 1}, b64[3] = {64, 64, 1};
    const cuuint64_t nh = (cuuint64_t)plan.n_wh;
    const cuuint64_t d1[2] = {128, nh * H}, s1[1] = {256};
    const cuuint64_t dl[2] = {128, nh * 128}, sl[1] = {256};
    const cuuint64_t d2[2] = {H, nh * 128}, s2[1] = {H * 2};
    const cuuint32_t bw[2] = {64, 128};
    const cuuint64_t dR[3] = {128, T, segs}, sR[2] = {256, T * 256};
    const cuuint64_t dU[3] = {H, T, segs}, sU[2] = {H * 2, T * H * 2};
    const cuuint64_t dO[2] = {64, 64}, sO[1] = {128};
    const cuuint32_t bO[2] = {64, 64};
    if (!tile_map(&mA2, BF, c.A, 3, dA, sA, bA) || !tile_map(&mB2, BF, c.Bt, 3, dB, sB, bB) ||
        !tile_map(&mC2, F16, Kt, 3, dK, sK, bC) || !tile_map(&mKt, F16, Kt, 3, dK, sK, bK) ||
        !tile_map(&mKt64, F16, Kt, 3, dK, sK, b64) ||
        !tile_map(&mW1, F16, ws + plan.w1h_off, 2, d1, s1, bw) || !tile_map(&mWl, F16, ws + plan.wlh_off, 2, dl, sl, bw) ||
        !tile_map(&mW2, F16, ws + plan.w2h_off, 2, d2, s2, bw) ||
        !tile_map(&mR, F16, ws + plan.r_off, 3, dR, sR, b64) || !tile_map(&mDU, F16, ws + plan.du_off, 3, dU, sU, b64) ||
        !tile_map(&mG, F16, ws + plan.g_off, 3, dU, sU, b64) || !tile_map(&mOnes, F16, ws + plan.ones_off, 2, dO, sO, bO))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = tc::launch_gemm_pair(g2, mA2, mB2, mC2, st);
  if (e != cudaSuccess) return e;
  if ((e = tc::launch_fit_ones(ws + plan.ones_off, st)) != cudaSuccess) return e;
  float* grad = (float*)(ws + plan.grad_off);
  if ((e = cudaMemsetAsync(grad, 0, (size_t)plan.n_wh * plan.gstride * 4, st)) != cudaSuccess) return e;
  tc::FitUpdateArgs u{};
  u.n_heads = plan.n_wh; u.H = s.hidden; u.gstride = plan.gstride;
  u.grad = grad;
  u.W_lin = c.W_lin; u.W1 = c.W1; u.b1 = c.b1; u.W2 = c.W2; u.b2 = c.b2;
  u.Wlh = (__half*)(ws + plan.wlh_off); u.W1h = (__half*)(ws + plan.w1h_off); u.W2h = (__half*)(ws + plan.w2h_off);
  u.out_bf16 = s.dtype == LR_BF16;
  u.lr = 0.f; u.scale = 0.f;  // fp16 copies of the starting weights only
  if (c.n_steps == 0) {
    u.out_Wl = c.out_Wl; u.out_W1 = c.out_W1; u.out_b1 = c.out_b1; u.out_W2 = c.out_W2; u.out_b2 = c.out_b2;
  }
  if ((e = tc::launch_fit_update(u, st)) != cudaSuccess) return e;
  tc::PredictArgs p{};
  p.B = s.batch; p.T = s.T; p.L = s.n_layers; p.Hkv = s.n_kv_heads; p.H = s.hidden; p.D = (int)D; p.k = 0;
  p.pred_per_seq = c.per_sequence;
  p.gather = false;
  p.fit = true;
  p.Kt = Kt; p.V = c.V; p.b1 = c.b1; p.b2 = nullptr; p.b1f = c.b1; p.b2f = c.b2;
  p.DUout = ws + plan.du_off;
  CUtensorMap mGst, mRst;  // g and R leave the forward kernel through TMA stores
  {
    const cuuint64_t dR[3] = {128, T, segs}, sR[2] = {256, T * 256};
    const cuuint64_t dU[3] = {H, T, segs}, sU[2] = {H * 2, T * H * 2};
    const cuuint32_t b128[3] = {64, 128, 1};
    if (!tile_map(&mGst, F16, ws + plan.g_off, 3, dU, sU, b128) || !tile_map(&mRst, F16, ws + plan.r_off, 3, dR, sR, b128))
      return cudaErrorInvalidValue;
  }
  p.errword = errword;
  tc::FitGradArgs ga{};
  ga.B = s.batch; ga.T = s.T; ga.L = s.n_layers; ga.Hkv = s.n_kv_heads; ga.H = s.hidden;
  ga.pred_per_seq = c.per_sequence; ga.grad = grad; ga.gstride = plan.gstride; ga.errword = errword;
  {
    const int nkind = 2 + s.hidden / 128;
    const long long per_split = (long long)segs * nkind;
    const int nkc = (s.T + 63) / 64;
    long long S = (2LL * plan.grid + per_split - 1) / per_split;
    if (S > nkc) S = nkc;
    if (S < 1) S = 1;
    ga.S = (int)S;
  }
  u.lr = c.lr;
  u.scale = 2.0f / ((float)s.T * (c.per_sequence ? 1.0f : (float)s.batch) * (float)s.head_dim);
  for (int step = 0; step < c.n_steps; ++step) {
    if ((e = tc::launch_pack_predict_tc(p, mKt, mW1, mWl, mW2, &mGst, &mRst, st)) != cudaSuccess) return e;
    if ((e = tc::launch_fit_grad(ga, mR, mDU, mG, mKt64, mOnes, st)) != cudaSuccess) return e;
    if (step == c.n_steps - 1) {
      u.out_Wl = c.out_Wl; u.out_W1 = c.out_W1; u.out_b1 = c.out_b1; u.out_W2 = c.out_W2; u.out_b2 = c.out_b2;
    }
    if ((e = tc::launch_fit_update(u, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_pack(const PackArgs& a, const PackPlan& plan, lr_dtype dt, cudaStream_t st) {
  if (a.T == 0) return launch_block_ptr(a.res_idx, a.res_ptr ? a.B * a.L * a.Hkv : 0, a.k, a.T, a.res_ptr, st);
  if (plan.tensor) return launch_pack_tc(a, plan, st);
  cudaError_t e = launch_pack_project_general(a, dt, st);
  if (e != cudaSuccess) return e;
  if ((e = launch_pack_predict_general(a, dt, st)) != cudaSuccess) return e;
  const int n_seg = a.B * a.L * a.Hkv;
  if ((e = launch_topk(a.err, n_seg, a.T, a.k, a.res_idx, st)) != cudaSuccess) return e;
  if ((e = launch_pack_gather(a, dt, st)) != cudaSuccess) return e;
  if (a.res_ptr) return launch_block_ptr(a.res_idx, n_seg, a.k, a.T, a.res_ptr, st);
  return cudaSuccess;
}

}  // namespace lr
