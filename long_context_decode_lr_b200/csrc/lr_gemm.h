// Internal interface of the tensor-core kernels of the packer: the persistent CTA-pair
// GEMM (gemm_pair.cu) and the fused predictor / error kernel (pack_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace lr {
namespace tc {

// C[b, m, n] = sum_k Aop[b, m, k] Bop[b, n, k]; bf16 operands, fp32 accumulation, C in
// bf16 (round to nearest even) or fp16 (saturating). Tensor maps (128-byte swizzle):
//   mA over Aop [B, M, K], box {64, 128, 1};
//   mB over Bop [B, N, K], box {64, bn / 2, 1} (K-major), or over [B, K, N], box {64, 64, 1}
//      (b_mn_major);
//   mC over C [B, M, N], box {64, 32, 1}.
// Requirements: K % 64 == 0, N % bn == 0, bn in {128, 256}; M is arbitrary.
struct GemmArgs {
  int B, M, N, K;
  int bn;
  bool b_mn_major;
  bool out_f16;
  int* err;  // device error word (LR_DEVERR_TIMEOUT / LR_DEVERR_LAUNCH)
};
cudaError_t launch_gemm_pair(const GemmArgs& g, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC,
                             cudaStream_t st);

// Fused predictor of the packer, one (sequence, layer, KV head) segment at a time, 128 rows
// per tile: U = k~ W1^T, g = GELU(U + b1), v_hat = k~ W_lin^T + g W2^T + b2 on the tensor
// cores (fp16 operands, fp32 accumulation), then per row d = v - v_hat and
//   normal mode: err[seg, t] = sum_j d_j^2 for every token t;
//   gather mode: res_val[seg, i] = round(d) for the rows t = res_idx[seg, i].
struct PredictArgs {
  int B, T, L, Hkv, H, D, k;
  int pred_per_seq;
  bool gather;
  // fitting mode (test-time fitting of the predictor): per row R = v_hat - v, g = GELU(u),
  // dU' = (R W2) * GELU'(u) with u = k~ W1^T + b1; R, g and dU' go to global memory (fp16) for
  // the gradient contractions, and the biases come from the fp32 master copies
  bool fit;
  const float* b1f;      // fit: [(B,) L, Hkv, H] fp32
  const float* b2f;      // fit: [(B,) L, Hkv, 128] fp32 or null
  void* DUout;           // fit: [B * L * Hkv, T, H] fp16
  const void* Kt;        // [B, T, D] fp16 rebuilt keys of every (layer, KV head)
  const void* V;         // [B, L, T, Hkv, 128] bf16
  const void* b1;        // [(B,) L, Hkv, H] bf16
  const void* b2;        // [(B,) L, Hkv, 128] bf16 or null
  float* err;            // [B, L, Hkv, T]
  const int* res_idx;    // gather mode: [B, L, Hkv, k]
  void* res_val;         // gather mode: [B, L, Hkv, k, 128] bf16
  int* errword;
};
// Maps: mKt over Kt [B, T, D] fp16, box {64, 128, 1}; mW1 over the fp16 W1 copy
// [S * L * Hkv * H, 128], box {64, 128}; mWl over the fp16 W_lin copy [S * L * Hkv * 128, 128],
// box {64, 128}; mW2 over the fp16 W2 copy [S * L * Hkv * 128, H], box {64, 128}
// (S = B with per-sequence predictors, else 1).
// Fitting mode also takes mG over g [segs, T, H] and mR over R [segs, T, 128] (fp16, box
// {64, 128, 1}): the g halves and R leave shared memory through TMA stores (null elsewhere).
cudaError_t launch_pack_predict_tc(const PredictArgs& a, const CUtensorMap& mKt, const CUtensorMap& mW1,
                                   const CUtensorMap& mWl, const CUtensorMap& mW2, const CUtensorMap* mG,
                                   const CUtensorMap* mR, cudaStream_t st);

// fp16 copies of the predictor weights (saturating): W1 [n, H, 128], W_lin [n, 128, 128],
// W2 [n, 128, H] for n = S * L * Hkv heads.
cudaError_t launch_weights_f16(const void* W1, const void* Wl, const void* W2, int n_heads, int H, void* W1h,
                               void* Wlh, void* W2h, cudaStream_t st);

}  // namespace tc
}  // namespace lr
