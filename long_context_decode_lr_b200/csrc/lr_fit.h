// Internal interface of test-time predictor fitting (fit.cu; the forward pass is the fitting
// mode of the packer's predictor kernel, pack_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace lr {
namespace tc {

// fp32 gradient sums per weight head, in this order: dW_lin [128, 128], dW1 [H, 128],
// dW2 [128, H], db1 [H], db2 [128].
__host__ __device__ inline int fit_grad_stride(int H) { return 128 * 128 + 2 * H * 128 + H + 128; }

struct FitGradArgs {
  int B, T, L, Hkv, H;
  int S;              // token splits per (segment, kind): 1 <= S <= ceil(T / 64)
  int pred_per_seq;
  float* grad;        // [n weight heads, fit_grad_stride(H)]
  int gstride;
  int* errword;
};
// Maps (fp16, 128-byte swizzle): mR over R [segs, T, 128], box {64, 64, 1}; mDU and mG over
// dU' and g [segs, T, H], box {64, 64, 1}; mKt over K~ [B, T, D], box {64, 64, 1}; mOnes over
// the [64, 64] ones tile, box {64, 64}.
cudaError_t launch_fit_grad(const FitGradArgs& a, const CUtensorMap& mR, const CUtensorMap& mDU, const CUtensorMap& mG,
                            const CUtensorMap& mKt, const CUtensorMap& mOnes, cudaStream_t st);

struct FitUpdateArgs {
  int n_heads, H, gstride;
  float lr, scale;    // theta -= lr * scale * sum
  float* grad;
  float *W_lin, *W1, *b1, *W2, *b2;  // fp32 masters (b2 may be null)
  __half *Wlh, *W1h, *W2h;           // fp16 copies for the forward pass
  void *out_Wl, *out_W1, *out_b1, *out_W2, *out_b2;  // storage-dtype copies or null
  bool out_bf16;
};
cudaError_t launch_fit_update(const FitUpdateArgs& a, cudaStream_t st);
cudaError_t launch_fit_ones(void* ones, cudaStream_t st);

__device__ __forceinline__ void store_dtype(void* p, size_t o, float w, bool bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(p)[o] = __float2bfloat16_rn(w);
  else reinterpret_cast<float*>(p)[o] = w;
}

}  // namespace tc
}  // namespace lr
