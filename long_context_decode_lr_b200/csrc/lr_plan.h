// Workspace plans and kernel dispatch of the decode and pack calls (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "lowram.h"

namespace lr {

struct DecodeArgs;
struct PackArgs;

enum class DecodePath { General = 0, Pair = 2 };

struct DecodePlan {
  DecodePath path;
  int n_split;       // split partials per query head
  int n_pairs;       // pair path: CTA pairs per (sequence, KV head)
  int part_stride;   // floats per split partial
  size_t part_off;   // byte offset of the partials in the workspace
  size_t sched_off;  // byte offset of the pair path's block schedule
  size_t w1h_off;    // byte offset of the pair path's fp16 copy of the layer's W1
  size_t qhat_off;   // byte offset of the pair path's Qhat operand
  size_t ws_bytes;   // total workspace
};

struct PackPlan {
  bool tensor;       // tensor-core projection / key rebuild / predictor kernels
  size_t err_off;    // fp32 errors when the caller passes no err_out
  size_t diff_off;   // CUDA-core path: round(v - v_hat) for every token
  size_t kt_off;     // tensor path: fp16 rebuilt keys K~ [B, T, D]
  size_t w1h_off;    // tensor path: fp16 copies of W1, W_lin, W2
  size_t wlh_off;
  size_t w2h_off;
  size_t ws_bytes;
};

bool pack_tc_supported(const lr_cache_shape& s);

// Test-time fitting: workspace layout and the whole fit (rebuilt keys, then n_steps of
// forward, gradient and update launches).
struct FitPlan {
  size_t kt_off, r_off, g_off, du_off, grad_off, w1h_off, wlh_off, w2h_off, ones_off, ws_bytes;
  int n_wh, gstride, grid;
};
FitPlan plan_fit(const lr_cache_shape& s, int per_sequence, int sm_count);
struct FitCall {
  const void* A;
  const void* Bt;
  const void* V;
  float *W_lin, *W1, *b1, *W2, *b2;
  int per_sequence;
  int n_steps;
  float lr;
  void *out_Wl, *out_W1, *out_b1, *out_W2, *out_b2;
  void* ws;
};
cudaError_t launch_fit(const lr_cache_shape& s, const FitCall& c, const FitPlan& plan, cudaStream_t st);

bool decode_pair_supported(const lr_cache_shape& s, int n_q_heads);
DecodePlan plan_decode(const lr_cache_shape& s, int n_q_heads, int n_sel, int sm_count);
PackPlan plan_pack(const lr_cache_shape& s, int k);

cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& plan, lr_dtype dt, cudaStream_t st);
cudaError_t launch_pack(const PackArgs& a, const PackPlan& plan, lr_dtype dt, cudaStream_t st);

}  // namespace lr
