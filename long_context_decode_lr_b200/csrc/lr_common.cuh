// Shared device helpers and launch-argument structs of the LowRAM kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lowram.h"

namespace lr {

constexpr int kBlock = LR_BLOCK_TOKENS;  // tokens per selectable key block

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Round-to-nearest-even conversion from fp32 to the storage type.
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Exact-form GELU, x * Phi(x), through CUDA's erff.
__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

__device__ __forceinline__ void flag_error(int* word, int bits) {
  if (word) atomicOr(word, bits);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Predictor pointers for one (sequence, layer, KV head), already offset.
template <typename T>
struct HeadPredictor {
  const T* W_lin;  // [hd, hd]
  const T* W1;     // [H, hd]
  const T* b1;     // [H]
  const T* W2;     // [hd, H]
  const T* b2;     // [hd] or nullptr
};

// Everything a decode kernel needs; pointers are the caller's device buffers.
struct DecodeArgs {
  int B, T, L, Hkv, G, hd, r, H;
  int layer, k, n_sel, nblk;
  int pred_per_seq;
  float scale;
  const void* q;        // [B, Hq, hd]
  const void* A;        // [B, T, r]
  const void* Bt;       // [B, D, r]
  const void* W_lin;    // [(B,) L, Hkv, hd, hd]
  const void* W1;       // [(B,) L, Hkv, H, hd]
  const void* b1;       // [(B,) L, Hkv, H]
  const void* W2;       // [(B,) L, Hkv, hd, H]
  const void* b2;       // [(B,) L, Hkv, hd] or null
  const int* res_idx;   // [B, L, Hkv, k]
  const void* res_val;  // [B, L, Hkv, k, hd] rows in the cache dtype, or null with 2-bit rows
  const uint8_t* res_codes;  // 2-bit rows: [B, L, Hkv, k, hd / 4] codes (null otherwise)
  const float* res_lo;       // 2-bit rows: [B, L, Hkv, k] row minimum
  const float* res_step;     // 2-bit rows: [B, L, Hkv, k] level step
  const int* res_ptr;   // [B, L, Hkv, nblk + 1] or null
  const int* blocks;    // [B, Hkv, n_sel] or null
  const void* tail_K;   // [B, Hkv, n_tail, hd] exact recent tokens, or null
  const void* tail_V;   // [B, Hkv, n_tail, hd]
  int n_tail;
  void* o;              // [B, Hq, hd]
  float* partials;      // [B, Hq, n_split, part_stride]
  int n_split;
  int part_stride;      // floats per partial: 4 + hd + H + hd
  int* err;             // device error word
};

// Entry dd of residual row i of one (sequence, layer, KV head) segment: the stored value, or
// lo + code * step for 2-bit rows (seg_row = seg * k, the segment's first row).
template <typename T>
__device__ __forceinline__ float residual_entry(const DecodeArgs& a, size_t seg_row, int i, int dd) {
  const size_t row = seg_row + (size_t)i;
  if (a.res_codes) {
    const uint32_t byte = a.res_codes[row * (a.hd / 4) + (dd >> 2)];
    return fmaf((float)((byte >> (2 * (dd & 3))) & 3u), a.res_step[row], a.res_lo[row]);
  }
  return to_f32(((const T*)a.res_val)[row * a.hd + dd]);
}

template <typename T>
__device__ __forceinline__ HeadPredictor<T> head_predictor(const DecodeArgs& a, int b, int l, int h) {
  const size_t lh = (size_t)l * a.Hkv + h;
  const size_t per_seq_lh = (size_t)a.L * a.Hkv;
  const size_t s = a.pred_per_seq ? (size_t)b * per_seq_lh : 0;
  HeadPredictor<T> p;
  p.W_lin = (const T*)a.W_lin + (s + lh) * a.hd * a.hd;
  p.W1 = (const T*)a.W1 + (s + lh) * a.H * a.hd;
  p.b1 = (const T*)a.b1 + (s + lh) * a.H;
  p.W2 = (const T*)a.W2 + (s + lh) * a.hd * a.H;
  p.b2 = a.b2 ? (const T*)a.b2 + (s + lh) * a.hd : nullptr;
  return p;
}

// Block selection (select.cu): scores of every 64-token block per (sequence, KV head) and
// the top-n_sel block list.
struct SelectArgs {
  int B, T, L, Hkv, G, hd, r, layer, nblk, n_sel;
  float scale;
  const void* q;       // [B, Hq, hd]
  const float* abar;   // [B, nblk, r] block means of A
  const void* Bt;      // [B, D, r]
  float* qhat;         // workspace [B, Hkv, G, r]: scale * B_l^h q per query head
  float* scores;       // [B, Hkv, nblk]: the caller's scores_out, or workspace
  float* partial;      // workspace [n_split, B, nblk, Hkv * G]: partial dot products
  int n_split;         // rank splits of the score kernel (select_rank_splits(r))
  int* blocks_out;     // [B, Hkv, n_sel]
};

struct PackArgs {
  int B, T, L, Hkv, hd, r, H, D, k, nblk;
  int pred_per_seq;
  const void* K;        // [B, T, D]
  const void* V;        // [B, L, T, Hkv, hd]
  const void* Bt;       // [B, D, r]
  const void* W_lin;
  const void* W1;
  const void* b1;
  const void* W2;
  const void* b2;
  void* A;              // [B, T, r]
  float* err;           // [B, L, Hkv, T]
  void* diff;           // [B, L, Hkv, T, hd]: round(v - v_hat) for every token
  int* res_idx;         // [B, L, Hkv, k]
  void* res_val;        // [B, L, Hkv, k, hd]
  int* res_ptr;         // [B, L, Hkv, nblk + 1] or null
  int* errword;
};

template <typename T>
__device__ __forceinline__ HeadPredictor<T> head_predictor(const PackArgs& a, int b, int l, int h) {
  const size_t lh = (size_t)l * a.Hkv + h;
  const size_t s = a.pred_per_seq ? (size_t)b * a.L * a.Hkv : 0;
  HeadPredictor<T> p;
  p.W_lin = (const T*)a.W_lin + (s + lh) * a.hd * a.hd;
  p.W1 = (const T*)a.W1 + (s + lh) * a.H * a.hd;
  p.b1 = (const T*)a.b1 + (s + lh) * a.H;
  p.W2 = (const T*)a.W2 + (s + lh) * a.hd * a.H;
  p.b2 = a.b2 ? (const T*)a.b2 + (s + lh) * a.hd : nullptr;
  return p;
}

}  // namespace lr
