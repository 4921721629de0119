// On-GPU block selection: which 64-token blocks of the compressed cache the current query
// rebuilds (selective reconstruction, arXiv abstract; "Predicting the value cache from
// keys", paragraph on prefill and decode costs). The pages' trained selector is not
// available; a block's key is the mean of its rebuilt keys and its score for KV head h is
//   s_j = max_g scale * q_g . mean_{t in block j} k~_t = max_g Qhat_g . mean_{t in block j} A_t,
// with Qhat_g = scale * B_l^h q_g (the mean commutes with the linear key rebuild, so the
// score needs one mean of A rows per block and one rank-space dot product per query head).
// The n_sel blocks of highest score per (sequence, KV head) are then chosen by the exact
// top-k of topk.cu (ties to the lower block id, ascending).
#include "lr_common.cuh"
#include "lr_launch.h"

namespace lr {
namespace {

constexpr int SEL_THREADS = 256;

__device__ __forceinline__ float sel_warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Qhat [B, Hkv, G, r] fp32: one block per (KV head, sequence), threads over rank columns.
template <typename T>
__global__ void __launch_bounds__(SEL_THREADS) select_qhat_kernel(SelectArgs a) {
  extern __shared__ float qs[];  // [G][hd], scaled queries
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = a.G, hd = a.hd, r = a.r;
  const T* q = (const T*)a.q + ((size_t)b * a.Hkv + h) * G * hd;
  for (int i = tid; i < G * hd; i += SEL_THREADS) qs[i] = to_f32(q[i]) * a.scale;
  __syncthreads();
  const size_t D = (size_t)a.L * a.Hkv * hd;
  const T* bt = (const T*)a.Bt + (size_t)b * D * r + (size_t)(a.layer * a.Hkv + h) * hd * r;
  float* out = a.qhat + ((size_t)b * a.Hkv + h) * G * r;
  for (int j = tid; j < r; j += SEL_THREADS) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < hd; ++d) {
      const float v = to_f32(bt[(size_t)d * r + j]);
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < G) acc[g] = fmaf(v, qs[g * hd + d], acc[g]);
    }
#pragma unroll
    for (int g = 0; g < 8; ++g)
      if (g < G) out[(size_t)g * r + j] = acc[g];
  }
}

// Scores [B, Hkv, nblk]: one CTA per (block, sequence). The block's mean A row goes to
// shared memory; each warp then takes (KV head, query head) pairs, one rank-space dot
// product each, and the maximum over a head's query heads is the block's score.
template <typename T>
__global__ void __launch_bounds__(SEL_THREADS) select_score_kernel(SelectArgs a) {
  extern __shared__ float abar[];  // [r], then [Hkv * G] dot products
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = a.r, G = a.G, Hkv = a.Hkv;
  const int t0 = j * kBlock, t1 = min(a.T, t0 + kBlock);
  const T* A = (const T*)a.A + ((size_t)b * a.T + t0) * r;
  const float inv_n = 1.f / (float)(t1 - t0);
  for (int c = tid; c < r; c += SEL_THREADS) {
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    int t = 0;
    for (; t + 4 <= t1 - t0; t += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) s[u] += to_f32(A[(size_t)(t + u) * r + c]);
    }
    for (; t < t1 - t0; ++t) s[0] += to_f32(A[(size_t)t * r + c]);
    abar[c] = ((s[0] + s[1]) + (s[2] + s[3])) * inv_n;
  }
  __syncthreads();
  float* dots = abar + r;
  for (int p = warp; p < Hkv * G; p += SEL_THREADS / 32) {
    const float* qh = a.qhat + ((size_t)b * Hkv * G + p) * r;
    float acc = 0.f;
    for (int c = lane; c < r; c += 32) acc = fmaf(qh[c], abar[c], acc);
    acc = sel_warp_sum(acc);
    if (lane == 0) dots[p] = acc;
  }
  __syncthreads();
  for (int h = tid; h < Hkv; h += SEL_THREADS) {
    float m = dots[h * G];
    for (int g = 1; g < G; ++g) m = fmaxf(m, dots[h * G + g]);
    a.scores[((size_t)b * Hkv + h) * a.nblk + j] = m;
  }
}

template <typename T>
cudaError_t launch_select_t(const SelectArgs& a, cudaStream_t st) {
  const size_t qs_bytes = (size_t)a.G * a.hd * sizeof(float);
  select_qhat_kernel<T><<<dim3(a.Hkv, a.B), SEL_THREADS, qs_bytes, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sc_bytes = ((size_t)a.r + (size_t)a.Hkv * a.G) * sizeof(float);
  e = cudaFuncSetAttribute(select_score_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc_bytes);
  if (e != cudaSuccess) return e;
  select_score_kernel<T><<<dim3(a.nblk, a.B), SEL_THREADS, sc_bytes, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_topk(a.scores, a.B * a.Hkv, a.nblk, a.n_sel, a.blocks_out, st);
}

}  // namespace

cudaError_t launch_select_blocks(const SelectArgs& a, lr_dtype dt, cudaStream_t st) {
  if (a.B == 0 || a.nblk == 0) return cudaSuccess;
  return dt == LR_BF16 ? launch_select_t<__nv_bfloat16>(a, st) : launch_select_t<float>(a, st);
}

}  // namespace lr
