// CUDA-core building blocks shared by the general decode and pack kernels: the
// per-tile key rebuild k~ = A_tile . B_l^h and the GELU branch of the predictor.
#pragma once

#include "lr_common.cuh"

namespace lr {
namespace general {

constexpr int TT = 32;   // tokens per tile
constexpr int KC = 32;   // reduction chunk staged in shared memory
constexpr int NT = 256;  // threads per CTA
constexpr int kMaxOutK = 32;  // TT * 256 / NT: outputs per thread for hd <= 256
constexpr int HC = 128;  // hidden units per W1 pass

struct SmemPlan {
  int as, bs, ks, gs, ps, acc, qs, stat, total;
};

__host__ __device__ inline SmemPlan decode_smem_plan(int hd, int H, int G) {
  SmemPlan p;
  const int brow = hd > HC ? hd : HC;
  p.as = 0;
  p.bs = p.as + TT * (KC + 1);
  p.ks = p.bs + brow * (KC + 1);
  p.gs = p.ks + TT * (hd + 1);
  p.ps = p.gs + TT * (H + 1);
  p.acc = p.ps + G * TT;
  p.qs = p.acc + G * (2 * hd + H);
  p.stat = p.qs + G * hd;
  p.total = p.stat + 4 * G;
  return p;
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int lower_bound_i32(const int* a, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Ks[t][d] = sum_j A[t0 + t][j] * Bl[d][j] for t < nt (rows >= nt are zero);
// then Gs[t][c] = GELU(sum_d Ks[t][d] W1[c][d] + b1[c]).
template <typename T>
__device__ void tile_front(const T* __restrict__ A, int r, int t0, int nt, const T* __restrict__ Bl,
                           int hd, const HeadPredictor<T>& P, int H, float* sm, const SmemPlan& sp) {
  const int tid = threadIdx.x;
  float* As = sm + sp.as;
  float* Bs = sm + sp.bs;
  float* Ks = sm + sp.ks;
  float* Gs = sm + sp.gs;
  const int n_out = TT * hd / NT;  // hd is a multiple of 8
  float kacc[kMaxOutK];
#pragma unroll
  for (int i = 0; i < kMaxOutK; ++i) kacc[i] = 0.f;
  for (int c0 = 0; c0 < r; c0 += KC) {
    const int cn = min(KC, r - c0);
    for (int x = tid; x < TT * KC; x += NT) {
      const int t = x / KC, j = x % KC;
      As[t * (KC + 1) + j] = (t < nt && j < cn) ? to_f32(A[(size_t)(t0 + t) * r + c0 + j]) : 0.f;
    }
    for (int x = tid; x < hd * KC; x += NT) {
      const int d = x / KC, j = x % KC;
      Bs[d * (KC + 1) + j] = j < cn ? to_f32(Bl[(size_t)d * r + c0 + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxOutK; ++i) {
      if (i < n_out) {
        const int o = tid + NT * i;
        const int t = o / hd, d = o % hd;
        const float* ar = As + t * (KC + 1);
        const float* br = Bs + d * (KC + 1);
        float s = kacc[i];
#pragma unroll 8
        for (int j = 0; j < KC; ++j) s = fmaf(ar[j], br[j], s);
        kacc[i] = s;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kMaxOutK; ++i) {
    if (i < n_out) {
      const int o = tid + NT * i;
      Ks[(o / hd) * (hd + 1) + (o % hd)] = kacc[i];
    }
  }
  __syncthreads();
  // GELU branch, HC hidden units per pass
  for (int cc0 = 0; cc0 < H; cc0 += HC) {
    const int ccn = min(HC, H - cc0);
    float uacc[TT * HC / NT];
#pragma unroll
    for (int i = 0; i < TT * HC / NT; ++i) uacc[i] = 0.f;
    for (int d0 = 0; d0 < hd; d0 += KC) {
      const int dn = min(KC, hd - d0);
      for (int x = tid; x < HC * KC; x += NT) {
        const int c = x / KC, j = x % KC;
        Bs[c * (KC + 1) + j] = (c < ccn && j < dn) ? to_f32(P.W1[(size_t)(cc0 + c) * hd + d0 + j]) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < TT * HC / NT; ++i) {
        const int o = tid + NT * i;
        const int t = o / HC, c = o % HC;
        const float* kr = Ks + t * (hd + 1) + d0;
        const float* wr = Bs + c * (KC + 1);
        float s = uacc[i];
        for (int j = 0; j < dn; ++j) s = fmaf(kr[j], wr[j], s);
        uacc[i] = s;
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TT * HC / NT; ++i) {
      const int o = tid + NT * i;
      const int t = o / HC, c = o % HC;
      if (c < ccn) Gs[t * (H + 1) + cc0 + c] = gelu_erf(uacc[i] + to_f32(P.b1[cc0 + c]));
    }
  }
  __syncthreads();
}

}  // namespace general
}  // namespace lr
