// On-GPU block selection: which 64-token blocks of the compressed cache the current query
// rebuilds (selective reconstruction, arXiv abstract; "Predicting the value cache from
// keys", paragraph on prefill and decode costs). The pages' trained selector is not
// available; a block's key is the mean of its rebuilt keys and its score for KV head h is
//   s_j = max_g scale * q_g . mean_{t in block j} k~_t = max_g Qhat_g . Abar_j,
// with Qhat_g = scale * B_l^h q_g and Abar_j the mean of the block's A rows (the mean
// commutes with the linear key rebuild). Abar does not depend on the query: it is formed
// once per packed cache (block_means_kernel), so a selection step reads 1/64 of A. The n_sel
// blocks of highest score per (sequence, KV head) are then chosen by the exact top-k of
// topk.cu (ties to the lower block id, ascending).
#include <math_constants.h>

#include <algorithm>

#include "lr_common.cuh"
#include "lr_launch.h"

namespace lr {
namespace {

constexpr int SEL_THREADS = 256;

// 8 consecutive storage elements as fp32 (one 16-byte load for bf16, two for fp32).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Abar [B, nblk, r] fp32: one CTA per (block, sequence); a thread owns 8 rank columns and
// sums the block's rows (up to 64) with four independent partial sums.
template <typename T>
__global__ void __launch_bounds__(SEL_THREADS) block_means_kernel(const T* __restrict__ A, int T_len, int r,
                                                                  float* __restrict__ abar) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int t0 = j * kBlock, n = min(T_len, t0 + kBlock) - t0;
  const float inv_n = 1.f / (float)n;
  const T* src = A + ((size_t)b * T_len + t0) * r;
  float* dst = abar + ((size_t)b * gridDim.x + j) * r;
  for (int c = threadIdx.x * 8; c < r; c += SEL_THREADS * 8) {
    float s[4][8] = {};
    int t = 0;
    for (; t + 4 <= n; t += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float v[8];
        load8<T>(src + (size_t)(t + u) * r + c, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[u][i] += v[i];
      }
    }
    for (; t < n; ++t) {
      float v[8];
      load8<T>(src + (size_t)t * r + c, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) s[0][i] += v[i];
    }
    float4 o0, o1;
    o0.x = ((s[0][0] + s[1][0]) + (s[2][0] + s[3][0])) * inv_n;
    o0.y = ((s[0][1] + s[1][1]) + (s[2][1] + s[3][1])) * inv_n;
    o0.z = ((s[0][2] + s[1][2]) + (s[2][2] + s[3][2])) * inv_n;
    o0.w = ((s[0][3] + s[1][3]) + (s[2][3] + s[3][3])) * inv_n;
    o1.x = ((s[0][4] + s[1][4]) + (s[2][4] + s[3][4])) * inv_n;
    o1.y = ((s[0][5] + s[1][5]) + (s[2][5] + s[3][5])) * inv_n;
    o1.z = ((s[0][6] + s[1][6]) + (s[2][6] + s[3][6])) * inv_n;
    o1.w = ((s[0][7] + s[1][7]) + (s[2][7] + s[3][7])) * inv_n;
    reinterpret_cast<float4*>(dst + c)[0] = o0;
    reinterpret_cast<float4*>(dst + c)[1] = o1;
  }
}

// Qhat [B, Hkv * G, r] fp32: one CTA per (32 rank columns, KV head, sequence). Warp w sums
// the key dims d = w, w + 8, ... for rank column lane (loads issued 16 at a time); an 8-way
// reduction in shared memory.
template <typename T>
__global__ void __launch_bounds__(SEL_THREADS) select_qhat_kernel(SelectArgs a) {
  __shared__ float qs[8][256];
  __shared__ float part[8][32][9];
  const int jc = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int G = a.G, hd = a.hd, r = a.r;
  const T* q = (const T*)a.q + ((size_t)b * a.Hkv + h) * G * hd;
  for (int i = tid; i < G * hd; i += SEL_THREADS) qs[i / hd][i % hd] = to_f32(q[i]) * a.scale;
  __syncthreads();
  const int c = tid & 31, dg = tid >> 5;
  const int j = jc * 32 + c;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (j < r) {
    const size_t D = (size_t)a.L * a.Hkv * hd;
    const T* bt = (const T*)a.Bt + (size_t)b * D * r + (size_t)(a.layer * a.Hkv + h) * hd * r + j;
    for (int d0 = dg; d0 < hd; d0 += 8 * 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int d = d0 + 8 * u;
        v[u] = d < hd ? to_f32(bt[(size_t)d * r]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int d = d0 + 8 * u;
        if (d >= hd) break;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (g < G) acc[g] = fmaf(v[u], qs[g][d], acc[g]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < 8; ++g) part[dg][c][g] = acc[g];
  __syncthreads();
  if (dg != 0 || j >= r) return;
  float* out = a.qhat + ((size_t)b * a.Hkv + h) * G * r + j;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if (g >= G) continue;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) x += part[w][c][g];
    out[(size_t)g * r] = x;
  }
}

constexpr int kScBlocks = 32;  // blocks per CTA (4 per warp)
constexpr int kScPairs = 32;   // (KV head, query head) pairs per pass: one per lane
constexpr int kScCols = 128;   // rank columns staged per pass
constexpr int kScPad = 4;      // Qhat row padding: 16-byte rows without bank conflicts
static_assert(kScBlocks == kScPairs && kScBlocks == 4 * SEL_THREADS / 32, "staging loop and warp split");

// Partial dot products [n_split, B, nblk, Hkv * G]: one CTA per (32 blocks, sequence, rank
// split); split z covers the 128-column chunks [z * n_chunks / n_split, (z + 1) * n_chunks /
// n_split). Lane l of every warp owns the (KV head, query head) pair l of the current pass
// and accumulates its dot products with the warp's 4 block means; rank columns are staged
// 128 at a time and read four at a time (Qhat rows padded against bank conflicts, block
// means read as broadcasts).
__global__ void __launch_bounds__(SEL_THREADS) select_score_kernel(SelectArgs a) {
  __shared__ __align__(16) float qs[kScPairs][kScCols + kScPad];
  __shared__ __align__(16) float as[kScBlocks][kScCols];
  const int j0 = blockIdx.x * kScBlocks, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = a.r, G = a.G, P = a.Hkv * G;
  const int nb = min(kScBlocks, a.nblk - j0);
  const float* qh = a.qhat + (size_t)b * P * r;
  const float* ab = a.abar + ((size_t)b * a.nblk + j0) * r;
  const int pass = (kScPairs / G) * G;  // whole heads per pass: a head never straddles two
  const int n_chunks = (r + kScCols - 1) / kScCols, z = blockIdx.z;
  const int c_begin = (z * n_chunks / a.n_split) * kScCols;
  const int c_end = min(r, ((z + 1) * n_chunks / a.n_split) * kScCols);
  for (int p0 = 0; p0 < P; p0 += pass) {
    const int np = min(pass, P - p0);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = c_begin; c0 < c_end; c0 += kScCols) {
      const int nc = min(kScCols, r - c0);  // r is a multiple of 8, so nc is a multiple of 4
      __syncthreads();
      for (int i = tid; i < kScPairs * (kScCols / 4); i += SEL_THREADS) {
        const int p = i / (kScCols / 4), c = 4 * (i % (kScCols / 4));
        const bool cin = c < nc;
        *reinterpret_cast<float4*>(&qs[p][c]) =
            (p < np && cin) ? __ldg(reinterpret_cast<const float4*>(qh + (size_t)(p0 + p) * r + c0 + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(&as[p][c]) =
            (p < nb && cin) ? __ldg(reinterpret_cast<const float4*>(ab + (size_t)p * r + c0 + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < kScCols; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(&qs[lane][c]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 av = *reinterpret_cast<const float4*>(&as[warp * 4 + i][c]);
          acc[i] = fmaf(qv.x, av.x, acc[i]);
          acc[i] = fmaf(qv.y, av.y, acc[i]);
          acc[i] = fmaf(qv.z, av.z, acc[i]);
          acc[i] = fmaf(qv.w, av.w, acc[i]);
        }
      }
    }
    float* part = a.partial + (((size_t)z * a.B + b) * a.nblk + j0) * P + p0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int blk = warp * 4 + i;
      if (blk < nb && lane < np) part[(size_t)blk * P + lane] = acc[i];
    }
  }
}

// Scores [B, Hkv, nblk]: s = max over the head's query heads of the summed partial dot
// products (splits added in a fixed order).
__global__ void __launch_bounds__(SEL_THREADS) select_reduce_kernel(SelectArgs a) {
  // one thread per (sequence, block, KV head), the head fastest: a warp reads contiguous
  // partial sums
  const long long x = (long long)blockIdx.x * SEL_THREADS + threadIdx.x;
  const long long n = (long long)a.B * a.Hkv * a.nblk;
  if (x >= n) return;
  const int h = (int)(x % a.Hkv), j = (int)((x / a.Hkv) % a.nblk), b = (int)(x / ((long long)a.nblk * a.Hkv));
  const int G = a.G, P = a.Hkv * G;
  // every partial sum is loaded before any is added (G <= 8, n_split <= 4)
  float t[4][8];
#pragma unroll
  for (int z = 0; z < 4; ++z)
#pragma unroll
    for (int g = 0; g < 8; ++g)
      t[z][g] = (z < a.n_split && g < G) ? a.partial[(((size_t)z * a.B + b) * a.nblk + j) * P + h * G + g] : 0.f;
  float m = -CUDART_INF_F;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    if (g >= G) break;
    const float v = ((t[0][g] + t[1][g]) + t[2][g]) + t[3][g];
    m = g == 0 ? v : fmaxf(m, v);
  }
  a.scores[((size_t)b * a.Hkv + h) * a.nblk + j] = m;
}

template <typename T>
cudaError_t launch_select_t(const SelectArgs& a, cudaStream_t st) {
  select_qhat_kernel<T><<<dim3((a.r + 31) / 32, a.Hkv, a.B), SEL_THREADS, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_score_kernel<<<dim3((a.nblk + kScBlocks - 1) / kScBlocks, a.B, a.n_split), SEL_THREADS, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long n = (long long)a.B * a.Hkv * a.nblk;
  select_reduce_kernel<<<(unsigned)((n + SEL_THREADS - 1) / SEL_THREADS), SEL_THREADS, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_topk(a.scores, a.B * a.Hkv, a.nblk, a.n_sel, a.blocks_out, st);
}

}  // namespace

int select_rank_splits(int r) { return std::max(1, std::min(4, (r + kScCols - 1) / kScCols)); }

cudaError_t launch_select_blocks(const SelectArgs& a, lr_dtype dt, cudaStream_t st) {
  if (a.B == 0 || a.nblk == 0) return cudaSuccess;
  return dt == LR_BF16 ? launch_select_t<__nv_bfloat16>(a, st) : launch_select_t<float>(a, st);
}

cudaError_t launch_block_means(const void* A, int B, int T, int r, lr_dtype dt, float* abar, cudaStream_t st) {
  const int nblk = ceil_div(T, kBlock);
  if (B == 0 || nblk == 0) return cudaSuccess;
  const dim3 grid(nblk, B);
  if (dt == LR_BF16)
    block_means_kernel<__nv_bfloat16><<<grid, SEL_THREADS, 0, st>>>((const __nv_bfloat16*)A, T, r, abar);
  else
    block_means_kernel<float><<<grid, SEL_THREADS, 0, st>>>((const float*)A, T, r, abar);
  return cudaGetLastError();
}

}  // namespace lr
