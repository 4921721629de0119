// General decode path: split-K flash-decoding over the compressed cache with plain
// CUDA-core arithmetic. It serves every supported shape and both storage types
// (fp32 caches, small head dims); the tensor-core kernel takes the bf16 production
// shapes.
//
// One CTA owns one (split, KV head, sequence). It walks its share of 64-token
// blocks (all blocks, or its slice of the selected-block list) in tiles of 32
// tokens. Per tile: rebuild keys k~ = A_tile . B_l^h ("LowRAM" project page,
// Figure 3), scores for the G query heads, the GELU branch g = GELU(k~ W1^T + b1)
// ("Predicting the value cache from keys", paragraph 3), then an online softmax
// that accumulates sum p k~, sum p g and sum p r over the residual rows of the tile
// (paragraph 2). The combine kernel merges splits and applies W_lin, W2 and b2 once
// per query head: o = (acc_k W_lin^T + acc_g W2^T + acc_r) / l + b2, which equals
// the per-token value rebuild because both maps are linear.
#include <math_constants.h>

#include "lr_common.cuh"
#include "lr_launch.h"
#include "general_front.cuh"

namespace lr {
namespace {

using namespace general;

template <typename T>
__global__ void __launch_bounds__(NT) decode_general_kernel(DecodeArgs a) {
  extern __shared__ float sm[];
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hd = a.hd, H = a.H, G = a.G, r = a.r, Hq = a.Hkv * a.G;
  const int W = 2 * hd + H;
  const SmemPlan sp = decode_smem_plan(hd, H, G);
  float* Ks = sm + sp.ks;
  float* Gs = sm + sp.gs;
  float* Ps = sm + sp.ps;
  float* acc = sm + sp.acc;
  float* qs = sm + sp.qs;
  float* m_run = sm + sp.stat;
  float* l_run = m_run + G;
  float* alpha = l_run + G;

  const size_t D = (size_t)a.L * a.Hkv * hd;
  const T* A = (const T*)a.A + (size_t)b * a.T * r;
  const T* Bl = (const T*)a.Bt + (size_t)b * D * r + (size_t)(a.layer * a.Hkv + h) * hd * r;
  const HeadPredictor<T> P = head_predictor<T>(a, b, a.layer, h);
  const size_t seg = ((size_t)b * a.L + a.layer) * a.Hkv + h;
  const int* ridx = a.k ? a.res_idx + seg * a.k : nullptr;
  const T* rval = a.k ? (const T*)a.res_val + seg * a.k * hd : nullptr;
  const int* rptr = (a.k && a.res_ptr) ? a.res_ptr + seg * (a.nblk + 1) : nullptr;
  const T* q = (const T*)a.q + ((size_t)b * Hq + h * G) * hd;

  for (int i = tid; i < G * hd; i += NT) qs[i] = to_f32(q[i]) * a.scale;
  for (int i = tid; i < G * W; i += NT) acc[i] = 0.f;
  if (tid < G) {
    m_run[tid] = -CUDART_INF_F;
    l_run[tid] = 0.f;
  }
  __syncthreads();

  const int n_units = a.blocks ? a.n_sel : a.nblk;
  const int u0 = (int)((long long)s * n_units / a.n_split);
  const int u1 = (int)((long long)(s + 1) * n_units / a.n_split);
  const int* blist = a.blocks ? a.blocks + ((size_t)b * a.Hkv + h) * a.n_sel : nullptr;

  for (int u = u0; u < u1; ++u) {
    int blk = u;
    if (blist) {
      blk = blist[u];
      const bool bad_range = blk < 0 || blk >= a.nblk;
      const bool bad_order = u > 0 && blist[u - 1] >= blk;
      if (bad_range || bad_order) {
        if (tid == 0) flag_error(a.err, (bad_range ? LR_DEVERR_BLOCK_RANGE : 0) | (bad_order ? LR_DEVERR_BLOCK_ORDER : 0));
        continue;
      }
    }
    int e0 = 0, e1 = 0;
    if (ridx) {
      if (rptr) {
        e0 = rptr[blk];
        e1 = rptr[blk + 1];
        if (e0 < 0 || e1 < e0 || e1 > a.k) {
          if (tid == 0) flag_error(a.err, LR_DEVERR_PTR);
          e0 = e1 = 0;
        }
      } else {
        e0 = lower_bound_i32(ridx, a.k, blk * kBlock);
        e1 = lower_bound_i32(ridx, a.k, blk * kBlock + kBlock);
      }
      if (tid == 0) {
        int bits = 0;
        for (int i = e0; i < e1; ++i) {
          const int t = ridx[i];
          if (t < blk * kBlock || t >= min(blk * kBlock + kBlock, a.T)) bits |= LR_DEVERR_RES_RANGE;
          if (i > e0 && ridx[i - 1] >= t) bits |= LR_DEVERR_RES_ORDER;
        }
        if (bits) flag_error(a.err, bits);
      }
    }
    for (int half = 0; half < kBlock / TT; ++half) {
      const int t0 = blk * kBlock + half * TT;
      const int nt = min(TT, a.T - t0);
      if (nt <= 0) break;
      tile_front<T>(A, r, t0, nt, Bl, hd, P, H, sm, sp);
      for (int x = tid; x < G * TT; x += NT) {
        const int g = x / TT, t = x % TT;
        float sc = -CUDART_INF_F;
        if (t < nt) {
          sc = 0.f;
          const float* kr = Ks + t * (hd + 1);
          const float* qr = qs + g * hd;
          for (int d = 0; d < hd; ++d) sc = fmaf(kr[d], qr[d], sc);
        }
        Ps[g * TT + t] = sc;
      }
      __syncthreads();
      if (warp < G) {
        const int g = warp;
        const float sc = Ps[g * TT + lane];
        const float m_new = fmaxf(m_run[g], warp_max(sc));
        const float al = __expf(m_run[g] - m_new);
        const float p = lane < nt ? __expf(sc - m_new) : 0.f;
        Ps[g * TT + lane] = p;
        const float psum = warp_sum(p);
        if (lane == 0) {
          l_run[g] = l_run[g] * al + psum;
          m_run[g] = m_new;
          alpha[g] = al;
        }
      }
      __syncthreads();
      for (int x = tid; x < G * W; x += NT) {
        const int g = x / W, e = x % W;
        const float* pg = Ps + g * TT;
        float v = acc[x] * alpha[g];
        if (e < hd) {
          for (int t = 0; t < nt; ++t) v = fmaf(pg[t], Ks[t * (hd + 1) + e], v);
        } else if (e < hd + H) {
          const int c = e - hd;
          for (int t = 0; t < nt; ++t) v = fmaf(pg[t], Gs[t * (H + 1) + c], v);
        } else {
          const int dd = e - hd - H;
          for (int i = e0; i < e1; ++i) {
            const int t = ridx[i] - t0;
            if (t >= 0 && t < nt) v = fmaf(pg[t], to_f32(rval[(size_t)i * hd + dd]), v);
          }
        }
        acc[x] = v;
      }
      __syncthreads();
    }
  }
  for (int x = tid; x < G * a.part_stride; x += NT) {
    const int g = x / a.part_stride, e = x % a.part_stride;
    float v = 0.f;
    if (e == 0) v = m_run[g];
    else if (e == 1) v = l_run[g];
    else if (e >= 4) v = acc[g * W + e - 4];
    a.partials[(((size_t)b * Hq + h * G + g) * a.n_split + s) * a.part_stride + e] = v;
  }
}

// Merge the split partials of the G query heads of one (sequence, KV head) and apply
// the linear maps once per query head: o = (acc_k W_lin^T + acc_g W2^T + acc_r) / l + b2.
// Partial sums are read coalesced (threads over entries); each output element is a
// warp-wide dot product over a contiguous weight row.
constexpr int CT = 512;  // combine threads

template <typename T>
__global__ void __launch_bounds__(CT) decode_combine_kernel(DecodeArgs a) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hd = a.hd, H = a.H, G = a.G, Hq = a.Hkv * a.G, S = a.n_split, W = 2 * hd + H;
  float* wsplit = sm;              // [G][S]
  float* accs = wsplit + G * S;    // [G][W]
  float* inv_l = accs + G * W;     // [G]
  float* mx = inv_l + G;           // [G]
  const float* part0 = a.partials + ((size_t)b * Hq + (size_t)h * G) * S * a.part_stride;
  // split maxima and weights, one warp per query head
  for (int g = warp; g < G; g += CT / 32) {
    const float* part = part0 + (size_t)g * S * a.part_stride;
    float m = -CUDART_INF_F;
    for (int s = lane; s < S; s += 32) m = fmaxf(m, part[(size_t)s * a.part_stride]);
    m = warp_max(m);
    float l = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float ms = part[(size_t)s * a.part_stride];
      const float wgt = (m == -CUDART_INF_F || ms == -CUDART_INF_F) ? 0.f : __expf(ms - m);
      wsplit[g * S + s] = wgt;
      l = fmaf(wgt, part[(size_t)s * a.part_stride + 1], l);
    }
    l = warp_sum(l);
    if (lane == 0) {
      mx[g] = m;
      inv_l[g] = l > 0.f ? 1.f / l : 0.f;
    }
  }
  __syncthreads();
  // weighted sums over the splits, 8 independent loads in flight per step
  for (int x = tid; x < G * W; x += CT) {
    const int g = x / W, e = x % W;
    const float* part = part0 + (size_t)g * S * a.part_stride + 4 + e;
    const float* wg = wsplit + g * S;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int s = 0;
    for (; s + 8 <= S; s += 8) {
      float t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) t[u] = part[(size_t)(s + u) * a.part_stride];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = fmaf(wg[s + u], t[u], v[u]);
    }
    for (; s < S; ++s) v[0] = fmaf(wg[s], part[(size_t)s * a.part_stride], v[0]);
    accs[x] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
  }
  __syncthreads();
  const HeadPredictor<T> P = head_predictor<T>(a, b, a.layer, h);
  T* o = (T*)a.o + ((size_t)b * Hq + (size_t)h * G) * hd;
  for (int j0 = warp; j0 < hd; j0 += 2 * (CT / 32)) {
    float wlv[2][8], w2v[2][16], bj[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = j0 + r * (CT / 32);
      const bool on = j < hd;
      const T* wl = P.W_lin + (size_t)(on ? j : 0) * hd;
      const T* w2 = P.W2 + (size_t)(on ? j : 0) * H;
#pragma unroll
      for (int q = 0; q < 8; ++q) wlv[r][q] = (on && lane + 32 * q < hd) ? to_f32(wl[lane + 32 * q]) : 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) w2v[r][q] = (on && lane + 32 * q < H) ? to_f32(w2[lane + 32 * q]) : 0.f;
      bj[r] = (on && P.b2) ? to_f32(P.b2[j]) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = j0 + r * (CT / 32);
      if (j >= hd) continue;
      for (int g = 0; g < G; ++g) {
        const float* ac = accs + g * W;
        float y = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (lane + 32 * q < hd) y = fmaf(ac[lane + 32 * q], wlv[r][q], y);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (lane + 32 * q < H) y = fmaf(ac[hd + lane + 32 * q], w2v[r][q], y);
        y = warp_sum(y);
        if (lane == 0) {
          const float out = mx[g] == -CUDART_INF_F ? 0.f : (y + ac[hd + H + j]) * inv_l[g] + bj[r];
          o[(size_t)g * hd + j] = from_f32<T>(out);
        }
      }
    }
  }
}

}  // namespace

size_t decode_general_smem_bytes(int hd, int H, int G) {
  return (size_t)decode_smem_plan(hd, H, G).total * sizeof(float);
}

size_t decode_combine_smem_bytes(int hd, int H, int G, int n_split) {
  return (size_t)(G * n_split + G * (2 * hd + H) + 2 * G) * sizeof(float);
}

cudaError_t launch_decode_general(const DecodeArgs& a, lr_dtype dt, cudaStream_t st) {
  const size_t smem = decode_general_smem_bytes(a.hd, a.H, a.G);
  dim3 grid(a.n_split, a.Hkv, a.B);
  cudaError_t e;
  if (dt == LR_BF16) {
    e = cudaFuncSetAttribute(decode_general_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_general_kernel<__nv_bfloat16><<<grid, NT, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(decode_general_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_general_kernel<float><<<grid, NT, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const DecodeArgs& a, lr_dtype dt, cudaStream_t st) {
  const size_t smem = decode_combine_smem_bytes(a.hd, a.H, a.G, a.n_split);
  dim3 grid(a.Hkv, a.B);
  cudaError_t e;
  if (dt == LR_BF16) {
    e = cudaFuncSetAttribute(decode_combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_combine_kernel<__nv_bfloat16><<<grid, CT, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(decode_combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_combine_kernel<float><<<grid, CT, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace lr
