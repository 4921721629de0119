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
  const size_t seg_row = seg * a.k;
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
            if (t >= 0 && t < nt) v = fmaf(pg[t], residual_entry<T>(a, seg_row, i, dd), v);
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

// Merge the split partials of one query head and apply the linear maps once:
// o = (acc_k W_lin^T + acc_g W2^T + acc_r + l_c b2 + sum_tail w_t v_t) / (l_c + l_tail),
// where the exact tail tokens (newly generated, stored exactly) join the softmax here with
// their own keys and values, all weights taken relative to one maximum over the splits
// and the tail; without a tail this is (acc_k W_lin^T + acc_g W2^T + acc_r) / l + b2.
// One block per (chunk of CJ output
// columns, query head, sequence), so that even a single sequence spreads over many SMs;
// every block of a head re-merges acc_k and acc_g (hd + H floats per split, read from
// L2) and only its own CJ columns of acc_r. The kernel may start while the split kernel
// drains (programmatic dependent launch): it stages its weight rows in shared memory
// first, then waits for the split kernel before the first partial is read. The merge
// runs over (entry, split chunk) items so that each thread keeps eight loads in flight,
// and the chunk sums are added in a fixed order.
constexpr int CT = 512;      // combine threads
constexpr int CJ = 32;       // output columns per combine block
constexpr int kMaxChunk = 8; // split chunks per merged entry

struct CombineSmem {
  int n_ch, cs, n_acc, w_floats;
  int off_ml, off_w, off_red, off_acc, off_tail, off_q, off_tred, total;  // in floats
};

__host__ __device__ inline CombineSmem combine_smem(int hd, int H, int S, int elem_bytes, int n_tail) {
  CombineSmem c;
  c.n_ch = ceil_div(S, 8) < kMaxChunk ? ceil_div(S, 8) : kMaxChunk;
  c.cs = ceil_div(S, c.n_ch);
  c.n_acc = hd + H + CJ;
  c.w_floats = ceil_div(CJ * (hd + H) * elem_bytes, 16) * 4;  // weight rows, 16-byte padded
  c.off_w = 0;
  c.off_ml = c.w_floats;
  c.off_red = c.off_ml + 2 * S;
  c.off_acc = c.off_red + c.n_ch * c.n_acc;
  c.off_tail = c.off_acc + c.n_acc;                    // [n_tail] tail scores, then weights
  c.off_q = c.off_tail + n_tail;                       // [hd] the query
  c.off_tred = c.off_q + (n_tail ? hd : 0);            // [warps][CJ] tail value sums
  c.total = c.off_tred + (n_tail ? (CT / 32) * CJ : 0);
  return c;
}

template <typename T>
__global__ void __launch_bounds__(CT) decode_combine_kernel(DecodeArgs a) {
  extern __shared__ float sm[];
  __shared__ float s_lc, s_lt, s_b2[CJ];
  const int jc = blockIdx.x, qh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hd = a.hd, H = a.H, Hq = a.Hkv * a.G, S = a.n_split, nt = a.n_tail;
  const int j0 = jc * CJ, nj = min(CJ, hd - j0);
  const CombineSmem L = combine_smem(hd, H, S, (int)sizeof(T), nt);
  T* wl_s = reinterpret_cast<T*>(sm + L.off_w);  // [nj][hd]
  T* w2_s = wl_s + CJ * hd;                      // [nj][H]
  float* mls = sm + L.off_ml;                    // [S] maxima, then [S] sums
  float* red = sm + L.off_red;                   // [n_ch][n_acc]
  float* acc = sm + L.off_acc;                   // [hd + H + nj]: merged sum p k~, sum p g, own columns of sum p r
  float* ts = sm + L.off_tail;                   // [nt] exact tail tokens: scores, then softmax weights
  float* tred = sm + L.off_tred;                 // [warps][CJ] tail value sums per warp

  // weight rows are inputs of the call, independent of the split kernel
  const HeadPredictor<T> P = head_predictor<T>(a, b, a.layer, qh / a.G);
  for (int i = tid; i < nj * hd; i += CT) wl_s[i] = P.W_lin[(size_t)j0 * hd + i];
  for (int i = tid; i < nj * H; i += CT) w2_s[i] = P.W2[(size_t)j0 * H + i];
  if (tid < nj) s_b2[tid] = P.b2 ? to_f32(P.b2[j0 + tid]) : 0.f;
  // scores of the exact tail tokens (inputs of the call as well): scale q . key_t
  const int h = qh / a.G;
  if (nt > 0) {
    float* qv = sm + L.off_q;
    const T* qp = (const T*)a.q + ((size_t)b * Hq + qh) * hd;
    for (int d = tid; d < hd; d += CT) qv[d] = to_f32(qp[d]);
    __syncthreads();
    // one warp per tail token, lanes across the key's dims (coalesced rows), four tokens
    // of a warp in flight at once
    const T* kt = (const T*)a.tail_K + ((size_t)b * a.Hkv + h) * nt * hd;
    for (int t0 = warp; t0 < nt; t0 += 4 * (CT / 32)) {
      float sv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * (CT / 32);
        float acc_d = 0.f;
        if (t < nt) {
          const T* kr = kt + (size_t)t * hd;
          for (int d = lane; d < hd; d += 32) acc_d = fmaf(qv[d], to_f32(kr[d]), acc_d);
        }
        sv[u] = acc_d;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * (CT / 32);
        const float v = warp_sum(sv[u]);
        if (lane == 0 && t < nt) ts[t] = v * a.scale;
      }
    }
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* part = a.partials + ((size_t)b * Hq + qh) * S * a.part_stride;
  for (int s = tid; s < S; s += CT) {
    mls[s] = part[(size_t)s * a.part_stride];
    mls[S + s] = part[(size_t)s * a.part_stride + 1];
  }
  __syncthreads();
  if (warp == 0) {  // one max over the splits and the tail; weights relative to it
    float m = -CUDART_INF_F;
    for (int s = lane; s < S; s += 32) m = fmaxf(m, mls[s]);
    for (int t = lane; t < nt; t += 32) m = fmaxf(m, ts[t]);
    m = warp_max(m);
    float lc = 0.f, lt = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float ms = mls[s];
      const float wgt = (m == -CUDART_INF_F || ms == -CUDART_INF_F) ? 0.f : __expf(ms - m);
      mls[s] = wgt;
      lc = fmaf(wgt, mls[S + s], lc);
    }
    for (int t = lane; t < nt; t += 32) {
      const float wgt = m == -CUDART_INF_F ? 0.f : __expf(ts[t] - m);
      ts[t] = wgt;
      lt += wgt;
    }
    lc = warp_sum(lc);
    lt = warp_sum(lt);
    if (lane == 0) {
      s_lc = lc;
      s_lt = lt;
    }
  }
  __syncthreads();
  if (nt > 0) {  // tail values weighted by their softmax weights, this block's columns
    const T* vt = (const T*)a.tail_V + ((size_t)b * a.Hkv + h) * nt * hd + j0;
    float av[4] = {0.f, 0.f, 0.f, 0.f};
    if (lane < nj) {
      int t = warp;
      for (; t + 3 * (CT / 32) < nt; t += 4 * (CT / 32)) {
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = to_f32(vt[(size_t)(t + u * (CT / 32)) * hd + lane]);
#pragma unroll
        for (int u = 0; u < 4; ++u) av[u] = fmaf(ts[t + u * (CT / 32)], x[u], av[u]);
      }
      for (; t < nt; t += CT / 32) av[0] = fmaf(ts[t], to_f32(vt[(size_t)t * hd + lane]), av[0]);
    }
    tred[warp * CJ + lane] = (av[0] + av[1]) + (av[2] + av[3]);
  }
  const int n_acc = hd + H + nj;
  for (int it = tid; it < L.n_ch * n_acc; it += CT) {
    const int c = it / n_acc, x = it % n_acc;
    const int e = x < hd + H ? x : x + j0;
    const int s0 = c * L.cs, s1 = min(S, s0 + L.cs);
    const float* pe = part + 4 + e;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int s = s0;
    for (; s + 8 <= s1; s += 8) {
      float t[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) t[u] = pe[(size_t)(s + u) * a.part_stride];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = fmaf(mls[s + u], t[u], v[u]);
    }
    for (; s < s1; ++s) v[0] = fmaf(mls[s], pe[(size_t)s * a.part_stride], v[0]);
    red[c * L.n_acc + x] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
  }
  __syncthreads();
  for (int x = tid; x < n_acc; x += CT) {
    float v = 0.f;
    for (int c = 0; c < L.n_ch; ++c) v += red[c * L.n_acc + x];
    acc[x] = v;
  }
  __syncthreads();
  T* o = (T*)a.o + ((size_t)b * Hq + qh) * hd;
  const float lc = s_lc, lsum = s_lc + s_lt;
  for (int jj = warp; jj < nj; jj += CT / 32) {
    const T* wl = wl_s + jj * hd;
    const T* w2 = w2_s + jj * H;
    float y0 = 0.f, y1 = 0.f;
    for (int c = lane; c < hd; c += 32) y0 = fmaf(acc[c], to_f32(wl[c]), y0);
    for (int c = lane; c < H; c += 32) y1 = fmaf(acc[hd + c], to_f32(w2[c]), y1);
    const float y = warp_sum(y0 + y1);
    if (lane == 0) {
      float tv = 0.f;
      for (int w = 0; w < (nt > 0 ? CT / 32 : 0); ++w) tv += tred[w * CJ + jj];
      const float out = lsum > 0.f ? (y + acc[hd + H + jj] + lc * s_b2[jj] + tv) / lsum : 0.f;
      o[j0 + jj] = from_f32<T>(out);
    }
  }
}

}  // namespace

size_t decode_general_smem_bytes(int hd, int H, int G) {
  return (size_t)decode_smem_plan(hd, H, G).total * sizeof(float);
}

size_t decode_combine_smem_bytes(int hd, int H, int G, int n_split, int elem_bytes, int n_tail) {
  (void)G;
  return (size_t)combine_smem(hd, H, n_split, elem_bytes, n_tail).total * sizeof(float);
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
  const size_t smem = decode_combine_smem_bytes(a.hd, a.H, a.G, a.n_split, dt == LR_BF16 ? 2 : 4, a.n_tail);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(ceil_div(a.hd, CJ), a.Hkv * a.G, a.B);
  cfg.blockDim = dim3(CT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (dt == LR_BF16) {
    e = cudaFuncSetAttribute(decode_combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<__nv_bfloat16>, a);
  } else {
    e = cudaFuncSetAttribute(decode_combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<float>, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lr
