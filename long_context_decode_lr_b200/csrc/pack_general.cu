// General packer path (CUDA cores; every supported shape, fp32 or bf16 storage).
//
//   project : A = round(K_group . Bt)                 ("LowRAM" project page, Figure 3)
//   predict : per (layer, KV head, 32-token tile): k~ = A . B_l^h, v_hat = f_theta(k~),
//             e_t = ||v_t - v_hat_t||^2 (fp32) and d_t = round(v_t - v_hat_t)
//             ("Predicting the value cache from keys", paragraphs 2-4)
//   gather  : res_val[i] = d[res_idx[i]] once the top-k step has chosen the tokens.
#include "general_front.cuh"
#include "lr_common.cuh"
#include "lr_launch.h"

namespace lr {
namespace {

using namespace general;

constexpr int PT = 64;   // projection tile (tokens and basis columns)
constexpr int PK = 16;   // projection reduction chunk

template <typename T>
__global__ void __launch_bounds__(256) pack_project_general_kernel(PackArgs a) {
  __shared__ float As[PK][PT + 4];
  __shared__ float Bs[PK][PT + 4];
  const int j0 = blockIdx.x * PT, t0 = blockIdx.y * PT, b = blockIdx.z;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const T* K = (const T*)a.K + (size_t)b * a.T * a.D;
  const T* Bt = (const T*)a.Bt + (size_t)b * a.D * a.r;
  float acc[4][4] = {};
  for (int d0 = 0; d0 < a.D; d0 += PK) {
    for (int x = tid; x < PK * PT; x += 256) {
      const int t = x / PK, kk = x % PK;
      As[kk][t] = (t0 + t < a.T && d0 + kk < a.D) ? to_f32(K[(size_t)(t0 + t) * a.D + d0 + kk]) : 0.f;
      const int kk2 = x / PT, j = x % PT;
      Bs[kk2][j] = (j0 + j < a.r && d0 + kk2 < a.D) ? to_f32(Bt[(size_t)(d0 + kk2) * a.r + j0 + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < PK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) bv[i] = Bs[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  T* A = (T*)a.A + (size_t)b * a.T * a.r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= a.T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = j0 + tx * 4 + j;
      if (c < a.r) A[(size_t)t * a.r + c] = from_f32<T>(acc[i][j]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(NT) pack_predict_general_kernel(PackArgs a) {
  extern __shared__ float sm[];
  const int t0 = blockIdx.x * TT, lh = blockIdx.y, b = blockIdx.z;
  const int l = lh / a.Hkv, h = lh % a.Hkv;
  const int nt = min(TT, a.T - t0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hd = a.hd, H = a.H, r = a.r;
  const SmemPlan sp = decode_smem_plan(hd, H, 1);
  float* Bs = sm + sp.bs;
  float* Ks = sm + sp.ks;
  float* Gs = sm + sp.gs;
  const T* A = (const T*)a.A + (size_t)b * a.T * r;
  const T* Bl = (const T*)a.Bt + (size_t)b * a.D * r + (size_t)(l * a.Hkv + h) * hd * r;
  const HeadPredictor<T> P = head_predictor<T>(a, b, l, h);
  tile_front<T>(A, r, t0, nt, Bl, hd, P, H, sm, sp);

  const int n_out = TT * hd / NT;
  float vacc[kMaxOutK];
#pragma unroll
  for (int i = 0; i < kMaxOutK; ++i) vacc[i] = 0.f;
  for (int i0 = 0; i0 < hd; i0 += KC) {  // k~ W_lin^T
    const int n = min(KC, hd - i0);
    for (int x = tid; x < hd * KC; x += NT) {
      const int j = x / KC, jj = x % KC;
      Bs[j * (KC + 1) + jj] = jj < n ? to_f32(P.W_lin[(size_t)j * hd + i0 + jj]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxOutK; ++i) {
      if (i < n_out) {
        const int o = tid + NT * i, t = o / hd, j = o % hd;
        const float* kr = Ks + t * (hd + 1) + i0;
        const float* wr = Bs + j * (KC + 1);
        float s = vacc[i];
        for (int jj = 0; jj < n; ++jj) s = fmaf(kr[jj], wr[jj], s);
        vacc[i] = s;
      }
    }
    __syncthreads();
  }
  for (int c0 = 0; c0 < H; c0 += KC) {  // GELU(.) W2^T
    const int n = min(KC, H - c0);
    for (int x = tid; x < hd * KC; x += NT) {
      const int j = x / KC, jj = x % KC;
      Bs[j * (KC + 1) + jj] = jj < n ? to_f32(P.W2[(size_t)j * H + c0 + jj]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxOutK; ++i) {
      if (i < n_out) {
        const int o = tid + NT * i, t = o / hd, j = o % hd;
        const float* gr = Gs + t * (H + 1) + c0;
        const float* wr = Bs + j * (KC + 1);
        float s = vacc[i];
        for (int jj = 0; jj < n; ++jj) s = fmaf(gr[jj], wr[jj], s);
        vacc[i] = s;
      }
    }
    __syncthreads();
  }
  const size_t seg = ((size_t)b * a.L + l) * a.Hkv + h;
  const T* V = (const T*)a.V + ((size_t)(b * a.L + l) * a.T) * a.Hkv * hd;
#pragma unroll
  for (int i = 0; i < kMaxOutK; ++i) {
    if (i < n_out) {
      const int o = tid + NT * i, t = o / hd, j = o % hd;
      float d = 0.f;
      if (t < nt) {
        const float vh = vacc[i] + (P.b2 ? to_f32(P.b2[j]) : 0.f);
        d = to_f32(V[((size_t)(t0 + t) * a.Hkv + h) * hd + j]) - vh;
      }
      Ks[t * (hd + 1) + j] = d;
    }
  }
  __syncthreads();
  for (int t = warp; t < nt; t += NT / 32) {
    float s = 0.f;
    for (int j = lane; j < hd; j += 32) {
      const float d = Ks[t * (hd + 1) + j];
      s = fmaf(d, d, s);
    }
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) a.err[seg * a.T + t0 + t] = s;
  }
  T* dout = (T*)a.diff + (seg * a.T + t0) * hd;
  for (int x = tid; x < nt * hd; x += NT) dout[x] = from_f32<T>(Ks[(x / hd) * (hd + 1) + (x % hd)]);
}

template <typename T>
__global__ void __launch_bounds__(256) pack_gather_kernel(PackArgs a) {
  const int seg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  if (i >= a.k) return;
  const int t = a.res_idx[(size_t)seg * a.k + i];
  const T* src = (const T*)a.diff + ((size_t)seg * a.T + t) * a.hd;
  T* dst = (T*)a.res_val + ((size_t)seg * a.k + i) * a.hd;
  for (int j = lane; j < a.hd; j += 32) dst[j] = src[j];
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t smem) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

}  // namespace

cudaError_t launch_pack_project_general(const PackArgs& a, lr_dtype dt, cudaStream_t st) {
  dim3 grid(ceil_div(a.r, PT), ceil_div(a.T, PT), a.B);
  if (dt == LR_BF16) pack_project_general_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else pack_project_general_kernel<float><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_pack_predict_general(const PackArgs& a, lr_dtype dt, cudaStream_t st) {
  const size_t smem = (size_t)decode_smem_plan(a.hd, a.H, 1).total * sizeof(float);
  dim3 grid(ceil_div(a.T, TT), a.L * a.Hkv, a.B);
  cudaError_t e;
  if (dt == LR_BF16) {
    if ((e = set_smem(pack_predict_general_kernel<__nv_bfloat16>, smem)) != cudaSuccess) return e;
    pack_predict_general_kernel<__nv_bfloat16><<<grid, NT, smem, st>>>(a);
  } else {
    if ((e = set_smem(pack_predict_general_kernel<float>, smem)) != cudaSuccess) return e;
    pack_predict_general_kernel<float><<<grid, NT, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_pack_gather(const PackArgs& a, lr_dtype dt, cudaStream_t st) {
  if (a.k == 0) return cudaSuccess;
  dim3 grid(ceil_div(a.k, 8), a.B * a.L * a.Hkv);
  if (dt == LR_BF16) pack_gather_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else pack_gather_kernel<float><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace lr
