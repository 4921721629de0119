// Test-time fitting of the value predictor on the GPU ("Predicting the value cache from
// keys", paragraph on prefill cost: the per-head network is fitted to each context with
// gradient steps; arXiv abstract: the predictor is fitted at test time).
//
// One step of full-batch gradient descent on the mean squared value error
//   L = mean_{t, j} (v_hat_t[j] - v_t[j])^2,   v_hat = k~ W_lin^T + GELU(k~ W1^T + b1) W2^T + b2,
// over the context's own rebuilt keys k~ (K~ = A . Bt^T, computed once) and values v:
//   1. forward (pack_predict_tc_kernel in fitting mode): R = v_hat - v, g = GELU(u) and
//      dU' = (R W2) * GELU'(u) per token, stored fp16;
//   2. gradients (fit_grad_kernel below), contractions over the tokens on the tensor cores:
//        dW_lin = R^T k~,  db2 = R^T 1      (one MMA with B = [k~ | 1])
//        dW2    = R^T g
//        dW1    = dU'^T k~, db1 = dU'^T 1   (per 128 hidden units)
//      each split over token ranges and added into fp32 gradient sums;
//   3. update (fit_update_kernel): theta -= lr * (2 / N) * sum, N = tokens x head_dim of the
//      loss, and fresh fp16 copies of W1, W_lin, W2 for the next forward.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lr_common.cuh"
#include "lr_fit.h"
#include "lr_gemm.h"
#include "sm100.cuh"

namespace lr {
namespace tc {
namespace {

using namespace sm100;

constexpr int kThreads = 192;       // warp 0 loads, warp 1 MMAs, warps 2-5 epilogue
constexpr int kStageBytes = 49152;  // A 16 KB + B up to 32 KB
constexpr int kStages = 4;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kOffMisc = kOffBar + 128;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum FBar { F_FULL0 = 0, F_EMPTY0 = kStages, F_TFULL0 = 2 * kStages, F_TEMPTY0 = 2 * kStages + 2,
            F_DRAIN = 2 * kStages + 4, N_FBARS };
static_assert(N_FBARS * 8 <= 128, "barrier area");

// Work item: (segment, kind, token split). kind 0: R^T [k~ | 1]; kind 1: R^T g;
// kind 2 + hf: dU'_hf^T [k~ | 1] for hidden units 128 hf .. 128 hf + 127.
struct GItem {
  int seg, kind, split, b, l, h, wh;
};

__device__ __forceinline__ GItem gitem(const FitGradArgs& a, int it) {
  const int nk = 2 + a.H / 128;
  GItem x;
  x.split = it % a.S;
  x.kind = (it / a.S) % nk;
  x.seg = it / (a.S * nk);
  x.h = x.seg % a.Hkv;
  x.l = (x.seg / a.Hkv) % a.L;
  x.b = x.seg / (a.Hkv * a.L);
  x.wh = ((a.pred_per_seq ? x.b : 0) * a.L + x.l) * a.Hkv + x.h;
  return x;
}

__device__ __forceinline__ int gitem_n(const FitGradArgs& a, int kind) { return kind == 1 ? a.H : 144; }

__global__ void __launch_bounds__(kThreads, 1)
fit_grad_kernel(const __grid_constant__ CUtensorMap mapR, const __grid_constant__ CUtensorMap mapDU,
                const __grid_constant__ CUtensorMap mapG, const __grid_constant__ CUtensorMap mapKt,
                const __grid_constant__ CUtensorMap mapOnes, const FitGradArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {
    if (threadIdx.x == 0) flag_error(a.errword, LR_DEVERR_LAUNCH);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkind = 2 + a.H / 128;
  const int n_items = a.B * a.L * a.Hkv * nkind * a.S;
  const int nkc = (a.T + 63) / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[F_FULL0 + i], 1);
      mbar_init(&bars[F_EMPTY0 + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[F_TFULL0 + i], 1);
      mbar_init(&bars[F_TEMPTY0 + i], 4);
    }
    mbar_init(&bars[F_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapR);
    tma_prefetch_desc(&mapDU);
    tma_prefetch_desc(&mapG);
    tma_prefetch_desc(&mapKt);
    tma_prefetch_desc(&mapOnes);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      uint32_t it_k = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const GItem x = gitem(a, it);
        const int c0 = x.split * nkc / a.S, c1 = (x.split + 1) * nkc / a.S;
        const int n = gitem_n(a, x.kind);
        const uint32_t bytes = 16384u + (uint32_t)((n + 63) / 64) * 8192u;
        const int kcol = (x.l * a.Hkv + x.h) * 128;
        for (int c = c0; c < c1 && ok; ++c, ++it_k) {
          const uint32_t st = it_k % kStages, ph = (it_k / kStages) & 1;
          if (!(ok = mbar_wait(&bars[F_EMPTY0 + st], ph ^ 1, abort_flag))) break;
          uint8_t* dst = sm + st * kStageBytes;
          uint64_t* full = &bars[F_FULL0 + st];
          mbar_arrive_expect_tx(full, bytes);
          const int t0 = c * 64;
          // A operand (MN-major): 128 rows of the gradient (j or hidden units) x 64 tokens
          for (int i = 0; i < 2; ++i) {
            if (x.kind <= 1) tma_load_3d(dst + i * 8192, &mapR, full, 64 * i, t0, x.seg);
            else tma_load_3d(dst + i * 8192, &mapDU, full, 128 * (x.kind - 2) + 64 * i, t0, x.seg);
          }
          uint8_t* bdst = dst + 16384;
          if (x.kind == 1) {
            for (int i = 0; i < a.H / 64; ++i) tma_load_3d(bdst + i * 8192, &mapG, full, 64 * i, t0, x.seg);
          } else {
            tma_load_3d(bdst, &mapKt, full, kcol, t0, x.b);
            tma_load_3d(bdst + 8192, &mapKt, full, kcol + 64, t0, x.b);
            tma_load_2d(bdst + 16384, &mapOnes, full, 0, 0);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(a.errword, LR_DEVERR_TIMEOUT);
      }
      for (uint32_t j = it_k > (uint32_t)kStages ? it_k - kStages : 0; j < it_k; ++j)
        mbar_wait_drain(&bars[F_FULL0 + j % kStages], (j / kStages) & 1, kWaitCycles / 4);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMAs
    if (lane == 0) {
      uint32_t it_k = 0;
      bool ok = true;
      int i = 0;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++i) {
        const GItem x = gitem(a, it);
        const int c0 = x.split * nkc / a.S, c1 = (x.split + 1) * nkc / a.S;
        const uint32_t idesc = idesc_f16_f32(128, gitem_n(a, x.kind), true, true);
        const int buf = i & 1;
        if (i >= 2 && !(ok = mbar_wait(&bars[F_TEMPTY0 + buf], ((i >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t d = tmem + 256 * buf;
        for (int c = c0; c < c1 && ok; ++c, ++it_k) {
          const uint32_t st = it_k % kStages, ph = (it_k / kStages) & 1;
          if (!(ok = mbar_wait(&bars[F_FULL0 + st], ph, abort_flag))) break;
          tc_fence_after();
          const uint32_t base = smem_u32(sm + st * kStageBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16_ss(d, sw128_desc(base + ks * 2048, 8192, 1024), sw128_desc(base + 16384 + ks * 2048, 8192, 1024),
                       idesc, (c > c0 || ks > 0) ? 1u : 0u);
          mma_commit(&bars[F_EMPTY0 + st]);
        }
        if (!ok) break;
        // every split holds at least one 64-token chunk (the host keeps S <= ceil(T / 64)),
        // so the accumulator was written by this item
        mma_commit(&bars[F_TFULL0 + buf]);
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(a.errword, LR_DEVERR_TIMEOUT);
      }
      mma_commit(&bars[F_DRAIN]);
      mbar_wait_drain(&bars[F_DRAIN], 0, kWaitCycles / 4);
    }
  } else {
    // ---------------------------------------------------------------- epilogue: add into the sums
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    int i = 0;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++i) {
      const GItem x = gitem(a, it);
      const int buf = i & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[F_TFULL0 + buf], (i >> 1) & 1, abort_flag)))) break;
      tc_fence_after();
      float* gw = a.grad + (size_t)x.wh * a.gstride;
      const int H = a.H;
      float* dst;       // this row of the weight gradient
      float* dst_bias;  // this row's bias gradient, or null
      int ncols;
      if (x.kind == 0) {
        dst = gw + (size_t)row * 128;                                      // dW_lin [128, 128]
        dst_bias = gw + 128 * 128 + 2 * (size_t)H * 128 + H + row;         // db2 [128]
        ncols = 128;
      } else if (x.kind == 1) {
        dst = gw + 128 * 128 + (size_t)H * 128 + (size_t)row * H;          // dW2 [128, H]
        dst_bias = nullptr;
        ncols = H;
      } else {
        const int c = 128 * (x.kind - 2) + row;
        dst = gw + 128 * 128 + (size_t)c * 128;                            // dW1 [H, 128]
        dst_bias = gw + 128 * 128 + 2 * (size_t)H * 128 + c;               // db1 [H]
        ncols = 128;
      }
      const uint32_t col = trow + 256 * buf;
      for (int c0 = 0; c0 < ncols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(col + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          atomicAdd(reinterpret_cast<float4*>(dst + c0) + j,
                    make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
      }
      if (dst_bias) {
        uint32_t v[8];
        tmem_ld8(col + 128, v);
        tmem_ld_wait();
        atomicAdd(dst_bias, __uint_as_float(v[0]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[F_TEMPTY0 + buf]);
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(a.errword, LR_DEVERR_TIMEOUT);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// theta -= lr * scale * sum for every parameter of every weight head; the sums are cleared and
// the fp16 copies of W1, W_lin, W2 refreshed (update = 0 with lr = 0: only the copies and the
// clearing, used before the first step). One grid row per weight head (blockIdx.y), so each
// thread's position within the head's parameters needs no division. Each thread takes
// kUpdPer parameters of its weight head, strided by the block, and loads
// all their gradient sums and fp32 masters before it stores anything (a grid of one CTA per
// 256 parameters left every warp waiting on one load at a time).
constexpr int kUpdPer = 8;

struct UpdTarget {
  float* w;
  __half* wh16;
  void* out;
  size_t o;
};

__device__ __forceinline__ UpdTarget upd_target(const FitUpdateArgs& a, size_t wh, int e) {
  const int H = a.H, n_wl = 128 * 128, n_w1 = H * 128, n_w2 = 128 * H;
  if (e < n_wl) return {a.W_lin, a.Wlh, a.out_Wl, wh * n_wl + e};
  if (e < n_wl + n_w1) return {a.W1, a.W1h, a.out_W1, wh * n_w1 + (e - n_wl)};
  if (e < n_wl + n_w1 + n_w2) return {a.W2, a.W2h, a.out_W2, wh * n_w2 + (e - n_wl - n_w1)};
  if (e < n_wl + n_w1 + n_w2 + H) return {a.b1, nullptr, a.out_b1, wh * H + (e - n_wl - n_w1 - n_w2)};
  return {a.b2, nullptr, a.out_b2, wh * 128 + (e - n_wl - n_w1 - n_w2 - H)};  // b2 may be null
}

__global__ void __launch_bounds__(256) fit_update_kernel(FitUpdateArgs a) {
  const size_t wh = blockIdx.y;
  float* g = a.grad + wh * (size_t)a.gstride;
  const int e0 = blockIdx.x * (256 * kUpdPer) + threadIdx.x;
  float gv[kUpdPer], wv[kUpdPer];
#pragma unroll
  for (int u = 0; u < kUpdPer; ++u) {
    const int e = e0 + 256 * u;
    gv[u] = wv[u] = 0.f;
    if (e < a.gstride) {
      const UpdTarget t = upd_target(a, wh, e);
      gv[u] = g[e];
      if (t.w) wv[u] = t.w[t.o];
    }
  }
#pragma unroll
  for (int u = 0; u < kUpdPer; ++u) {
    const int e = e0 + 256 * u;
    if (e >= a.gstride) break;
    g[e] = 0.f;
    const UpdTarget t = upd_target(a, wh, e);
    if (!t.w) continue;
    const float v = wv[u] - a.lr * a.scale * gv[u];
    t.w[t.o] = v;
    if (t.wh16) t.wh16[t.o] = __float2half_rn(v);
    if (t.out) store_dtype(t.out, t.o, v, a.out_bf16);
  }
}

// The [64 tokens, 64 columns] fp16 tile whose first column is 1: the B operand columns that
// turn the token sums of R and dU' into the bias gradients.
__global__ void fit_ones_kernel(__half* ones) {
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) ones[i] = __float2half_rn((i % 64) == 0 ? 1.f : 0.f);
}

}  // namespace

cudaError_t launch_fit_grad(const FitGradArgs& a, const CUtensorMap& mR, const CUtensorMap& mDU, const CUtensorMap& mG,
                            const CUtensorMap& mKt, const CUtensorMap& mOnes, cudaStream_t st) {
  const long long n_items = (long long)a.B * a.L * a.Hkv * (2 + a.H / 128) * a.S;
  if (n_items == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(n_items < sms ? n_items : sms);
  cudaError_t e = cudaFuncSetAttribute(fit_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  fit_grad_kernel<<<grid, kThreads, kSmemBytes, st>>>(mR, mDU, mG, mKt, mOnes, a);
  return cudaGetLastError();
}

cudaError_t launch_fit_update(const FitUpdateArgs& a, cudaStream_t st) {
  if (a.n_heads == 0) return cudaSuccess;
  fit_update_kernel<<<dim3((a.gstride + 256 * kUpdPer - 1) / (256 * kUpdPer), a.n_heads), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fit_ones(void* ones, cudaStream_t st) {
  fit_ones_kernel<<<1, 256, 0, st>>>((__half*)ones);
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace lr
