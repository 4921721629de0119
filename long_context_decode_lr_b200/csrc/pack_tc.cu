// Tensor-core predictor of the packer (bf16 cache, head_dim 128, hidden 128 or 256, sm_100a).
//
// For one (sequence b, layer l, KV head h) segment and 128 rebuilt keys k~ at a time (read
// from the K~ = A . Bt^T buffer that the CTA-pair GEMM wrote), the kernel evaluates the
// value predictor ("Predicting the value cache from keys", paragraphs 2-3):
//   MMA2   U      = k~ W1^T                    (M 128, N H, K 128)
//   MMA3a  v_hat  = k~ W_lin^T                 (M 128, N 128, K 128)
//   GELU   g      = GELU(U + b1)               (epilogue warps, fp16 into shared memory)
//   MMA3b  v_hat += g W2^T                     (M 128, N 128, K H, one 128-unit half at a time)
// and then, per row, d = v - (v_hat + b2):
//   normal mode: the per-token error err[seg, t] = sum_j d_j^2 (paragraph 4: tokens are ranked
//                by this error), for every token of the context;
//   gather mode: the residual row res_val[seg, i] = round(d) of the tokens t = res_idx[seg, i]
//                that the top-k step kept, recomputed for those rows only;
//   fit mode:    the pieces of one gradient step of test-time fitting (explainer, paragraph on
//                prefill cost): R = v_hat - v, g = GELU(u) and, after one more MMA per
//                128-unit half, MMA4 dG = R W2_half (M 128, N 128, K 128; W2 read MN-major from
//                the same tile, into TMEM columns 384-511), dU' = dG * GELU'(u) with u read
//                again from TMEM; R, g and dU' are stored (fp16) for the gradient contractions.
// Operands are fp16 with fp32 accumulation; GELU is the tanh form fitted to x Phi(x) (within
// 2.71e-4). A CTA owns a contiguous range of (segment, tile) items; the segment's weights
// (W1, W_lin, W2 as fp16, 160 KB at H = 256) stay in shared memory while its tiles stream.
// Warp 0 loads (TMA for whole tiles, plain loads for gathered rows), warp 1 issues the MMAs,
// warps 2-17 are the epilogue (four per TMEM lane quarter, each on a quarter of the columns
// of every 128-column half: with eighteen warps a thread keeps at most 104 registers). The k~
// buffer is released as soon as MMA2 and MMA3a have read it, so the next tile's keys load
// while this tile's GELU halves (one after the other through one fp16 buffer), MMA3b and
// error run; each epilogue thread starts its value-row loads before it waits for v_hat.
// Every wait is bounded; a timeout raises the abort flag and sets LR_DEVERR_TIMEOUT.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lr_common.cuh"
#include "lr_gemm.h"
#include "sm100.cuh"

namespace lr {
namespace tc {
namespace {

using namespace sm100;

constexpr int kEpiWarps = 16;                // four per TMEM lane quarter, 32 columns each
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kOffW1 = 0;          // [k atom 0..1][H rows][128 B]
constexpr int kOffWl = 65536;      // [k atom 0..1][128 rows][128 B]
constexpr int kOffW2 = 98304;      // [k atom 0..H/64-1][128 rows][128 B]
constexpr int kOffKt = 163840;     // k~ tile [atom 0..1][128 rows][128 B]
constexpr int kOffG0 = 196608;     // one GELU half at a time (fit mode: then R) [atom 0..1][128 rows][128 B]
constexpr int kOffEsum = 229376;   // [sub 1..3][128] partial errors (sub 0 adds them)
constexpr int kOffBar = 231424;
constexpr int kOffMisc = kOffBar + 192;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum PBar { W_FULL, W_FREE, K_FULL, K_FREE, U_FULL, U_FREE, G_READY0, G_READY1, G0_FREE, V_FULL0, V_FULL1,
            V_FREE0, V_FREE1, E_READY0, E_READY1, DRAIN, R_READY, DG_FULL, DG_FREE, G_STORED, N_PBARS };
static_assert(N_PBARS * 8 <= 192, "barrier area");

constexpr float kGeluC1 = 0.80015708f;  // tanh-form GELU: c1, c3 minimise the largest error
                                        // against x Phi(x) on [-10, 10] (2.71e-4)
constexpr float kGeluC3 = 0.03470089f;

__device__ __forceinline__ float gelu_f32(float x) {
  const float z = x * fmaf(kGeluC3, x * x, kGeluC1);
  const float h = 0.5f * x;
  return fmaf(h, tanh_fast(z), h);
}

// GELU and its derivative in the same tanh form: with z = x (c1 + c3 x^2) and th = tanh z,
// GELU = x/2 (1 + th) and GELU' = (1 + th)/2 + x/2 (1 - th^2)(c1 + 3 c3 x^2).
__device__ __forceinline__ void gelu_and_grad(float x, float& g, float& gp) {
  const float x2 = x * x;
  const float th = tanh_fast(x * fmaf(kGeluC3, x2, kGeluC1));
  const float h = 0.5f * x;
  g = fmaf(h, th, h);
  gp = fmaf(0.5f, th, 0.5f) + h * fmaf(-th, th, 1.f) * fmaf(3.f * kGeluC3, x2, kGeluC1);
}

struct Item {
  int seg, tile, b, l, h, wh;
};

__device__ __forceinline__ Item item_of(const PredictArgs& a, int it, int n_t) {
  Item x;
  x.seg = it / n_t;
  x.tile = it % n_t;
  x.h = x.seg % a.Hkv;
  x.l = (x.seg / a.Hkv) % a.L;
  x.b = x.seg / (a.Hkv * a.L);
  x.wh = ((a.pred_per_seq ? x.b : 0) * a.L + x.l) * a.Hkv + x.h;
  return x;
}

// 8 bf16 at p (16-byte aligned) as fp32
__device__ __forceinline__ void ld_bf16x8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(q[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// The token a row of an item reads: every token (normal and fit modes) or a kept one
// (gather mode); -1 past the end or for an out-of-range index.
template <bool kGather>
__device__ __forceinline__ int item_token(const PredictArgs& a, const Item& x, int row) {
  const int ir = x.tile * 128 + row;
  if (kGather) {
    if (ir >= a.k) return -1;
    const int t = __ldg(a.res_idx + (size_t)x.seg * a.k + ir);
    return (t < 0 || t >= a.T) ? -1 : t;
  }
  return ir < a.T ? ir : -1;
}

__device__ __forceinline__ const __nv_bfloat16* value_row(const PredictArgs& a, const Item& x, int t, int sub) {
  return (const __nv_bfloat16*)a.V + ((((size_t)x.b * a.L + x.l) * a.T + (t < 0 ? 0 : t)) * a.Hkv + x.h) * 128 + sub * 32;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ bool ewait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <int kMode>  // 0 error of every token, 1 residual rows of the kept tokens, 2 fitting step
__global__ void __launch_bounds__(kThreads, 1)
pack_predict_tc_kernel(const __grid_constant__ CUtensorMap mapKt, const __grid_constant__ CUtensorMap mapW1,
                       const __grid_constant__ CUtensorMap mapWl, const __grid_constant__ CUtensorMap mapW2,
                       const __grid_constant__ CUtensorMap mapG, const __grid_constant__ CUtensorMap mapR,
                       const PredictArgs a) {
  constexpr bool kGather = kMode == 1, kFit = kMode == 2;
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
  const int H = a.H, nh = a.H / 128;
  const int n_t = kGather ? (a.k + 127) / 128 : (a.T + 127) / 128;
  const int n_items = a.B * a.L * a.Hkv * n_t;
  const int it0 = (int)((long long)blockIdx.x * n_items / gridDim.x);
  const int it1 = (int)((long long)(blockIdx.x + 1) * n_items / gridDim.x);

  if (threadIdx.x == 0) {
    mbar_init(&bars[W_FULL], 1);
    mbar_init(&bars[W_FREE], 1);
    mbar_init(&bars[K_FULL], 1);
    mbar_init(&bars[K_FREE], 1);
    mbar_init(&bars[U_FULL], 1);
    mbar_init(&bars[U_FREE], kEpiWarps);
    mbar_init(&bars[G_READY0], kEpiWarps);
    mbar_init(&bars[G_READY1], kEpiWarps);
    mbar_init(&bars[G0_FREE], 1);
    mbar_init(&bars[V_FULL0], 1);
    mbar_init(&bars[V_FULL1], 1);
    mbar_init(&bars[V_FREE0], kEpiWarps);
    mbar_init(&bars[V_FREE1], kEpiWarps);
    mbar_init(&bars[E_READY0], 12);  // the warps of subs 1-3
    mbar_init(&bars[E_READY1], 12);
    mbar_init(&bars[DRAIN], 1);
    mbar_init(&bars[R_READY], kEpiWarps);
    mbar_init(&bars[DG_FULL], 1);
    mbar_init(&bars[DG_FREE], kEpiWarps);
    mbar_init(&bars[G_STORED], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapKt);
    tma_prefetch_desc(&mapW1);
    tma_prefetch_desc(&mapWl);
    tma_prefetch_desc(&mapW2);
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
    bool ok = true;
    int cur_wh = -1;
    uint32_t nw = 0, nk_issued = 0;
    const uint32_t w_bytes = (uint32_t)(2 * H * 128 + 128 * 128) * 2u;  // W1 and W2 (H x 128 each), W_lin
    for (int it = it0, i = 0; it < it1 && ok; ++it, ++i) {
      const Item x = item_of(a, it, n_t);
      if (x.wh != cur_wh) {
        if (cur_wh >= 0 && !(ok = ewait(&bars[W_FREE], (nw - 1) & 1, abort_flag))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[W_FULL], w_bytes);
          for (int at = 0; at < 2; ++at)
            for (int rh = 0; rh < nh; ++rh)
              tma_load_2d(sm + kOffW1 + at * H * 128 + rh * 16384, &mapW1, &bars[W_FULL], 64 * at, x.wh * H + 128 * rh);
          for (int at = 0; at < 2; ++at)
            tma_load_2d(sm + kOffWl + at * 16384, &mapWl, &bars[W_FULL], 64 * at, x.wh * 128);
          for (int at = 0; at < H / 64; ++at)
            tma_load_2d(sm + kOffW2 + at * 16384, &mapW2, &bars[W_FULL], 64 * at, x.wh * 128);
        }
        ++nw;
        cur_wh = x.wh;
      }
      if (i > 0 && !(ok = ewait(&bars[K_FREE], (i - 1) & 1, abort_flag))) break;
      const int col0 = (x.l * a.Hkv + x.h) * 128;
      if (!kGather) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars[K_FULL], 32768u);
          tma_load_3d(sm + kOffKt, &mapKt, &bars[K_FULL], col0, x.tile * 128, x.b);
          tma_load_3d(sm + kOffKt + 16384, &mapKt, &bars[K_FULL], col0 + 64, x.tile * 128, x.b);
        }
        ++nk_issued;
      } else {
        int bad = 0;
#pragma unroll 1
        for (int rr = 0; rr < 4; ++rr) {
          const int row = lane + 32 * rr;
          const int ir = x.tile * 128 + row;
          int t = -1;
          if (ir < a.k) {
            t = __ldg(a.res_idx + (size_t)x.seg * a.k + ir);
            if (t < 0 || t >= a.T) {
              bad |= LR_DEVERR_RES_RANGE;
              t = -1;
            }
          }
          const uint4* src = reinterpret_cast<const uint4*>(
              (const __half*)a.Kt + ((size_t)x.b * a.T + (t < 0 ? 0 : t)) * a.D + col0);
#pragma unroll
          for (int h4 = 0; h4 < 4; ++h4) {  // half a 64-column atom at a time
            uint4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = t >= 0 ? __ldg(src + 4 * h4 + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int q16 = 4 * (h4 & 1) + c;
              *reinterpret_cast<uint4*>(sm + kOffKt + (h4 >> 1) * 16384 + row * 128 + ((q16 ^ (row & 7)) << 4)) = v[c];
            }
          }
        }
        if (bad) flag_error(a.errword, bad);
        fence_proxy_async_smem();
        warp_arrive(&bars[K_FULL], lane);
      }
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(a.errword, LR_DEVERR_TIMEOUT);
    }
    // loads still in flight land before the CTA may exit (the last phase of each barrier)
    if (lane == 0 && nk_issued > 0) mbar_wait_drain(&bars[K_FULL], (nk_issued - 1) & 1, kWaitCycles / 4);
    if (lane == 0 && nw > 0) mbar_wait_drain(&bars[W_FULL], (nw - 1) & 1, kWaitCycles / 4);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMAs
    if (lane == 0) {
      const uint32_t id_u = idesc_f16_f32(128, H, false, false);
      const uint32_t id_v = idesc_f16_f32(128, 128, false, false);
      const uint32_t kt = smem_u32(sm + kOffKt), g0 = smem_u32(sm + kOffG0);
      const uint32_t w1 = smem_u32(sm + kOffW1), wl = smem_u32(sm + kOffWl), w2 = smem_u32(sm + kOffW2);
      bool ok = true;
      int cur_wh = -1;
      uint32_t nw = 0;
      for (int it = it0, i = 0; it < it1 && ok; ++it, ++i) {
        const Item x = item_of(a, it, n_t);
        if (x.wh != cur_wh) {
          if (cur_wh >= 0) mma_commit(&bars[W_FREE]);
          if (!(ok = mbar_wait(&bars[W_FULL], nw & 1, abort_flag))) break;
          ++nw;
          cur_wh = x.wh;
        }
        if (!(ok = mbar_wait(&bars[K_FULL], i & 1, abort_flag))) break;
        // U's columns are free again once the previous tile read them (the GELU branch; in
        // fitting mode also GELU' in the last phase). v_hat is double-buffered, except in fitting
        // mode, where columns 384-511 hold dG.
        if (i > 0 && !(ok = mbar_wait(&bars[U_FREE], (i - 1) & 1, abort_flag))) break;
        if (kFit) {
          if (i > 0 && !(ok = mbar_wait(&bars[V_FREE0], (i - 1) & 1, abort_flag))) break;
        } else {
          if (i >= 2 && !(ok = mbar_wait(&bars[V_FREE0 + (i & 1)], ((i >> 1) - 1) & 1, abort_flag))) break;
        }
        tc_fence_after();
        const uint32_t vcol = tmem + 256 + (kFit ? 0 : 128 * (i & 1));
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16_ss(tmem, sw128_desc(kt + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                     sw128_desc(w1 + (ks >> 2) * (H * 128) + (ks & 3) * 32, 16, 1024), id_u, ks != 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16_ss(vcol, sw128_desc(kt + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                     sw128_desc(wl + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), id_v, ks != 0);
        mma_commit(&bars[U_FULL]);
        mma_commit(&bars[K_FREE]);  // the keys are read: the next tile's may load
        // the GELU halves pass through G0 one after the other; G0_FREE completes after every
        // reader of G0 (nh per tile: after each half but the last, and at the tile's end)
        for (int hf = 0; hf < nh && ok; ++hf) {
          if (!(ok = mbar_wait(&bars[G_READY0 + hf], i & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_f16_ss(vcol, sw128_desc(g0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                       sw128_desc(w2 + (2 * hf + (ks >> 2)) * 16384 + (ks & 3) * 32, 16, 1024), id_v, 1);
          if (hf < nh - 1) mma_commit(&bars[G0_FREE]);
        }
        if (!ok) break;
        mma_commit(&bars[V_FULL0 + (kFit ? 0 : (i & 1))]);
        if (kFit) {  // MMA4, per 128-unit half: dG = R W2_half (R in G0, W2 read MN-major) -> cols 384+
          if (!(ok = mbar_wait(&bars[R_READY], i & 1, abort_flag))) break;
          const uint32_t id_dg = idesc_f16_f32(128, 128, false, true);
          for (int hf = 0; hf < nh && ok; ++hf) {
            const int c = i * nh + hf - 1;  // DG_FREE completion that frees the dG columns
            if (c >= 0 && !(ok = mbar_wait(&bars[DG_FREE], c & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_f16_ss(tmem + 384, sw128_desc(g0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                         sw128_desc(w2 + 2 * hf * 16384 + ks * 2048, 16384, 1024), id_dg, ks != 0);
            mma_commit(&bars[DG_FULL]);
          }
          if (!ok) break;
        }
        mma_commit(&bars[G0_FREE]);
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(a.errword, LR_DEVERR_TIMEOUT);
      }
      mma_commit(&bars[DRAIN]);
      mbar_wait_drain(&bars[DRAIN], 0, kWaitCycles / 4);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-17)
    const int q = warp & 3, sub = (warp - 2) >> 2;  // lane quarter, 32-column slice
    const int row = q * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    float* esum = reinterpret_cast<float*>(sm + kOffEsum);
    bool ok = true;
    if (it0 < it1) {  // the first tile's value rows start coming from HBM into L2
      const Item x0 = item_of(a, it0, n_t);
      const int t0 = item_token<kGather>(a, x0, row);
      if (t0 >= 0) prefetch_l2(value_row(a, x0, t0, sub));
    }
    for (int it = it0, i = 0; it < it1 && ok; ++it, ++i) {
      const Item x = item_of(a, it, n_t);
      const int ir = x.tile * 128 + row;
      const int t = item_token<kGather>(a, x, row);
      if (it + 1 < it1) {  // the next tile's value rows, one tile ahead
        const Item xn = item_of(a, it + 1, n_t);
        const int tn = item_token<kGather>(a, xn, row);
        if (tn >= 0) prefetch_l2(value_row(a, xn, tn, sub));
      }
      const __nv_bfloat16* b1 = (const __nv_bfloat16*)a.b1 + (size_t)x.wh * H;
      const float* b1f = kFit ? a.b1f + (size_t)x.wh * H : nullptr;
      // ---- GELU branch: this warp's 64 of every 128 hidden units
      if (!(ok = ewait(&bars[U_FULL], i & 1, abort_flag))) break;
      tc_fence_after();
      // this warp's 32 of every 128 hidden units
      for (int hf = 0; hf < nh && ok; ++hf) {
        const int c0 = hf * 128 + sub * 32;
        uint8_t* gt = sm + kOffG0 + (sub >> 1) * 16384 + row * 128;  // atom sub/2, chunks 4(sub&1)..+3
        uint4 b1raw[4];  // bf16 biases, loaded while the TMEM read is in flight
        if (!b1f) {
#pragma unroll
          for (int j = 0; j < 4; ++j) b1raw[j] = __ldg(reinterpret_cast<const uint4*>(b1 + c0) + j);
        }
        uint32_t u[32];
        tmem_ld32(trow + c0, u);
        tmem_ld_wait();
        if (!kFit && hf == nh - 1) {  // fitting mode reads U again for GELU'
          tc_fence_before();
          warp_arrive(&bars[U_FREE], lane);
        }
        // G0's previous reader is done: the last MMA of the previous tile (commit i nh - 1), or
        // MMA3b of half 0 of this tile (commit i nh); in fitting mode also the TMA store of
        // G0's previous contents (the previous tile's R, or this tile's half 0)
        const int commit = hf == 0 ? i * nh - 1 : i * nh;
        if (commit >= 0 && !(ok = ewait(&bars[G0_FREE], commit & 1, abort_flag))) break;
        if (kFit) {
          const int stored = i * (nh + 1) + hf - 1;
          if (stored >= 0 && !(ok = ewait(&bars[G_STORED], stored & 1, abort_flag))) break;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float bb[8];
          if (b1f) {
            const float4 f0 = __ldg(reinterpret_cast<const float4*>(b1f + c0 + 8 * j));
            const float4 f1 = __ldg(reinterpret_cast<const float4*>(b1f + c0 + 8 * j) + 1);
            bb[0] = f0.x; bb[1] = f0.y; bb[2] = f0.z; bb[3] = f0.w;
            bb[4] = f1.x; bb[5] = f1.y; bb[6] = f1.z; bb[7] = f1.w;
          } else {
            const __nv_bfloat162* bp = reinterpret_cast<const __nv_bfloat162*>(&b1raw[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float2 f = __bfloat1622float2(bp[c]);
              bb[2 * c] = f.x;
              bb[2 * c + 1] = f.y;
            }
          }
          float g[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) g[c] = gelu_f32(__uint_as_float(u[8 * j + c]) + bb[c]);
          uint4 w;
          w.x = pack_f16x2_sat(g[0], g[1]);
          w.y = pack_f16x2_sat(g[2], g[3]);
          w.z = pack_f16x2_sat(g[4], g[5]);
          w.w = pack_f16x2_sat(g[6], g[7]);
          const int q16 = 4 * (sub & 1) + j;  // 16-byte chunk of the row within the atom
          *reinterpret_cast<uint4*>(gt + ((q16 ^ (row & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
        warp_arrive(&bars[G_READY0 + hf], lane);
        if (kFit && warp == 2 && lane == 0) {  // the storer: g of this half to global memory
          if (!(ok = mbar_wait(&bars[G_READY0 + hf], i & 1, abort_flag))) break;
          for (int at = 0; at < 2; ++at)
            tma_store_3d(&mapG, sm + kOffG0 + at * 16384, hf * 128 + 64 * at, x.tile * 128, x.seg);
          bulk_commit_group();
          bulk_wait_read_le0();
          mbar_arrive(&bars[G_STORED]);
        }
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      if (!ok) break;
      // ---- value prediction done: d = v - (v_hat + b2); the value row is loaded first
      const int par = i & 1;
      uint4 vrow[4];
      {
        const uint4* vsrc = reinterpret_cast<const uint4*>(value_row(a, x, t, sub));
#pragma unroll
        for (int j = 0; j < 4; ++j) vrow[j] = t >= 0 ? __ldg(vsrc + j) : make_uint4(0, 0, 0, 0);
      }
      if (!(ok = ewait(&bars[V_FULL0 + (kFit ? 0 : par)], kFit ? (i & 1) : ((i >> 1) & 1), abort_flag))) break;
      tc_fence_after();
      float e = 0.f;
      {
        const __nv_bfloat16* b2 = (!kFit && a.b2) ? (const __nv_bfloat16*)a.b2 + (size_t)x.wh * 128 + sub * 32 : nullptr;
        const float* b2f = (kFit && a.b2f) ? a.b2f + (size_t)x.wh * 128 + sub * 32 : nullptr;
        __nv_bfloat16* out = (kGather && t >= 0) ? (__nv_bfloat16*)a.res_val + ((size_t)x.seg * a.k + ir) * 128 + sub * 32
                                                  : nullptr;
        uint8_t* rt = sm + kOffG0 + (sub >> 1) * 16384 + row * 128;  // fit: R as the A operand of MMA4
        if (kFit) {  // the store of the last g half has read G0
          const int stored = i * (nh + 1) + nh - 1;
          if (!(ok = ewait(&bars[G_STORED], stored & 1, abort_flag))) break;
        }
        uint32_t vh[32];
        tmem_ld32(trow + 256 + (kFit ? 0 : 128 * par) + sub * 32, vh);
        tmem_ld_wait();
        tc_fence_before();
        warp_arrive(&bars[V_FREE0 + (kFit ? 0 : par)], lane);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[8], bb[8];
          {
            const __nv_bfloat162* vp = reinterpret_cast<const __nv_bfloat162*>(&vrow[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float2 f = __bfloat1622float2(vp[c]);
              v[2 * c] = f.x;
              v[2 * c + 1] = f.y;
            }
          }
          if (b2) ld_bf16x8(b2 + 8 * j, bb);
          if (b2f) {
#pragma unroll
            for (int c = 0; c < 8; ++c) bb[c] = __ldg(b2f + 8 * j + c);
          }
          float d[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float p = __uint_as_float(vh[8 * j + c]) + ((b2 || b2f) ? bb[c] : 0.f);
            d[c] = t >= 0 ? v[c] - p : 0.f;
            e = fmaf(d[c], d[c], e);
          }
          if (out) {
            uint4 w;
            w.x = pack_bf16x2(d[0], d[1]);
            w.y = pack_bf16x2(d[2], d[3]);
            w.z = pack_bf16x2(d[4], d[5]);
            w.w = pack_bf16x2(d[6], d[7]);
            reinterpret_cast<uint4*>(out)[j] = w;
          }
          if (kFit) {  // R = v_hat - v
            uint4 w;
            w.x = pack_f16x2_sat(-d[0], -d[1]);
            w.y = pack_f16x2_sat(-d[2], -d[3]);
            w.z = pack_f16x2_sat(-d[4], -d[5]);
            w.w = pack_f16x2_sat(-d[6], -d[7]);
            const int q16 = 4 * (sub & 1) + j;
            *reinterpret_cast<uint4*>(rt + ((q16 ^ (row & 7)) << 4)) = w;
          }
        }
      }
      if (kFit) {
        fence_proxy_async_smem();
        warp_arrive(&bars[R_READY], lane);
        if (warp == 2 && lane == 0) {  // the storer: R to global memory
          if (!(ok = mbar_wait(&bars[R_READY], i & 1, abort_flag))) break;
          for (int at = 0; at < 2; ++at) tma_store_3d(&mapR, sm + kOffG0 + at * 16384, 64 * at, x.tile * 128, x.seg);
          bulk_commit_group();
          bulk_wait_read_le0();
          mbar_arrive(&bars[G_STORED]);
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        // ---- dU' = (R W2) * GELU'(u) per 128-unit half; u = U + b1 is read again from TMEM
        for (int hf = 0; hf < nh && ok; ++hf) {
          if (!(ok = ewait(&bars[DG_FULL], (i * nh + hf) & 1, abort_flag))) break;
          tc_fence_after();
          const int c0 = hf * 128 + sub * 32;
          uint32_t dg[32];
          tmem_ld32(trow + 384 + sub * 32, dg);
          tmem_ld_wait();
          tc_fence_before();
          warp_arrive(&bars[DG_FREE], lane);  // the next half's dG may overwrite the columns
          for (int ch = 0; ch < 2; ++ch) {    // U in two 16-column pieces
            uint32_t uu[16];
            tmem_ld16(trow + c0 + 16 * ch, uu);
            tmem_ld_wait();
            if (hf == nh - 1 && ch == 1) {
              tc_fence_before();
              warp_arrive(&bars[U_FREE], lane);
            }
            if (t < 0) continue;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const int j = 2 * ch + jj;
              const float4 f0 = __ldg(reinterpret_cast<const float4*>(b1f + c0 + 8 * j));
              const float4 f1 = __ldg(reinterpret_cast<const float4*>(b1f + c0 + 8 * j) + 1);
              const float bb[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
              float du[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                float g, gp;
                gelu_and_grad(__uint_as_float(uu[8 * jj + c]) + bb[c], g, gp);
                du[c] = __uint_as_float(dg[8 * j + c]) * gp;
              }
              uint4 w;
              w.x = pack_f16x2_sat(du[0], du[1]);
              w.y = pack_f16x2_sat(du[2], du[3]);
              w.z = pack_f16x2_sat(du[4], du[5]);
              w.w = pack_f16x2_sat(du[6], du[7]);
              reinterpret_cast<uint4*>((__half*)a.DUout + ((size_t)x.seg * a.T + t) * H + c0)[j] = w;
            }
          }
        }
      } else if (!kGather) {  // the row's error: sub 0 adds the partial sums of subs 1-3
        if (sub != 0) {
          esum[(sub - 1) * 128 + row] = e;
          warp_arrive(&bars[E_READY0 + par], lane);
        } else {
          if (!(ok = ewait(&bars[E_READY0 + par], (i >> 1) & 1, abort_flag))) break;
          if (t >= 0) a.err[(size_t)x.seg * a.T + t] = ((e + esum[row]) + esum[128 + row]) + esum[256 + row];
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      flag_error(a.errword, LR_DEVERR_TIMEOUT);
    }
    if (kFit && warp == 2 && lane == 0) bulk_wait_all();  // the stored g and R rows have landed
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

__global__ void weights_f16_kernel(const __nv_bfloat16* __restrict__ W1, const __nv_bfloat16* __restrict__ Wl,
                                   const __nv_bfloat16* __restrict__ W2, size_t n1, size_t nl, __half* __restrict__ W1h,
                                   __half* __restrict__ Wlh, __half* __restrict__ W2h) {
  const size_t n = n1 + nl + n1;  // W2 has as many entries as W1
  for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += (size_t)gridDim.x * blockDim.x * 4) {
    const __nv_bfloat16* src;
    __half* dst;
    size_t j;
    if (i < n1) { src = W1; dst = W1h; j = i; }
    else if (i < n1 + nl) { src = Wl; dst = Wlh; j = i - n1; }
    else { src = W2; dst = W2h; j = i - n1 - nl; }
    const uint2 v = *reinterpret_cast<const uint2*>(src + j);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    uint2 o;
    o.x = pack_f16x2_sat(__low2float(lo), __high2float(lo));
    o.y = pack_f16x2_sat(__low2float(hi), __high2float(hi));
    *reinterpret_cast<uint2*>(dst + j) = o;
  }
}

}  // namespace

cudaError_t launch_pack_predict_tc(const PredictArgs& a, const CUtensorMap& mKt, const CUtensorMap& mW1,
                                   const CUtensorMap& mWl, const CUtensorMap& mW2, const CUtensorMap* mG,
                                   const CUtensorMap* mR, cudaStream_t st) {
  const int n_t = a.gather ? (a.k + 127) / 128 : (a.T + 127) / 128;
  const long long n_items = (long long)a.B * a.L * a.Hkv * n_t;
  if (n_items == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(n_items < sms ? n_items : sms);
  auto kern = a.fit ? pack_predict_tc_kernel<2> : (a.gather ? pack_predict_tc_kernel<1> : pack_predict_tc_kernel<0>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the g and R maps are used in fitting mode only; the other modes get placeholders
  kern<<<grid, kThreads, kSmemBytes, st>>>(mKt, mW1, mWl, mW2, mG ? *mG : mKt, mR ? *mR : mKt, a);
  return cudaGetLastError();
}

cudaError_t launch_weights_f16(const void* W1, const void* Wl, const void* W2, int n_heads, int H, void* W1h,
                               void* Wlh, void* W2h, cudaStream_t st) {
  const size_t n1 = (size_t)n_heads * H * 128, nl = (size_t)n_heads * 128 * 128;
  const size_t vec = (n1 + nl + n1) / 4;
  const int grid = (int)((vec + 255) / 256 < 1024 ? (vec + 255) / 256 : 1024);
  weights_f16_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)W1, (const __nv_bfloat16*)Wl,
                                           (const __nv_bfloat16*)W2, n1, nl, (__half*)W1h, (__half*)Wlh, (__half*)W2h);
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace lr
