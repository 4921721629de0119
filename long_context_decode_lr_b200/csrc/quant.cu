// 2-bit residual rows ("Predicting the value cache from keys", comparison table: LowRAM
// combined with quantisation keeps its residuals at 2 bits per number).
//
// Per row of hd entries: lo = min, hi = max, step = (hi - lo) / 3, and each entry x gets the
// code c = nearest integer of (x - lo) / step (ties to even), clamped to 0..3; a row whose
// entries are all equal gets code 0 everywhere. Every step is one correctly rounded fp32
// operation (explicit _rn intrinsics), so the codes are a deterministic function of the
// stored row. Codes are packed four to a byte: entry 4i + s in bits 2s..2s+1 of byte i. A
// decode step adds lo + c * step in place of the row.
#include <math_constants.h>

#include "lr_common.cuh"
#include "lr_launch.h"

namespace lr {
namespace {

// One warp per row; lane l owns the 4-entry groups l and l + 32 (hd <= 256).
template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ rows, long long n_rows, int hd,
                                                            uint8_t* __restrict__ codes, float* __restrict__ lo_out,
                                                            float* __restrict__ step_out) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const T* x = rows + row * hd;
  const int n_groups = hd / 4;
  float v[2][4];
  float mn = CUDART_INF_F, mx = -CUDART_INF_F;
#pragma unroll
  for (int gi = 0; gi < 2; ++gi) {
    const int g = lane + 32 * gi;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      v[gi][c] = g < n_groups ? to_f32(x[4 * g + c]) : 0.f;
      if (g < n_groups) {
        mn = fminf(mn, v[gi][c]);
        mx = fmaxf(mx, v[gi][c]);
      }
    }
  }
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float step = __fdiv_rn(__fsub_rn(mx, mn), 3.0f);
  if (lane == 0) {
    lo_out[row] = mn;
    step_out[row] = step;
  }
#pragma unroll
  for (int gi = 0; gi < 2; ++gi) {
    const int g = lane + 32 * gi;
    if (g >= n_groups) continue;
    uint32_t byte = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      int code = 0;
      if (step > 0.f) {
        code = __float2int_rn(__fdiv_rn(__fsub_rn(v[gi][c], mn), step));
        code = code < 0 ? 0 : (code > 3 ? 3 : code);
      }
      byte |= (uint32_t)code << (2 * c);
    }
    codes[row * n_groups + g] = (uint8_t)byte;
  }
}

}  // namespace

cudaError_t launch_quantize_rows(const void* rows, lr_dtype dt, long long n_rows, int hd, uint8_t* codes, float* lo,
                                 float* step, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const long long grid = (n_rows + 7) / 8;
  if (dt == LR_BF16)
    quantize_rows_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, st>>>((const __nv_bfloat16*)rows, n_rows, hd, codes,
                                                                         lo, step);
  else
    quantize_rows_kernel<float><<<(unsigned)grid, 256, 0, st>>>((const float*)rows, n_rows, hd, codes, lo, step);
  return cudaGetLastError();
}

}  // namespace lr
