// Residual token selection ("Predicting the value cache from keys", paragraph 4:
// exact corrections go to the tokens the predictor reconstructs worst).
//
// Per segment (one (sequence, layer, KV head)) the k tokens of largest error are
// chosen, ties to the lower token index, and written in ascending index order.
// Errors are mapped to order-preserving 32-bit keys; an MSB-first radix select
// (four 8-bit passes with warp-aggregated shared-memory histograms) finds the key
// K* of the k-th largest error and how many tokens tie at K*; one ordered
// compaction pass then emits every token above K* plus the lowest-index ties.
// Every (key, index) pair is distinct, so the result is unique and the step is
// exact integer work.
#include "lr_common.cuh"
#include "lr_launch.h"
#include "sm100.cuh"

namespace lr {
namespace {

constexpr int TK_THREADS = 1024;
constexpr int TK_WARPS = TK_THREADS / 32;

// IEEE order as unsigned order; -0 maps with +0, NaN below every number.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix of one flag per thread over the block; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(bool flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  int before = 0, sum = 0;
  for (int w = 0; w < TK_WARPS; ++w) {
    const int c = warp_tot[w];
    if (w < warp) before += c;
    sum += c;
  }
  total = sum;
  __syncthreads();
  return before + in_warp;
}

// Digit of the kr-th largest key among those matching the current prefix, from the 256-bin
// histogram h of the pass: the largest d with (sum of h above d) + h[d] >= kr (0 if none), and
// kr minus the count above d. Run by one whole warp: lane l owns bins 8l .. 8l+7, a suffix
// scan over lanes finds the lane that holds the digit, that lane scans its bins.
__device__ __forceinline__ void find_digit_warp(const int* h, int kr, int* out_digit, int* out_kr) {
  const int lane = threadIdx.x & 31;
  int v[8], s = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = h[8 * lane + i];
    s += v[i];
  }
  int incl = s;  // sum over lanes >= this one (higher digits)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += x;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= kr);
  if (hit == 0u) {  // fewer than kr keys left: the scan of the serial form ends at digit 0
    const int above0 = __shfl_sync(0xffffffffu, incl, 0) - __shfl_sync(0xffffffffu, v[0], 0);
    if (lane == 0) {
      *out_digit = 0;
      *out_kr = kr - above0;
    }
    return;
  }
  const int L = 31 - __clz((int)hit);
  if (lane == L) {
    int cum = incl - s;  // keys in the bins above this lane's
    int d = 8 * lane + 7;
#pragma unroll
    for (int i = 7; i > 0; --i, --d) {
      if (cum + v[i] >= kr) break;
      cum += v[i];
    }
    *out_digit = d;
    *out_kr = kr - cum;
  }
}

// Segments of up to kTkKeys * TK_THREADS tokens: thread tid keeps the keys of tokens
// tid + i * TK_THREADS (i < kTkKeys) in registers for all passes.
constexpr int kTkKeys = 8;

__global__ void __launch_bounds__(TK_THREADS) topk_kernel(const float* __restrict__ err, int T, int k,
                                                         int* __restrict__ out_all) {
  __shared__ int whist[TK_WARPS][256];
  __shared__ int hist[256];
  __shared__ int sh_digit, sh_kr;
  __shared__ int warp_tot[TK_WARPS];
  const int seg = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* e = err + (size_t)seg * T;
  int* out = out_all + (size_t)seg * k;
  if (k == 0) return;
  if (k == T) {
    for (int t = tid; t < T; t += TK_THREADS) out[t] = t;
    return;
  }
  const int n_it = (T + TK_THREADS - 1) / TK_THREADS;  // <= kTkKeys (checked by the launcher)
  uint32_t key[kTkKeys];
#pragma unroll
  for (int i = 0; i < kTkKeys; ++i) {
    const int t = tid + i * TK_THREADS;
    key[i] = (i < n_it && t < T) ? order_key(e[t]) : 0u;
  }
  uint32_t prefix = 0, mask = 0;
  int kr = k;  // rank still to locate among keys that match the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < TK_WARPS * 256; i += TK_THREADS) (&whist[0][0])[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kTkKeys; ++i) {
      if (i >= n_it) break;
      const int t = tid + i * TK_THREADS;
      const bool act = t < T && (key[i] & mask) == prefix;
      const int digit = (key[i] >> shift) & 255;
      const unsigned actmask = __ballot_sync(0xffffffffu, act);
      if (act) {
        const unsigned same = __match_any_sync(actmask, digit);
        if ((__ffs(same) - 1) == lane) atomicAdd(&whist[warp][digit], __popc(same));
      }
    }
    __syncthreads();
    if (tid < 256) {
      int s = 0;
      for (int w = 0; w < TK_WARPS; ++w) s += whist[w][tid];
      hist[tid] = s;
    }
    __syncthreads();
    if (warp == 0) find_digit_warp(hist, kr, &sh_digit, &sh_kr);
    __syncthreads();
    prefix |= (uint32_t)sh_digit << shift;
    mask |= 255u << shift;
    kr = sh_kr;
    __syncthreads();
  }
  // prefix is the key of the k-th largest error; kr ties at that key are taken.
  const uint32_t kstar = prefix;
  const int n_tie = kr;
  int ties_before = 0, taken_before = 0;
#pragma unroll
  for (int i = 0; i < kTkKeys; ++i) {
    if (i >= n_it || taken_before >= k) break;
    const int t = tid + i * TK_THREADS;
    const bool valid = t < T;
    const bool is_eq = valid && key[i] == kstar;
    int eq_total;
    const int eq_rank = ties_before + block_exclusive_scan(is_eq, warp_tot, eq_total);
    const bool take = valid && (key[i] > kstar || (is_eq && eq_rank < n_tie));
    int take_total;
    const int pos = taken_before + block_exclusive_scan(take, warp_tot, take_total);
    if (take) out[pos] = t;
    ties_before += eq_total;
    taken_before += take_total;
  }
}

// The same selection for long segments, spread over a cluster of kTkCluster CTAs: CTA r owns
// the tokens [r * chunk, (r + 1) * chunk). Each radix pass histograms the CTA's tokens, the
// cluster's histograms are summed through distributed shared memory, and every CTA takes the
// same digit decision. The compaction then emits each CTA's tokens after those of the CTAs
// before it (counts exchanged the same way), so the output is ascending and unique as above.
constexpr int kTkCluster = 8;
constexpr int TKC_THREADS = 512;
constexpr int TKC_WARPS = TKC_THREADS / 32;

__device__ __forceinline__ int cta_exclusive_scan(bool flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  int before = 0, sum = 0;
  for (int w = 0; w < TKC_WARPS; ++w) {
    const int c = warp_tot[w];
    if (w < warp) before += c;
    sum += c;
  }
  total = sum;
  __syncthreads();
  return before + in_warp;
}

__global__ void __cluster_dims__(kTkCluster, 1, 1) __launch_bounds__(TKC_THREADS)
    topk_cluster_kernel(const float* __restrict__ err, int T, int k, int* __restrict__ out_all) {
  __shared__ int whist[TKC_WARPS][256];
  __shared__ int hist[256];        // this CTA's histogram (read by the whole cluster)
  __shared__ int counts[2];        // this CTA's tokens above K* and tied at K* (read by the cluster)
  __shared__ int sh_digit, sh_kr;
  __shared__ int warp_tot[TKC_WARPS];
  const int seg = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = sm100::cluster_cta_rank();
  const float* e = err + (size_t)seg * T;
  int* out = out_all + (size_t)seg * k;
  const int chunk = (T + kTkCluster - 1) / kTkCluster;
  const int lo = min(T, (int)rank * chunk), hi = min(T, lo + chunk);
  // k == 0 and k == T are handled on the host side of the launch (every CTA takes this path)
  uint32_t prefix = 0, mask = 0;
  int kr = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < TKC_WARPS * 256; i += TKC_THREADS) (&whist[0][0])[i] = 0;
    __syncthreads();
    for (int t0 = lo; t0 < hi; t0 += TKC_THREADS) {
      const int t = t0 + tid;
      bool act = false;
      int digit = 0;
      if (t < hi) {
        const uint32_t key = order_key(e[t]);
        act = (key & mask) == prefix;
        digit = (key >> shift) & 255;
      }
      const unsigned actmask = __ballot_sync(0xffffffffu, act);
      if (act) {
        const unsigned same = __match_any_sync(actmask, digit);
        if ((__ffs(same) - 1) == lane) atomicAdd(&whist[warp][digit], __popc(same));
      }
    }
    __syncthreads();
    if (tid < 256) {
      int s = 0;
      for (int w = 0; w < TKC_WARPS; ++w) s += whist[w][tid];
      hist[tid] = s;
    }
    sm100::cluster_sync();  // every CTA's histogram is complete
    if (tid < 256) {
      int s = 0;
      for (uint32_t r = 0; r < kTkCluster; ++r) s += (int)sm100::ld_cluster_u32(sm100::mapa_shared(&hist[tid], r));
      whist[0][tid] = s;  // the cluster's histogram
    }
    __syncthreads();
    if (warp == 0) find_digit_warp(&whist[0][0], kr, &sh_digit, &sh_kr);
    sm100::cluster_sync();  // no CTA rewrites its histogram while another still reads it
    prefix |= (uint32_t)sh_digit << shift;
    mask |= 255u << shift;
    kr = sh_kr;
  }
  const uint32_t kstar = prefix;
  const int n_tie = kr;
  // this CTA's counts above K* and tied at K*
  int gt = 0, eq = 0;
  for (int t = lo + tid; t < hi; t += TKC_THREADS) {
    const uint32_t key = order_key(e[t]);
    gt += key > kstar;
    eq += key == kstar;
  }
  for (int o = 16; o; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  if (lane == 0) {
    whist[0][warp] = gt;
    whist[1][warp] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    int g = 0, q = 0;
    for (int w = 0; w < TKC_WARPS; ++w) {
      g += whist[0][w];
      q += whist[1][w];
    }
    counts[0] = g;
    counts[1] = q;
  }
  sm100::cluster_sync();
  int ties_before = 0, taken_before = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    const int g = (int)sm100::ld_cluster_u32(sm100::mapa_shared(&counts[0], r));
    const int q = (int)sm100::ld_cluster_u32(sm100::mapa_shared(&counts[1], r));
    const int tie_take = max(0, min(q, n_tie - ties_before));
    taken_before += g + tie_take;
    ties_before += q;
  }
  sm100::cluster_sync();  // every CTA has read the counts it needs before any CTA may exit
  for (int t0 = lo; t0 < hi; t0 += TKC_THREADS) {
    const int t = t0 + tid;
    uint32_t key = 0;
    const bool valid = t < hi;
    if (valid) key = order_key(e[t]);
    const bool is_eq = valid && key == kstar;
    int eq_total;
    const int eq_rank = ties_before + cta_exclusive_scan(is_eq, warp_tot, eq_total);
    const bool take = valid && (key > kstar || (is_eq && eq_rank < n_tie));
    int take_total;
    const int pos = taken_before + cta_exclusive_scan(take, warp_tot, take_total);
    if (take) out[pos] = t;
    ties_before += eq_total;
    taken_before += take_total;
  }
}

__global__ void __launch_bounds__(TK_THREADS) topk_all_kernel(int T, int* __restrict__ out_all) {
  int* out = out_all + (size_t)blockIdx.x * T;
  for (int t = threadIdx.x; t < T; t += TK_THREADS) out[t] = t;
}

__global__ void block_ptr_kernel(const int* __restrict__ idx, int n_seg, int k, int T, int nblk,
                                 int* __restrict__ ptr) {
  const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= (long long)n_seg * (nblk + 1)) return;
  const int seg = (int)(x / (nblk + 1)), j = (int)(x % (nblk + 1));
  const int* a = idx + (size_t)seg * k;
  const int key = j * kBlock;
  int lo = 0, hi = k;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  ptr[x] = lo;
}

}  // namespace

cudaError_t launch_topk(const float* err, int n_seg, int T, int k, int* idx_out, cudaStream_t st) {
  if (n_seg == 0 || k == 0) return cudaSuccess;
  if (T >= 4096 && k < T) {  // long segments: one cluster of CTAs per segment
    topk_cluster_kernel<<<dim3(kTkCluster, n_seg), TKC_THREADS, 0, st>>>(err, T, k, idx_out);
    return cudaGetLastError();
  }
  if (T > kTkKeys * TK_THREADS) {  // k == T on a long segment: every index, in order
    topk_all_kernel<<<n_seg, TK_THREADS, 0, st>>>(T, idx_out);
    return cudaGetLastError();
  }
  topk_kernel<<<n_seg, TK_THREADS, 0, st>>>(err, T, k, idx_out);
  return cudaGetLastError();
}

cudaError_t launch_block_ptr(const int* idx, int n_seg, int k, int T, int* ptr_out, cudaStream_t st) {
  const int nblk = ceil_div(T, kBlock);
  const long long n = (long long)n_seg * (nblk + 1);
  if (n == 0) return cudaSuccess;
  block_ptr_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(idx, n_seg, k, T, nblk, ptr_out);
  return cudaGetLastError();
}

}  // namespace lr
