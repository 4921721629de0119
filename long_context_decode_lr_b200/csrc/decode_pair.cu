// Tensor-core decode on CTA pairs (bf16 cache, head_dim 128, sm_100a).
//
// A pair of CTAs (a 2-CTA cluster on two SMs) owns (split, KV head h, sequence) and
// walks 256-token tiles: four 64-token blocks, consecutive in full mode, consecutive
// entries of the head's selected list in selective mode. CTA r holds blocks 2r and 2r+1
// of a tile, i.e. 128 token rows. CTA 0 issues every MMA for both (M = 256 rows):
//   MMA1  S1[256 x 144] = A_tile . [B_l^h | Qhat_h]^T   keys k~ = A B_l^h (128 columns,
//                                                       "LowRAM" project page, Figure 3) and
//                                                       scores q.k~ = A . (B_l^h q) (16 columns:
//                                                       scale B_l^h q as bf16 hi + lo rows)
//   MMA2  U[256 x 128]  = k~ . W1_half^T                GELU-branch input per 128 hidden units
//   MMA3  O3 = k~^T P, g^T P                           p-weighted sums over the tile's tokens
//                                                       ("Predicting the value cache from keys",
//                                                       paragraphs 2-3)
// Operand halves: CTA 0 holds key dims 0-71 of B_l^h, CTA 1 dims 72-127 and the Qhat rows;
// each CTA holds 64 of the 128 hidden units of a W1 half (resident for the whole kernel)
// and its own 8 rows of P. Each CTA's TMEM receives its own 128 token rows of S1 and U,
// and in O3 the columns of its own P rows are the ones it reads.
// S1 is double-buffered in TMEM: the key rebuild of the next tile runs on the tensor pipe
// while the epilogue drains, softmaxes and applies GELU to this one. Two threads of CTA 0
// issue MMAs: one streams the key rebuild stage by stage, the other issues the
// epilogue-driven MMAs as their inputs become ready; the tensor pipe interleaves them. Second-stage operands (k~, g, p, W1) are fp16 as in the single-CTA kernel. Each
// CTA writes its own split partial (m, l, sum p k~, sum p g, sum p r); the combine kernel
// merges them. Every wait is bounded: a CTA that times out raises its own and its peer's
// abort flag, records LR_DEVERR_TIMEOUT, drains what was issued and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "lr_common.cuh"
#include "lr_launch.h"
#include "lr_tc.h"
#include "sm100.cuh"

namespace lr {
namespace tc {
namespace {

using namespace sm100;

constexpr int kHd = 128;
constexpr int kChunk = 64;     // rank columns per ring stage
constexpr int kStages = 5;
constexpr int kThreads = 384;  // warp 0 TMA, 1 key-rebuild MMAs, 2-9 epilogue (two groups of 4),
                               // 10 residual rows, 11 epilogue-driven MMAs (MMAs: CTA 0 only)
constexpr int kEpiWarps = 8;
constexpr int kArrive = 2 * kEpiWarps;  // per-warp arrivals of both CTAs on CTA 0's barriers
constexpr int kBRows0 = 72;             // B_l^h rows (key dims) held by CTA 0
constexpr int kBRows1 = 56;             // held by CTA 1, followed by the 16 Qhat rows
constexpr int kN1 = 144;                // MMA1 N: 128 key dims + 16 score columns

constexpr uint32_t kColS1 = 0;     // two buffers of 144 columns
constexpr uint32_t kColU = 288;    // GELU-branch input of one 128-unit half
constexpr uint32_t kColO3 = 416;   // two parities of [sum p k~ | sum p g half 0 | half 1], 16 columns each
constexpr uint32_t kTmemCols = 512;

struct Layout {
  static constexpr uint32_t kStageBytes = 16384 + 9216;  // A rows (2 x 64 x 64) + B part (72 rows)
  static constexpr uint32_t kOffRing = 0;
  // two 32 KB fp16 tiles of the own 128 rows that trade roles every tile: tile t keeps its
  // keys in X[t & 1], the GELU outputs of hidden half 0 in X[(t + 1) & 1] and of half 1 in
  // X[t & 1] once the keys are consumed
  static constexpr uint32_t kOffX = kStages * kStageBytes;
  static constexpr uint32_t kOffW1 = kOffX + 2 * 32768;      // resident W1 part: [half][dim atom][64 rows]
  static constexpr uint32_t kOffP = kOffW1 + 32768;          // [parity] 8 rows x 128 tokens fp16
  static constexpr uint32_t kOffB1 = kOffP + 4096;           // b1 of the head, fp16 (256)
  static constexpr uint32_t kOffRed = kOffB1 + 512;          // [group][parity][warp][8] floats
  static constexpr uint32_t kOffAlpha = kOffRed + 512;       // [parity][8] softmax rescale
  static constexpr uint32_t kOffBar = kOffAlpha + 64;
  static constexpr uint32_t kOffMisc = kOffBar + 320;
  static constexpr uint32_t kSmemBytes = kOffMisc + 64;  // the dynamic base is 1024-byte aligned (checked)
};
static_assert(Layout::kOffX % 1024 == 0 && Layout::kOffW1 % 1024 == 0 && Layout::kOffP % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(Layout::kSmemBytes <= 232448, "shared memory budget");

enum Bar {
  FULL0 = 0, EMPTY0 = kStages, W1_FULL = 2 * kStages, S1_FULL0, S1_FULL1, S1_FREE0, S1_FREE1, KT_READY, KT_FREE,
  P_READY, U_FULL, U_FREE, G_READY, GF0, GF1, O3_FULL0, O3_FULL1, O3_FREE0, O3_FREE1, EPI_SYNC0, EPI_SYNC1,
  SOFT_DONE, RES_DONE, DRAIN, DRAIN2, N_BARS
};
static_assert(N_BARS * 8 <= 320, "barrier area");

constexpr float kGeluC1 = 0.80015708f;  // tanh-form GELU: c1, c3 minimise the largest error
                                        // against x Phi(x) on [-10, 10] (2.71e-4)
constexpr float kGeluC3 = 0.03470089f;

// GELU of two GELU-branch inputs: x = u + b1 in fp32, rounded once to fp16 (saturating), then
// the tanh form evaluated on the fp16 pair (packed half2 arithmetic and the half2 tanh
// approximation: half the instructions of the fp32 form; the result is stored as fp16 for
// the next contraction either way).
__device__ __forceinline__ uint32_t gelu_pair(uint32_t u0, uint32_t u1, uint32_t bias_h2) {
  const float2 bf = __half22float2(*reinterpret_cast<const __half2*>(&bias_h2));
  const uint32_t xb = pack_f16x2_sat(__uint_as_float(u0) + bf.x, __uint_as_float(u1) + bf.y);
  const __half2 x = *reinterpret_cast<const __half2*>(&xb);
  const __half2 z = __hmul2(x, __hfma2(__float2half2_rn(kGeluC3), __hmul2(x, x), __float2half2_rn(kGeluC1)));
  const uint32_t zb = *reinterpret_cast<const uint32_t*>(&z);
  uint32_t tb;
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(tb) : "r"(zb));
  const __half2 t = *reinterpret_cast<const __half2*>(&tb);
  const __half2 h = __hmul2(__float2half2_rn(0.5f), x);
  const __half2 g = __hfma2(h, t, h);
  return *reinterpret_cast<const uint32_t*>(&g);
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// byte offset of element (row, col) of a 128-byte-swizzled 16-bit tile whose 64-column
// atoms are `atom_bytes` apart
__device__ __forceinline__ uint32_t sw128_off(int row, int col, uint32_t atom_bytes) {
  const int at = col >> 6, c = col & 63;
  return at * atom_bytes + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + ((c & 7) << 1);
}

__device__ __forceinline__ int lower_bound_i32(const int* p, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Tiles of (sequence b, KV head h): 4 blocks each.
__device__ __forceinline__ int pair_tile_count(const PairArgs& a, int b, int h) {
  if (!a.sched) return (a.nblk + 3) >> 2;
  return (a.sched[((size_t)b * a.Hkv + h) * a.sched_stride] + 3) >> 2;
}

// The two blocks CTA `rank` holds in tile i (-1 where the tile runs out).
struct Blocks {
  int blk[2];
};
__device__ __forceinline__ Blocks pair_blocks(const PairArgs& a, int b, int h, int i, uint32_t rank) {
  Blocks t;
  const int e0 = 4 * i + 2 * (int)rank;
  if (!a.sched) {
#pragma unroll
    for (int x = 0; x < 2; ++x) t.blk[x] = e0 + x < a.nblk ? e0 + x : -1;
    return t;
  }
  const int* s = a.sched + ((size_t)b * a.Hkv + h) * a.sched_stride;
  const int n = s[0];
#pragma unroll
  for (int x = 0; x < 2; ++x) t.blk[x] = e0 + x < n ? s[1 + e0 + x] : -1;
  return t;
}

// Raise the abort flag of both CTAs of the pair.
__device__ __forceinline__ void abort_pair(uint8_t* sm_misc, volatile int* abort_flag, uint32_t rank) {
  *abort_flag = 1;
  st_cluster_u32(mapa_shared(sm_misc + 4, rank ^ 1u), 1u);
}

// Epilogue-side wait: every lane polls, the outcome is made uniform across the warp.
__device__ __forceinline__ bool ewait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait_cl(bar, parity, abort_flag));
}

// One arrival per warp on a barrier of CTA 0; the warp's shared-memory writes made before
// are released to the cluster (and were made visible to the tensor core by the caller).
__device__ __forceinline__ void warp_arrive_leader(uint32_t bar_cluster, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(bar_cluster);
}

template <int MG>
struct PairEpi {
  const PairArgs& a;
  uint8_t* sm;
  uint64_t* bars;
  volatile int* abort_flag;
  uint32_t rank, tmem;
  int grp, wl, lane, row, nh;
  uint32_t trow;
  uint32_t sync_phase;
  uint32_t c_kt_ready, c_s1_free0, c_p_ready, c_u_free, c_g_ready, c_o3_free0;
  // softmax state (both groups track it; group 0 owns l and sum p k~, group 1 sum p g)
  float m[MG], l[MG], acc1[MG], acc2[MG], alpha[MG], alpha_prev[MG];

  __device__ PairEpi(const PairArgs& a_, uint8_t* sm_, uint64_t* bars_, volatile int* ab, uint32_t rank_, int warp,
                     int lane_, uint32_t tmem_)
      : a(a_), sm(sm_), bars(bars_), abort_flag(ab), rank(rank_), tmem(tmem_) {
    grp = (warp - 2) >> 2;
    wl = (warp - 2) & 3;
    lane = lane_;
    const int lq = warp & 3;
    row = lq * 32 + lane;
    trow = tmem + ((uint32_t)(lq * 32) << 16);
    nh = a.H / 128;
    sync_phase = 0;
    c_kt_ready = mapa_shared(&bars[KT_READY], 0);
    c_s1_free0 = mapa_shared(&bars[S1_FREE0], 0);
    c_p_ready = mapa_shared(&bars[P_READY], 0);
    c_u_free = mapa_shared(&bars[U_FREE], 0);
    c_g_ready = mapa_shared(&bars[G_READY], 0);
    c_o3_free0 = mapa_shared(&bars[O3_FREE0], 0);
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      m[g] = -CUDART_INF_F;
      l[g] = acc1[g] = acc2[g] = 0.f;
      alpha[g] = alpha_prev[g] = 1.f;
    }
  }

  __device__ __forceinline__ bool sync_grp() {  // barrier over this epilogue group (128 threads)
    mbar_arrive(&bars[EPI_SYNC0 + grp]);
    const bool ok = ewait(&bars[EPI_SYNC0 + grp], sync_phase & 1, abort_flag);
    ++sync_phase;
    return ok;
  }

  // Scores and keys of tile tl: scores to registers, this group's 64 key columns to the
  // fp16 key tile; then S1 of this buffer is released and the keys announced.
  __device__ __forceinline__ bool drain(int tl, float (&sc)[MG]) {
    const int buf = tl & 1;
    const uint32_t col = kColS1 + buf * kN1;
    if (!ewait(&bars[S1_FULL0 + buf], (tl >> 1) & 1, abort_flag)) return false;
    tc_fence_after();
    uint32_t hi[8], lo[8];
    tmem_ld8(trow + col + 128, hi);
    tmem_ld8(trow + col + 136, lo);
    // X[tl & 1] last held the half-0 GELU outputs of tile tl-1
    if (tl > 0 && !ewait(&bars[GF0], (tl - 1) & 1, abort_flag)) return false;
    uint8_t* kt = sm + Layout::kOffX + (tl & 1) * 32768;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t v[32];
      tmem_ld32(trow + col + grp * 64 + cc * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_f16x2_sat(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
        w.y = pack_f16x2_sat(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
        w.z = pack_f16x2_sat(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
        w.w = pack_f16x2_sat(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
        *reinterpret_cast<uint4*>(kt + sw128_off(row, grp * 64 + cc * 32 + q * 8, 16384)) = w;
      }
    }
#pragma unroll
    for (int g = 0; g < MG; ++g) sc[g] = __uint_as_float(hi[g]) + __uint_as_float(lo[g]);
    tc_fence_before();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_cluster(c_s1_free0 + 8u * buf);
      mbar_arrive_cluster(c_kt_ready);
    }
    return true;
  }

  // Online softmax of tile tl (both groups, identical arithmetic); group 0 writes p and
  // the rescale factors.
  __device__ __forceinline__ bool softmax(int tl, const float (&sc_in)[MG], bool valid) {
    const int par = tl & 1;
    float* red = reinterpret_cast<float*>(sm + Layout::kOffRed) + (grp * 2 + par) * 32;
    float sc[MG];
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      sc[g] = valid ? sc_in[g] : -CUDART_INF_F;
      const float mx = warp_max(sc[g]);
      if (lane == 0) red[wl * 8 + g] = mx;
    }
    if (!sync_grp()) return false;
    float p[MG];
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      const float mt = fmaxf(fmaxf(red[g], red[8 + g]), fmaxf(red[16 + g], red[24 + g]));
      const float m_new = fmaxf(m[g], mt);
      alpha_prev[g] = alpha[g];
      alpha[g] = m_new == -CUDART_INF_F ? 1.f : __expf(m[g] - m_new);
      p[g] = valid ? __expf(sc[g] - m_new) : 0.f;
      l[g] = l[g] * alpha[g] + p[g];
      m[g] = m_new;
    }
    if (grp != 0) return true;
    // p of this parity was last read by the MMAs of tile tl-2 (merged already) and by the
    // residual warp, which finishes each tile before the next softmax
    if (tl > 0 && !ewait(&bars[RES_DONE], (tl - 1) & 1, abort_flag)) return false;
    uint8_t* ptile = sm + Layout::kOffP + par * 2048;
#pragma unroll
    for (int g = 0; g < MG; ++g)
      if (g < a.G) *reinterpret_cast<__half*>(ptile + sw128_off(g, row, 1024)) = __float2half_rn(p[g]);
    if (row == 0) {
      float* al = reinterpret_cast<float*>(sm + Layout::kOffAlpha) + par * 8;
#pragma unroll
      for (int g = 0; g < MG; ++g) al[g] = alpha[g];
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_cluster(c_p_ready);
      mbar_arrive(&bars[SOFT_DONE]);
    }
    return true;
  }

  // GELU branch of tile tl: this group's 64 of every 128 hidden units.
  __device__ __forceinline__ bool gelu(int tl) {
    const uint4* b1h = reinterpret_cast<const uint4*>(sm + Layout::kOffB1);
#pragma unroll 1
    for (int half = 0; half < nh; ++half) {
      const int j = tl * nh + half;
      uint8_t* gtile = sm + Layout::kOffX + ((tl + 1 - half) & 1) * 32768;
      if (!ewait(&bars[U_FULL], j & 1, abort_flag)) return false;
      tc_fence_after();
      uint32_t u[2][32];
      tmem_ld32(trow + kColU + grp * 64, u[0]);
      tmem_ld32(trow + kColU + grp * 64 + 32, u[1]);
      tmem_ld_wait();
      tc_fence_before();
      warp_arrive_leader(c_u_free, lane);
      if (half == 0) {  // X[(tl + 1) & 1]: keys and last GELU outputs of tile tl-1 consumed
        if (tl > 0 && !ewait(&bars[nh == 2 ? GF1 : GF0], (tl - 1) & 1, abort_flag)) return false;
      } else {          // X[tl & 1]: this tile's keys consumed
        if (!ewait(&bars[KT_FREE], tl & 1, abort_flag)) return false;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* uu = &u[q >> 2][(q & 3) * 8];
        const uint4 bb = b1h[half * 16 + grp * 8 + q];
        uint4 w;
        w.x = gelu_pair(uu[0], uu[1], bb.x);
        w.y = gelu_pair(uu[2], uu[3], bb.y);
        w.z = gelu_pair(uu[4], uu[5], bb.z);
        w.w = gelu_pair(uu[6], uu[7], bb.w);
        *reinterpret_cast<uint4*>(gtile + sw128_off(row, grp * 64 + q * 8, 16384)) = w;
      }
      fence_proxy_async_smem();
      warp_arrive_leader(c_g_ready, lane);
    }
    return true;
  }

  // Merge the p-weighted sums of tile tl (rescale factor al of that tile).
  __device__ __forceinline__ bool merge(int tl, const float (&al)[MG]) {
    const int par = tl & 1;
    if (!ewait(&bars[O3_FULL0 + par], (tl >> 1) & 1, abort_flag)) return false;
    tc_fence_after();
    const uint32_t base = trow + kColO3 + par * 48 + 8 * rank;
    uint32_t v0[8], v1[8];
    if (grp == 0) {
      tmem_ld8(base, v0);
    } else {
      tmem_ld8(base + 16, v0);
      if (nh == 2) tmem_ld8(base + 32, v1);
    }
    tmem_ld_wait();
    tc_fence_before();
    warp_arrive_leader(c_o3_free0 + 8u * par, lane);
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      acc1[g] = fmaf(acc1[g], al[g], __uint_as_float(v0[g]));
      if (grp == 1 && nh == 2) acc2[g] = fmaf(acc2[g], al[g], __uint_as_float(v1[g]));
    }
    return true;
  }

  __device__ __forceinline__ void write_partials(int b, int h, int split) {
    float* red = reinterpret_cast<float*>(sm + Layout::kOffRed);  // group 0, parity 0 slot
    const int Hq = a.Hkv * a.G;
    const int S = 2 * a.n_pairs;
    if (grp == 0) {
      sync_grp();
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        const float v = warp_sum(l[g]);
        if (lane == 0) red[wl * 8 + g] = v;
      }
      sync_grp();
    }
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      if (g >= a.G) continue;
      float* part = a.partials + (((size_t)b * Hq + h * a.G + g) * S + split) * a.part_stride;
      if (grp == 0) {
        if (row == 0) {
          part[0] = m[g];
          part[1] = red[g] + red[8 + g] + red[16 + g] + red[24 + g];
          part[2] = part[3] = 0.f;
        }
        part[4 + row] = acc1[g];
      } else {
        part[4 + kHd + row] = acc1[g];
        if (nh == 2) part[4 + kHd + 128 + row] = acc2[g];
      }
    }
  }
};

// The residual warp of a CTA: for each tile it scatters p_t r_t over the residual rows of
// the CTA's two blocks ("Predicting the value cache from keys", paragraph 2). Lane l owns
// dims 4l .. 4l+3; rows of a block are contiguous in res_val (indices ascending), so a batch
// of 16 rows is one coalesced 256-byte read per row (Q2: 2-bit rows, one 32-byte code read
// per row, lane l's byte holding its four dims, dequantised as lo + code * step). Loads are
// issued before waiting for p.
template <int MG, bool Q2>
__device__ __forceinline__ void pair_residual_warp(const PairArgs& a, uint8_t* sm, uint64_t* bars,
                                                   volatile int* abort_flag, uint32_t rank, int b, int h, int split,
                                                   int t_begin, int t_end) {
  const int lane = threadIdx.x & 31, G = a.G;
  const float* alphas = reinterpret_cast<const float*>(sm + Layout::kOffAlpha);
  float acc[MG][4];
#pragma unroll
  for (int g = 0; g < MG; ++g)
#pragma unroll
    for (int d = 0; d < 4; ++d) acc[g][d] = 0.f;
  int bad = 0;
  bool ok = true;
  const size_t seg = ((size_t)b * a.L + a.layer) * a.Hkv + h;
  const int* ridx = a.k > 0 ? a.res_idx + seg * a.k : nullptr;
  const __nv_bfloat16* rval = (a.k > 0 && !Q2) ? a.res_val + seg * a.k * kHd : nullptr;
  const size_t segk = seg * a.k;
  const int* rptr = (a.k > 0 && a.res_ptr) ? a.res_ptr + seg * (a.nblk + 1) : nullptr;
  int tl = 0;
  for (int ti = t_begin; ti < t_end && ok; ++ti, ++tl) {
    const Blocks t = pair_blocks(a, b, h, ti, rank);
    const int par = tl & 1;
    const uint8_t* ptile = sm + Layout::kOffP + par * 2048;
    int e0[2] = {0, 0}, ne[2] = {0, 0}, lo[2] = {0, 0}, hi[2] = {0, 0};
    if (a.k > 0) {
#pragma unroll
      for (int bh = 0; bh < 2; ++bh) {
        const int blk = t.blk[bh];
        if (blk < 0) continue;
        int x0, x1;
        if (rptr) {
          x0 = __ldg(rptr + blk);
          x1 = __ldg(rptr + blk + 1);
          if (x0 < 0 || x1 < x0 || x1 > a.k) {
            bad |= LR_DEVERR_PTR;
            continue;
          }
        } else {
          x0 = lower_bound_i32(ridx, a.k, blk * kBlock);
          x1 = lower_bound_i32(ridx, a.k, blk * kBlock + kBlock);
        }
        e0[bh] = x0;
        ne[bh] = x1 - x0;
        lo[bh] = blk * kBlock;
        hi[bh] = min(lo[bh] + kBlock, a.T);
      }
    }
    const int n_tot = ne[0] + ne[1];
    bool waited = false;
#pragma unroll 1
    for (int i0 = 0; i0 < n_tot || !waited; i0 += 16) {
      int tr[16], bh_of[16];
      uint2 rv[16];
      uint32_t cb[Q2 ? 16 : 1];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int i = i0 + j;
        const int bh = i < ne[0] ? 0 : 1;
        const int e = bh ? e0[1] + (i - ne[0]) : e0[0] + i;
        const bool in = i < n_tot;
        bh_of[j] = bh;
        tr[j] = in ? __ldg(ridx + e) : -1;
        if (Q2) {
          cb[j] = in ? (uint32_t)__ldg(a.res_codes + (segk + e) * (kHd / 4) + lane) : 0u;
          rv[j] = in ? make_uint2(__float_as_uint(__ldg(a.res_lo + segk + e)), __float_as_uint(__ldg(a.res_step + segk + e)))
                     : make_uint2(0, 0);
        } else {
          rv[j] = in ? __ldg(reinterpret_cast<const uint2*>(rval + (size_t)e * kHd) + lane) : make_uint2(0, 0);
        }
      }
      if (!waited) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait_cl(&bars[SOFT_DONE], tl & 1, abort_flag)))) break;
        waited = true;
#pragma unroll
        for (int g = 0; g < MG; ++g) {
          const float al = alphas[par * 8 + g];
#pragma unroll
          for (int d = 0; d < 4; ++d) acc[g][d] *= al;
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (i0 + j >= n_tot) break;
        const int bh = bh_of[j];
        if (j > 0 && bh_of[j - 1] == bh && tr[j - 1] >= tr[j]) bad |= LR_DEVERR_RES_ORDER;
        if (tr[j] < lo[bh] || tr[j] >= hi[bh]) {
          bad |= LR_DEVERR_RES_RANGE;
          continue;
        }
        const int prow = bh * 64 + (tr[j] - lo[bh]);
        float r0, r1, r2, r3;
        if (Q2) {
          const float qlo = __uint_as_float(rv[j].x), qst = __uint_as_float(rv[j].y);
          const uint32_t c = cb[j];
          r0 = fmaf((float)(c & 3u), qst, qlo);
          r1 = fmaf((float)((c >> 2) & 3u), qst, qlo);
          r2 = fmaf((float)((c >> 4) & 3u), qst, qlo);
          r3 = fmaf((float)((c >> 6) & 3u), qst, qlo);
        } else {
          const __nv_bfloat162 r01 = *reinterpret_cast<const __nv_bfloat162*>(&rv[j].x);
          const __nv_bfloat162 r23 = *reinterpret_cast<const __nv_bfloat162*>(&rv[j].y);
          r0 = __low2float(r01), r1 = __high2float(r01), r2 = __low2float(r23), r3 = __high2float(r23);
        }
#pragma unroll
        for (int g = 0; g < MG; ++g) {
          if (g < G) {
            const float pg = __half2float(*reinterpret_cast<const __half*>(ptile + sw128_off(g, prow, 1024)));
            acc[g][0] = fmaf(pg, r0, acc[g][0]);
            acc[g][1] = fmaf(pg, r1, acc[g][1]);
            acc[g][2] = fmaf(pg, r2, acc[g][2]);
            acc[g][3] = fmaf(pg, r3, acc[g][3]);
          }
        }
      }
    }
    if (!ok) break;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[RES_DONE]);
  }
  if (!ok) {
    abort_pair(sm + Layout::kOffMisc, abort_flag, rank);
    flag_error(a.err, LR_DEVERR_TIMEOUT);
  }
  if (bad && lane == 0) flag_error(a.err, bad);
  const int Hq = a.Hkv * G, S = 2 * a.n_pairs;
#pragma unroll
  for (int g = 0; g < MG; ++g) {
    if (g >= G) continue;
    float* part = a.partials + (((size_t)b * Hq + h * G + g) * S + split) * a.part_stride;
    *reinterpret_cast<float4*>(part + 4 + kHd + a.H + 4 * lane) =
        make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  }
}

template <int MG, bool Q2>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                   const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapQ,
                   const __grid_constant__ CUtensorMap mapW1, const PairArgs a) {
  using L = Layout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {  // same in both CTAs: neither starts, so no cluster wait is left open
    if (threadIdx.x == 0) flag_error(a.err, LR_DEVERR_LAUNCH);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffMisc + 4);

  const uint32_t rank = cluster_cta_rank();
  const int pair = blockIdx.x >> 1, h = blockIdx.y, b = blockIdx.z;
  const int split = 2 * pair + (int)rank;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H, nh = a.H / 128, nk = a.r / kChunk;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[FULL0 + i], 1);
      mbar_init(&bars[EMPTY0 + i], 1);
    }
    mbar_init(&bars[W1_FULL], 1);
    mbar_init(&bars[S1_FULL0], 1);
    mbar_init(&bars[S1_FULL1], 1);
    mbar_init(&bars[S1_FREE0], kArrive);
    mbar_init(&bars[S1_FREE1], kArrive);
    mbar_init(&bars[KT_READY], kArrive);
    mbar_init(&bars[KT_FREE], 1);
    mbar_init(&bars[P_READY], 2 * 4);
    mbar_init(&bars[U_FULL], 1);
    mbar_init(&bars[U_FREE], kArrive);
    mbar_init(&bars[G_READY], kArrive);
    mbar_init(&bars[GF0], 1);
    mbar_init(&bars[GF1], 1);
    mbar_init(&bars[O3_FULL0], 1);
    mbar_init(&bars[O3_FULL1], 1);
    mbar_init(&bars[O3_FREE0], kArrive);
    mbar_init(&bars[O3_FREE1], kArrive);
    mbar_init(&bars[EPI_SYNC0], 128);
    mbar_init(&bars[EPI_SYNC1], 128);
    mbar_init(&bars[SOFT_DONE], 4);
    mbar_init(&bars[RES_DONE], 1);
    mbar_init(&bars[DRAIN], 1);
    mbar_init(&bars[DRAIN2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB0);
    tma_prefetch_desc(&mapB1);
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapW1);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  {  // b1 of the head as fp16; zero both p tiles (rows of absent query heads stay zero)
    __half* b1s = reinterpret_cast<__half*>(sm + L::kOffB1);
    const size_t pseq = a.pred_per_seq ? (size_t)b : 0;
    for (int i = threadIdx.x; i < 256; i += kThreads)
      b1s[i] = __float2half_rn(i < H ? __bfloat162float(a.b1[((pseq * a.L + a.layer) * a.Hkv + h) * H + i]) : 0.f);
    uint32_t* pz = reinterpret_cast<uint32_t*>(sm + L::kOffP);
    for (int i = threadIdx.x; i < 1024; i += kThreads) pz[i] = 0u;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // The setup above overlaps the end of the prep grid (programmatic dependent launch); its
  // outputs (schedule, Qhat, fp16 W1) are read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_tiles = pair_tile_count(a, b, h);
  const int t_begin = (int)((long long)pair * n_tiles / a.n_pairs);
  const int t_end = (int)((long long)(pair + 1) * n_tiles / a.n_pairs);
  const int n_local = t_end - t_begin;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      const int rowB = (a.layer * a.Hkv + h) * kHd;
      const int rowQ = (b * a.Hkv + h) * kPairQRows;
      const int w1row = ((a.pred_per_seq ? b : 0) * a.Hkv + h) * H + 64 * (int)rank;
      if (n_local > 0) {
        const uint32_t cw = mapa_shared(&bars[W1_FULL], 0);
        if (rank == 0) mbar_arrive_expect_tx(&bars[W1_FULL], 2u * nh * 16384u);
        for (int half = 0; half < nh; ++half) {
          uint8_t* dst = sm + L::kOffW1 + half * 16384;
          tma_load_2d_pair(dst, &mapW1, cw, 0, w1row + half * 128);
          tma_load_2d_pair(dst + 8192, &mapW1, cw, 64, w1row + half * 128);
        }
      }
      for (int ti = t_begin; ti < t_end && ok; ++ti) {
        const Blocks t = pair_blocks(a, b, h, ti, rank);
        const int row0 = t.blk[0] >= 0 ? t.blk[0] * kBlock : a.T;
        const int row1 = t.blk[1] >= 0 ? t.blk[1] * kBlock : a.T;
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_cl(&bars[EMPTY0 + st], ph ^ 1, abort_flag))) break;
          uint8_t* dst = sm + L::kOffRing + st * L::kStageBytes;
          const uint32_t cf = mapa_shared(&bars[FULL0 + st], 0);
          if (rank == 0) mbar_arrive_expect_tx(&bars[FULL0 + st], 2u * L::kStageBytes);
          tma_load_3d_pair(dst, &mapA, cf, kc * kChunk, row0, b);
          tma_load_3d_pair(dst + 8192, &mapA, cf, kc * kChunk, row1, b);
          if (rank == 0) {
            tma_load_3d_pair(dst + 16384, &mapB0, cf, kc * kChunk, rowB, b);
          } else {
            tma_load_3d_pair(dst + 16384, &mapB1, cf, kc * kChunk, rowB + kBRows0, b);
            tma_load_2d_pair(dst + 16384 + kBRows1 * 128, &mapQ, cf, kc * kChunk, rowQ);
          }
        }
      }
      if (!ok) {
        abort_pair(sm + L::kOffMisc, abort_flag, rank);
        flag_error(a.err, LR_DEVERR_TIMEOUT);
      }
      // drain: the loads of the last stages have landed (CTA 0's barriers count both CTAs' bytes)
      if (rank == 0) {
        if (n_local > 0) mbar_wait_cl_drain(&bars[W1_FULL], 0, kWaitCycles / 4);
        for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
          mbar_wait_cl_drain(&bars[FULL0 + j % kStages], (j / kStages) & 1, kWaitCycles / 4);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- key-rebuild MMAs (CTA 0)
    if (rank == 0 && lane == 0 && n_local > 0) {
      const uint32_t id_s1 = idesc_bf16_f32(256, kN1, false, false);
      uint32_t it = 0;
      bool ok = true;
      for (int m1 = 0; m1 < n_local && ok; ++m1) {
        const int buf = m1 & 1;
        if (m1 >= 2 && !(ok = mbar_wait_cl(&bars[S1_FREE0 + buf], ((m1 >> 1) - 1) & 1, abort_flag))) break;
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_cl(&bars[FULL0 + st], ph, abort_flag))) break;
          tc_fence_after();
          const uint32_t base = smem_u32(sm + L::kOffRing + st * L::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16_pair(tmem + kColS1 + buf * kN1, sw128_desc(base + ks * 32, 16, 1024),
                         sw128_desc(base + 16384 + ks * 32, 16, 1024), id_s1, (kc | ks) != 0);
          mma_commit_pair_mc(&bars[EMPTY0 + st], 3);
        }
        if (ok) mma_commit_pair_mc(&bars[S1_FULL0 + buf], 3);
      }
      if (!ok) {
        abort_pair(sm + L::kOffMisc, abort_flag, rank);
        flag_error(a.err, LR_DEVERR_TIMEOUT);
      }
      // every MMA this thread issued has completed before either CTA releases TMEM or smem
      mma_commit_pair_mc(&bars[DRAIN], 1);
      mbar_wait_cl_drain(&bars[DRAIN], 0, kWaitCycles / 4);
    }
  } else if (warp == 11) {
    // ---------------------------------------------------------------- epilogue-driven MMAs (CTA 0)
    // In the order the epilogue produces their inputs: U = k~ W1_half^T, sum p k~, sum p g.
    if (rank == 0 && lane == 0 && n_local > 0) {
      const uint32_t id_u = idesc_f16_f32(256, 128, false, false);
      const uint32_t id_o3 = idesc_f16_f32(256, 16, true, false);
      const uint32_t x0 = smem_u32(sm + L::kOffX);
      const uint32_t w1 = smem_u32(sm + L::kOffW1), pt0 = smem_u32(sm + L::kOffP);
      uint32_t kt = x0;
      auto mma2 = [&](int half) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16_pair(tmem + kColU, sw128_desc(kt + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                       sw128_desc(w1 + half * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_u, ks != 0);
      };
      auto mma3 = [&](uint32_t a_base, uint32_t dcol, uint32_t pt) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16_pair(tmem + dcol, sw128_desc(a_base + ks * 2048, 16384, 1024),
                       sw128_desc(pt + (ks >> 2) * 1024 + (ks & 3) * 32, 16, 1024), id_o3, ks != 0);
      };
      bool ok = mbar_wait_cl(&bars[W1_FULL], 0, abort_flag);
      for (int e = 0; e < n_local && ok; ++e) {
        const int par = e & 1, jb = e * nh;
        const uint32_t pt = pt0 + par * 2048;
        const uint32_t o3 = kColO3 + par * 48;
        kt = x0 + (e & 1) * 32768;
        // U = k~ W1_half0^T
        if (!(ok = mbar_wait_cl(&bars[KT_READY], e & 1, abort_flag))) break;
        if (jb > 0 && !(ok = mbar_wait_cl(&bars[U_FREE], (jb - 1) & 1, abort_flag))) break;
        tc_fence_after();
        mma2(0);
        mma_commit_pair_mc(&bars[U_FULL], 3);
        // sum p k~
        if (!(ok = mbar_wait_cl(&bars[P_READY], e & 1, abort_flag))) break;
        if (e >= 2 && !(ok = mbar_wait_cl(&bars[O3_FREE0 + par], ((e >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        mma3(kt, o3, pt);
        if (nh == 2) {  // U = k~ W1_half1^T
          if (!(ok = mbar_wait_cl(&bars[U_FREE], jb & 1, abort_flag))) break;
          tc_fence_after();
          mma2(1);
          mma_commit_pair_mc(&bars[U_FULL], 3);
        }
        mma_commit_pair_mc(&bars[KT_FREE], 3);
        for (int half = 0; half < nh && ok; ++half) {  // sum p g
          if (!(ok = mbar_wait_cl(&bars[G_READY], (jb + half) & 1, abort_flag))) break;
          tc_fence_after();
          mma3(x0 + ((e + 1 - half) & 1) * 32768, o3 + 16 + 16 * half, pt);
          mma_commit_pair_mc(&bars[GF0 + half], 3);
        }
        if (ok) mma_commit_pair_mc(&bars[O3_FULL0 + par], 3);
      }
      if (!ok) {
        abort_pair(sm + L::kOffMisc, abort_flag, rank);
        flag_error(a.err, LR_DEVERR_TIMEOUT);
      }
      mma_commit_pair_mc(&bars[DRAIN2], 1);
      mbar_wait_cl_drain(&bars[DRAIN2], 0, kWaitCycles / 4);
    }
  } else if (warp == 10) {
    // ---------------------------------------------------------------- residual rows
    pair_residual_warp<MG, Q2>(a, sm, bars, abort_flag, rank, b, h, split, t_begin, t_end);
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-9)
    PairEpi<MG> e(a, sm, bars, abort_flag, rank, warp, lane, tmem);
    bool ok = true;
    for (int i = 0; i < n_local && ok; ++i) {
      const Blocks t = pair_blocks(a, b, h, t_begin + i, rank);
      const int blk = t.blk[e.row >> 6];
      const int tok = blk * kBlock + (e.row & 63);
      const bool valid = blk >= 0 && tok < a.T;
      float sc[MG];
      if (!(ok = e.drain(i, sc))) break;
      if (!(ok = e.softmax(i, sc, valid))) break;
      if (i > 0 && !(ok = e.merge(i - 1, e.alpha_prev))) break;
      if (!(ok = e.gelu(i))) break;
    }
    if (ok && n_local > 0) ok = e.merge(n_local - 1, e.alpha);
    if (!ok) {
      abort_pair(sm + L::kOffMisc, abort_flag, rank);
      flag_error(a.err, LR_DEVERR_TIMEOUT);
    }
    e.write_partials(b, h, split);
  }
  // ---------------------------------------------------------------- teardown
  __syncwarp();  // the cluster barrier is warp-aligned
  tc_fence_before();
  cluster_sync();  // no CTA frees TMEM or exits while the pair's MMAs or loads may touch it
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// Prep work of one decode call on the pair path, one launch:
//   blocks [0, n_w1)             the layer's W1 as fp16 (saturating outside the fp16 range)
//   blocks [n_w1, n_w1 + n_q)    Qhat = scale * B_l^h q per KV head: 16 rows, the bf16 hi
//                                parts of query heads 0-7 then the lo parts (x - hi), zero rows
//                                for absent query heads; one block per (64 rank columns, KV
//                                head, sequence)
//   blocks [n_w1 + n_q, ...)     selective mode: per (sequence, KV head) the valid entries of
//                                the block list (in range, strictly ascending); others are
//                                skipped and flagged
__global__ void __launch_bounds__(256) decode_pair_prep_kernel(PairArgs a, int n_w1, int n_q, const int* blocks,
                                                               int n_sel) {
  const int bid = blockIdx.x, tid = threadIdx.x;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs come from the kernels before this one
  if (bid < n_w1) {
    const size_t per_seq = (size_t)a.Hkv * a.H * kHd;
    const size_t n = (size_t)a.w1_seqs * per_seq;
    for (size_t i = ((size_t)bid * 256 + tid) * 4; i < n; i += (size_t)n_w1 * 256 * 4) {
      const size_t sq = i / per_seq, r = i % per_seq;
      const uint2 v = *reinterpret_cast<const uint2*>(a.W1 + (sq * a.L + a.layer) * per_seq + r);
      const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
      const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
      uint2 o;
      o.x = pack_f16x2_sat(__low2float(lo), __high2float(lo));
      o.y = pack_f16x2_sat(__low2float(hi), __high2float(hi));
      *reinterpret_cast<uint2*>(a.W1h + i) = o;
    }
    return;
  }
  if (bid < n_w1 + n_q) {
    // thread (dg, c) sums 32 of the 128 key dims for rank column c; then a 4-way reduction
    __shared__ float qs[8][kHd];
    __shared__ float part[4][64][8];
    const int nj = (a.r + 63) / 64;
    const int q = bid - n_w1;
    const int jc = q % nj, h = (q / nj) % a.Hkv, b = q / (nj * a.Hkv);
    const int G = a.G;
    for (int i = tid; i < 8 * kHd; i += 256) {
      const int g = i / kHd, d = i % kHd;
      qs[g][d] = g < G ? __bfloat162float(a.q[(((size_t)b * a.Hkv + h) * G + g) * kHd + d]) * a.scale : 0.f;
    }
    __syncthreads();
    const int c = tid & 63, dg = tid >> 6;
    const int j = jc * 64 + c;
    float acc[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) acc[g] = 0.f;
    if (j < a.r) {
      const size_t D = (size_t)a.L * a.Hkv * kHd;
      const __nv_bfloat16* bt =
          a.Bt + (size_t)b * D * a.r + ((size_t)(a.layer * a.Hkv + h) * kHd + dg * 32) * a.r + j;
      float v[32];
#pragma unroll
      for (int d = 0; d < 32; ++d) v[d] = __bfloat162float(bt[(size_t)d * a.r]);
#pragma unroll
      for (int d = 0; d < 32; ++d)
#pragma unroll
        for (int g = 0; g < 8; ++g) acc[g] = fmaf(v[d], qs[g][dg * 32 + d], acc[g]);
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) part[dg][c][g] = acc[g];
    __syncthreads();
    if (dg != 0 || j >= a.r) return;
    __nv_bfloat16* out = a.qhat + ((size_t)(b * a.Hkv + h) * kPairQRows) * a.r + j;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const float x = part[0][c][g] + part[1][c][g] + part[2][c][g] + part[3][c][g];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      out[(size_t)g * a.r] = hi;
      out[(size_t)(8 + g) * a.r] = lo;
    }
    return;
  }
  // One CTA per (sequence, KV head). An entry is taken when it lies in range, is above its
  // predecessor in the list and above every taken entry before it; the largest taken entry
  // before position k equals the largest in-range, in-order entry before k, so both the
  // test and the output positions are prefix scans (max and count) over the list.
  __shared__ int w_max[8], w_cnt[8];
  __shared__ int s_bits;
  const int q = bid - n_w1 - n_q;
  const int h = q % a.Hkv, b = q / a.Hkv;
  const int* l = blocks + ((size_t)b * a.Hkv + h) * n_sel;
  int* out = a.sched + ((size_t)b * a.Hkv + h) * a.sched_stride;
  const int lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_bits = 0;
  __syncthreads();
  int carry_max = -1, carry_n = 0, bits = 0;
  for (int k0 = 0; k0 < n_sel; k0 += 256) {
    const int k = k0 + tid;
    int v = -1;
    bool elig = false;
    if (k < n_sel) {
      v = l[k];
      const bool bad_range = v < 0 || v >= a.nblk;
      const bool bad_order = k > 0 && l[k - 1] >= v;
      if (bad_range) bits |= LR_DEVERR_BLOCK_RANGE;
      if (bad_order) bits |= LR_DEVERR_BLOCK_ORDER;
      elig = !bad_range && !bad_order;
    }
    // inclusive prefix max of eligible values within the warp, then across warps
    int mx = elig ? v : -1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, mx, o);
      if (lane >= o) mx = max(mx, y);
    }
    if (lane == 31) w_max[warp] = mx;
    __syncthreads();
    int before_max = carry_max;  // largest eligible value before this entry
    for (int w = 0; w < warp; ++w) before_max = max(before_max, w_max[w]);
    const int prev_lane = __shfl_up_sync(0xffffffffu, mx, 1);
    if (lane > 0) before_max = max(before_max, prev_lane);
    const bool take = elig && v > before_max;
    // exclusive prefix count of taken entries
    const unsigned bal = __ballot_sync(0xffffffffu, take);
    if (lane == 0) w_cnt[warp] = __popc(bal);
    __syncthreads();
    int pos = carry_n + __popc(bal & ((1u << lane) - 1u)), chunk_n = 0, chunk_max = carry_max;
    for (int w = 0; w < 8; ++w) {
      if (w < warp) pos += w_cnt[w];
      chunk_n += w_cnt[w];
      chunk_max = max(chunk_max, w_max[w]);
    }
    if (take) out[1 + pos] = v;
    carry_n += chunk_n;
    carry_max = chunk_max;
    __syncthreads();  // w_max / w_cnt are rewritten by the next chunk
  }
  if (bits) atomicOr(&s_bits, bits);
  __syncthreads();
  if (tid == 0) {
    out[0] = carry_n;
    if (s_bits) flag_error(a.err, s_bits);
  }
}

template <int MG, bool Q2>
cudaError_t launch_pair_mg(const PairArgs& a, const CUtensorMap& mA, const CUtensorMap& mB0, const CUtensorMap& mB1,
                           const CUtensorMap& mQ, const CUtensorMap& mW1, const int* blocks, int n_sel,
                           cudaStream_t st) {
  const size_t n_w1_vec = (size_t)a.w1_seqs * a.Hkv * a.H * kHd / 4;
  const int n_w1 = (int)((n_w1_vec + 255) / 256 < 512 ? (n_w1_vec + 255) / 256 : 512);
  const int n_q = ((a.r + 63) / 64) * a.Hkv * a.B;
  const int n_s = a.sched ? a.Hkv * a.B : 0;
  // both kernels may be launched while the previous grid drains; each waits for it
  // (griddepcontrol.wait) before it reads anything that grid writes
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_w1 + n_q + n_s);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_pair_prep_kernel, a, n_w1, n_q, blocks, n_sel);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_pair_kernel<MG, Q2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout::kSmemBytes);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(2 * a.n_pairs, a.Hkv, a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Layout::kSmemBytes;
  e = cudaLaunchKernelEx(&cfg, decode_pair_kernel<MG, Q2>, mA, mB0, mB1, mQ, mW1, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int pair_max_clusters() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev]) return cached[dev];
  if (cudaFuncSetAttribute(decode_pair_kernel<8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout::kSmemBytes) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Layout::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_pair_kernel<8, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cached[dev] = n;
  return n;
}

cudaError_t launch_decode_pair(const PairArgs& a, const CUtensorMap& mA, const CUtensorMap& mB0,
                               const CUtensorMap& mB1, const CUtensorMap& mQ, const CUtensorMap& mW1,
                               const int* blocks, int n_sel, cudaStream_t st) {
  if (a.res_codes)
    return a.G <= 4 ? launch_pair_mg<4, true>(a, mA, mB0, mB1, mQ, mW1, blocks, n_sel, st)
                    : launch_pair_mg<8, true>(a, mA, mB0, mB1, mQ, mW1, blocks, n_sel, st);
  return a.G <= 4 ? launch_pair_mg<4, false>(a, mA, mB0, mB1, mQ, mW1, blocks, n_sel, st)
                  : launch_pair_mg<8, false>(a, mA, mB0, mB1, mQ, mW1, blocks, n_sel, st);
}

}  // namespace tc
}  // namespace lr
