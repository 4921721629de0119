// Single-CTA tensor-core decode over the compressed cache (bf16 cache, head_dim 128,
// sm_100a). The CTA-pair kernel (decode_pair.cu) is the default path for these shapes;
// this one is the fallback (LOWRAM_DECODE_PATH=tensor), kept under the same parity tests.
//
// One CTA owns (split, KV-head pair, sequence) and walks 128-token tiles (two
// 64-token blocks: consecutive blocks in full mode, entries of the pair's
// selected-block union in selective mode). Per tile:
//   MMA1  S1[128 x 256] = A_tile[128 x r] . [B_l^a | B_l^b]^T   keys of both heads
//                                            ("LowRAM" project page, Figure 3)
//         SC[128 x 4G]  = A_tile . Qhat^T    scores q.k~ = A . (B_l^h q) for both heads,
//                                            Qhat split into bf16 hi + lo rows
//   epilogue  k~ -> fp16 tile in shared memory; online softmax -> p (fp16 tile)
//   MMA2  U[128 x 128]  = k~ . W1_half^T     GELU-branch input, per 128 hidden units
//   epilogue  g = GELU(U + b1) (fp32) -> fp16 tile  ("Predicting the value cache from keys",
//                                            paragraphs 2-3)
//   MMA3  O3 = g^T . p, k~^T . p             p-weighted sums per dim, fp32 in TMEM
//   epilogue  merge O3 into register accumulators with the softmax rescale and add
//             p r over the tile's residual rows (paragraph 2)
// The second-stage operands (k~, g, p and W1) are fp16: 11 significant bits keep the
// rebuilt values within the attention tolerance even when one token dominates.
// Roles: warp 0 issues TMA loads into a 3-stage ring (A, B_l and Qhat chunks of 64
// rank columns, then W1 halves), warp 1 issues the MMAs, warps 2-9 run the epilogue
// (two groups of four splitting the columns), warp 10 scatters the residual rows.
// A prep kernel converts the layer's W1 to fp16, forms Qhat and (selective mode)
// merges each pair's block lists. The split partials (m, l, sum p k~, sum p g,
// sum p r) go to the same combine kernel as the general path. Every wait is bounded:
// on a timeout the CTA records LR_DEVERR_TIMEOUT, drains what it issued and returns.
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
constexpr int kChunk = 64;  // rank columns per ring stage
constexpr int kStages = 3;
constexpr int kThreads = 352;  // warp 0 TMA, 1 MMA, 2-9 epilogue (two groups of 4), 10 residual rows
constexpr int kEpi = 256;      // epilogue threads
constexpr int kGrp = 128;      // threads of one epilogue group (one TMEM lane quarter per warp)

constexpr uint32_t kColS1 = 0;    // keys of both heads, fp32, 256 columns
constexpr uint32_t kColU = 256;   // GELU-branch input of one 128-unit half
constexpr uint32_t kColO3 = 384;  // per head slot: [sum p k~ | sum p g half0 | half1], 16 columns each
constexpr uint32_t kColSC = 480;  // scores, hi and lo parts
constexpr uint32_t kTmemCols = 512;

template <int MG>
struct Layout {
  static constexpr uint32_t kQRows = 4 * MG;                  // Qhat rows: 2 heads x (hi, lo) x MG
  static constexpr uint32_t kQBytes = kQRows * 128;           // one 64-column chunk of Qhat
  static constexpr uint32_t kStageBytes = 49152 + kQBytes;    // A 16 KB, B_l 32 KB, Qhat
  static constexpr uint32_t kOffRing = 0;
  static constexpr uint32_t kOffKt = (kStages * kStageBytes + 1023) & ~1023u;  // key tile of one head
  static constexpr uint32_t kOffG = kOffKt + 32768;
  static constexpr uint32_t kOffP = kOffG + 32768;
  static constexpr uint32_t kOffB1 = kOffP + 4096;      // fp16 b1 of both heads (1 KB)
  static constexpr uint32_t kOffRed = kOffB1 + 1024;    // 4 warps x 16 floats
  static constexpr uint32_t kOffAlpha = kOffRed + 256;  // [tile parity][head slot][8] softmax rescale
  static constexpr uint32_t kOffBar = kOffAlpha + 128;
  static constexpr uint32_t kOffMisc = kOffBar + 256;
  static constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
};
static_assert(Layout<8>::kSmemBytes <= 232448, "shared memory budget");

enum Bar {
  FULL0 = 0, EMPTY0 = kStages, S1_FULL = 2 * kStages, S1_FREE, KT_READY, KT_FREE, U_FULL, U_FREE, G_READY,
  G_FREE, O3_FULL0, O3_FULL1, O3_FREE0, O3_FREE1, EPI_SYNC, RES_READY, RES_DONE, DRAIN, N_BARS
};
static_assert(N_BARS * 8 <= 256, "barrier area");

// GELU(x) = x Phi(x) with Phi(x) ~ (1 + tanh(x (c1 + c3 x^2))) / 2 in fp32 with the
// hardware tanh; c1, c3 are a minimax fit to the exact erf form (max abs error 2.7e-4 in
// exact arithmetic; csrc/gelu_fit.py reproduces them). The fp32 form runs at about twice
// the rate of the same formula on fp16x2 pairs, whose tanh is the slower one.
constexpr float kGeluC1 = 0.80015708f;
constexpr float kGeluC3 = 0.03470089f;

__device__ __forceinline__ float gelu_f32(float x) {
  const float z = x * fmaf(kGeluC3, x * x, kGeluC1);
  const float h = 0.5f * x;
  return fmaf(h, tanh_fast(z), h);
}

// GELU of two fp32 pre-activations plus their fp16 biases, packed to fp16x2.
__device__ __forceinline__ uint32_t gelu_pair(uint32_t u0, uint32_t u1, uint32_t bias_h2) {
  const float2 bf = __half22float2(*reinterpret_cast<const __half2*>(&bias_h2));
  return pack_f16x2_sat(gelu_f32(__uint_as_float(u0) + bf.x), gelu_f32(__uint_as_float(u1) + bf.y));
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct TileInfo {
  int blk[2];
  int mask[2];
};

__device__ __forceinline__ int tile_count(const TcArgs& a, int b, int hp) {
  if (!a.sched) return (a.nblk + 1) >> 1;
  return (a.sched[((size_t)b * a.n_hp + hp) * a.sched_stride] + 1) >> 1;
}

__device__ __forceinline__ TileInfo tile_info(const TcArgs& a, int b, int hp, int i) {
  TileInfo t;
  if (!a.sched) {
    t.blk[0] = 2 * i;
    t.blk[1] = 2 * i + 1 < a.nblk ? 2 * i + 1 : -1;
    t.mask[0] = 3;
    t.mask[1] = t.blk[1] >= 0 ? 3 : 0;
    return t;
  }
  const int* s = a.sched + ((size_t)b * a.n_hp + hp) * a.sched_stride;
  const int n = s[0];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e = 2 * i + h;
    if (e < n) {
      const int v = s[1 + e];
      t.blk[h] = v & 0x0FFFFFFF;
      t.mask[h] = (v >> 28) & 3;
    } else {
      t.blk[h] = -1;
      t.mask[h] = 0;
    }
  }
  return t;
}

__device__ __forceinline__ int lower_bound_i32(const int* p, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// byte offset of element (row, col) of a 128-byte-swizzled 16-bit tile whose 64-column
// atoms are `atom_bytes` apart
__device__ __forceinline__ uint32_t sw128_off(int row, int col, uint32_t atom_bytes) {
  const int a = col >> 6, c = col & 63;
  return a * atom_bytes + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + ((c & 7) << 1);
}

// Epilogue-side wait: every lane polls, and the outcome is made uniform across the
// warp so that a timeout never leaves part of a warp inside a collective.
__device__ __forceinline__ bool ewait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

template <int MG>
struct Epi {
  const TcArgs& a;
  uint8_t* sm;
  uint64_t* bars;
  volatile int* abort_flag;
  int grp, wl, lane, row;
  uint32_t trow;
  uint32_t sync_phase;
  // group 0: softmax state and sum p k~; group 1: sum p g
  float m[2][MG], l[2][MG], ak[2][MG], ag0[2][MG], ag1[2][MG];
  float alpha[2][MG];

  __device__ Epi(const TcArgs& a_, uint8_t* sm_, uint64_t* bars_, volatile int* ab, int warp, int lane_, uint32_t tmem)
      : a(a_), sm(sm_), bars(bars_), abort_flag(ab) {
    grp = (warp - 2) >> 2;
    wl = (warp - 2) & 3;
    lane = lane_;
    const int lq = warp & 3;
    row = lq * 32 + lane;
    trow = tmem + ((uint32_t)(lq * 32) << 16);
    sync_phase = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        m[h][g] = -CUDART_INF_F;
        l[h][g] = ak[h][g] = ag0[h][g] = ag1[h][g] = 0.f;
        alpha[h][g] = 1.f;
      }
  }

  __device__ __forceinline__ bool sync0() {  // barrier over epilogue group 0
    mbar_arrive(&bars[EPI_SYNC]);
    const bool ok = ewait(&bars[EPI_SYNC], sync_phase & 1, abort_flag);
    ++sync_phase;
    return ok;
  }

  // Softmax of head slot HX on tile `tl` (group 0): scores -> p tile, alphas, KT_READY.
  template <int HX>
  __device__ __forceinline__ bool softmax(int tl, const float (&sc_in)[MG], bool hv) {
    using L = Layout<MG>;
    float* red = reinterpret_cast<float*>(sm + L::kOffRed);
    uint8_t* ptile = sm + L::kOffP;
    float sc[MG];
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      sc[g] = hv ? sc_in[g] : -CUDART_INF_F;
      const float mx = warp_max(sc[g]);
      if (lane == 0) red[wl * 16 + g] = mx;
    }
    if (!sync0()) return false;
    float p[MG];
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      const float mt = fmaxf(fmaxf(red[g], red[16 + g]), fmaxf(red[32 + g], red[48 + g]));
      const float m_new = fmaxf(m[HX][g], mt);
      alpha[HX][g] = m_new == -CUDART_INF_F ? 1.f : __expf(m[HX][g] - m_new);
      p[g] = hv ? __expf(sc[g] - m_new) : 0.f;
      l[HX][g] = l[HX][g] * alpha[HX][g] + p[g];
      m[HX][g] = m_new;
    }
    // the p tile is free: the previous head's MMA3 (KT_FREE, waited before the key drain)
    // and the residual warp are done with it
    const int n_res = 2 * tl + HX;
    if (n_res > 0 && !ewait(&bars[RES_DONE], (n_res - 1) & 1, abort_flag)) return false;
#pragma unroll
    for (int g = 0; g < MG; ++g)
      if (g < a.G) *reinterpret_cast<__half*>(ptile + sw128_off(g, row, 2048)) = __float2half_rn(p[g]);
    if (row == 0) {
      float* al = reinterpret_cast<float*>(sm + L::kOffAlpha) + ((tl & 1) * 2 + HX) * 8;
#pragma unroll
      for (int g = 0; g < MG; ++g) al[g] = alpha[HX][g];
    }
    fence_proxy_async_smem();
    if (!sync0()) return false;  // p tile and alphas complete; red consumed
    mbar_arrive(&bars[KT_READY]);
    if (row == 0) mbar_arrive(&bars[RES_READY]);
    return true;
  }

  // GELU branch of head slot HX on tile `tl`: this group's 64 of every 128 hidden units.
  template <int HX>
  __device__ __forceinline__ bool gelu(int tl) {
    using L = Layout<MG>;
    const int nh = a.H / 128;
    const uint4* b1h = reinterpret_cast<const uint4*>(sm + L::kOffB1 + HX * 512);
    uint8_t* gtile = sm + L::kOffG;
#pragma unroll 1
    for (int half = 0; half < nh; ++half) {
      const int j = (tl * 2 + HX) * nh + half;
      if (!ewait(&bars[U_FULL], j & 1, abort_flag)) return false;
      tc_fence_after();
      uint32_t u[2][32];
      tmem_ld32(trow + kColU + grp * 64, u[0]);
      tmem_ld32(trow + kColU + grp * 64 + 32, u[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars[U_FREE]);
      if (j > 0 && !ewait(&bars[G_FREE], (j - 1) & 1, abort_flag)) return false;
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
      mbar_arrive(&bars[G_READY]);
    }
    return true;
  }

  // Merge the tile's p-weighted sums of head slot HX into the running accumulators.
  template <int HX>
  __device__ __forceinline__ bool merge(int tl) {
    using L = Layout<MG>;
    if (!ewait(&bars[O3_FULL0 + HX], tl & 1, abort_flag)) return false;
    tc_fence_after();
    uint32_t v0[8], v1[8];
    if (grp == 0) {
      tmem_ld8(trow + kColO3 + HX * 48, v0);
    } else {
      tmem_ld8(trow + kColO3 + HX * 48 + 16, v0);
      tmem_ld8(trow + kColO3 + HX * 48 + 32, v1);
    }
    tmem_ld_wait();
    tc_fence_before();
    mbar_arrive(&bars[O3_FREE0 + HX]);
    if (grp == 0) {
#pragma unroll
      for (int g = 0; g < MG; ++g) ak[HX][g] = fmaf(ak[HX][g], alpha[HX][g], __uint_as_float(v0[g]));
    } else {
      // acquire group 0's alphas of this head (that phase has completed; the wait is immediate)
      if (!ewait(&bars[KT_READY], (2 * tl + HX) & 1, abort_flag)) return false;
      const float* al = reinterpret_cast<const float*>(sm + L::kOffAlpha) + ((tl & 1) * 2 + HX) * 8;
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        const float alg = al[g];
        ag0[HX][g] = fmaf(ag0[HX][g], alg, __uint_as_float(v0[g]));
        ag1[HX][g] = fmaf(ag1[HX][g], alg, __uint_as_float(v1[g]));
      }
    }
    return true;
  }

  // Drain this group's 64 key columns of head slot HX into the fp16 key tile.
  template <int HX>
  __device__ __forceinline__ void drain() {
    using L = Layout<MG>;
    uint8_t* kt = sm + L::kOffKt;
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t v[32];
      tmem_ld32(trow + kColS1 + HX * 128 + grp * 64 + cc * 32, v);
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
  }

  // One tile: for each head slot, drain its keys, then softmax, GELU branch and merge.
  // The key tile is single-buffered: slot 1's keys stay in TMEM until slot 0 is done.
  __device__ __forceinline__ bool tile(int tl, const TileInfo& t) {
    const int half_row = row >> 6;
    const int rblk = half_row ? t.blk[1] : t.blk[0];
    const int tok = rblk * kBlock + (row & 63);
    const bool row_valid = rblk >= 0 && tok < a.T;
    const int rmask = half_row ? t.mask[1] : t.mask[0];
    if (!ewait(&bars[S1_FULL], tl & 1, abort_flag)) return false;
    tc_fence_after();
    float sc[2][MG];
    if (grp == 0) {  // scores of both heads (hi + lo columns)
      uint32_t sv[32];
      if constexpr (MG == 4) {
        uint32_t t8[8];
        tmem_ld8(trow + kColSC, t8);
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[i] = t8[i];
        tmem_ld8(trow + kColSC + 8, t8);
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[16 + i] = t8[i];
      } else {
        tmem_ld32(trow + kColSC, sv);
      }
      tmem_ld_wait();
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        sc[0][g] = __uint_as_float(sv[g]) + __uint_as_float(sv[MG + g]);
        sc[1][g] = MG == 4 ? __uint_as_float(sv[16 + g]) + __uint_as_float(sv[16 + MG + g])
                           : __uint_as_float(sv[2 * MG + g]) + __uint_as_float(sv[3 * MG + g]);
      }
    }
    const bool hv0 = row_valid && (rmask & 1), hv1 = row_valid && ((rmask >> 1) & 1);
    // ---- head slot 0
    if (tl > 0 && !ewait(&bars[KT_FREE], (2 * tl - 1) & 1, abort_flag)) return false;
    drain<0>();
    fence_proxy_async_smem();
    if (grp == 1) mbar_arrive(&bars[KT_READY]);
    if (grp == 0 && !softmax<0>(tl, sc[0], hv0)) return false;
    if (!gelu<0>(tl)) return false;
    if (!merge<0>(tl)) return false;
    // ---- head slot 1 (its keys leave TMEM now, which frees S1 for the next tile)
    if (!ewait(&bars[KT_FREE], (2 * tl) & 1, abort_flag)) return false;
    drain<1>();
    tc_fence_before();
    mbar_arrive(&bars[S1_FREE]);
    fence_proxy_async_smem();
    if (grp == 1) mbar_arrive(&bars[KT_READY]);
    if (grp == 0 && !softmax<1>(tl, sc[1], hv1)) return false;
    if (!gelu<1>(tl)) return false;
    if (!merge<1>(tl)) return false;
    return true;
  }

  __device__ __forceinline__ void write_partials(int b, int split, int ha) {
    using L = Layout<MG>;
    float* red = reinterpret_cast<float*>(sm + L::kOffRed);
    const int Hq = a.Hkv * a.G;
    if (grp == 0) {
      sync0();  // red is free
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        const float v0 = warp_sum(l[0][g]);
        const float v1 = warp_sum(l[1][g]);
        if (lane == 0) {
          red[wl * 16 + g] = v0;
          red[wl * 16 + 8 + g] = v1;
        }
      }
      sync0();
    }
#pragma unroll
    for (int hx = 0; hx < 2; ++hx) {
#pragma unroll
      for (int g = 0; g < MG; ++g) {
        if (g >= a.G) continue;
        const int hq = (ha + hx) * a.G + g;
        float* part = a.partials + (((size_t)b * Hq + hq) * a.n_split + split) * a.part_stride;
        if (grp == 0) {
          if (row == 0) {
            part[0] = m[hx][g];
            part[1] = red[hx * 8 + g] + red[16 + hx * 8 + g] + red[32 + hx * 8 + g] + red[48 + hx * 8 + g];
            part[2] = part[3] = 0.f;
          }
          part[4 + row] = ak[hx][g];
        } else {
          part[4 + kHd + row] = ag0[hx][g];
          if (a.H == 256) part[4 + kHd + 128 + row] = ag1[hx][g];
        }
      }
    }
  }
};

// The residual warp: for each (tile, head) it scatters p_t r_t over the residual rows of the
// tile's blocks ("Predicting the value cache from keys", paragraph 2). Lane l owns dims
// 4l .. 4l+3; the rows of a block are contiguous in res_val (indices ascending), so a batch
// of 16 rows is one coalesced 256-byte read per row. Loads are issued before waiting for
// the epilogue's p tile, so their latency overlaps the softmax.
template <int MG>
__device__ __forceinline__ void residual_warp(const TcArgs& a, uint8_t* sm, uint64_t* bars, volatile int* abort_flag,
                                              int b, int hp, int split, int t_begin, int t_end) {
  using L = Layout<MG>;
  const int lane = threadIdx.x & 31, ha = 2 * hp, G = a.G;
  const uint8_t* ptile = sm + L::kOffP;
  const float* alphas = reinterpret_cast<const float*>(sm + L::kOffAlpha);
  float acc[2][MG][4];
#pragma unroll
  for (int hx = 0; hx < 2; ++hx)
#pragma unroll
    for (int g = 0; g < MG; ++g)
#pragma unroll
      for (int d = 0; d < 4; ++d) acc[hx][g][d] = 0.f;
  int bad = 0;
  bool ok = true;
  int tl = 0;
  const size_t pseg = ((size_t)b * a.L + a.layer) * a.Hkv + ha;
  for (int ti = t_begin; ti < t_end && ok; ++ti, ++tl) {
    const TileInfo t = tile_info(a, b, hp, ti);
#pragma unroll
    for (int hx = 0; hx < 2; ++hx) {
      if (!ok) break;
      const int n_kt = 2 * tl + hx;
      int e0[2] = {0, 0}, ne[2] = {0, 0}, lo[2] = {0, 0}, hi[2] = {0, 0};
      const int* ridx = nullptr;
      const __nv_bfloat16* rval = nullptr;
      if (a.k > 0) {
        const size_t seg = pseg + hx;
        ridx = a.res_idx + seg * a.k;
        rval = a.res_val + seg * a.k * kHd;
        const int* rptr = a.res_ptr ? a.res_ptr + seg * (a.nblk + 1) : nullptr;
#pragma unroll
        for (int bh = 0; bh < 2; ++bh) {
          const int blk = t.blk[bh];
          if (blk < 0 || !((t.mask[bh] >> hx) & 1)) continue;
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
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int i = i0 + j;
          const int bh = i < ne[0] ? 0 : 1;
          const int e = bh ? e0[1] + (i - ne[0]) : e0[0] + i;
          const bool in = i < n_tot;
          bh_of[j] = bh;
          tr[j] = in ? __ldg(ridx + e) : -1;
          rv[j] = in ? __ldg(reinterpret_cast<const uint2*>(rval + (size_t)e * kHd) + lane) : make_uint2(0, 0);
        }
        if (!waited) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[RES_READY], n_kt & 1, abort_flag)))) break;
          waited = true;
#pragma unroll
          for (int g = 0; g < MG; ++g) {
            const float al = alphas[((tl & 1) * 2 + hx) * 8 + g];
#pragma unroll
            for (int d = 0; d < 4; ++d) acc[hx][g][d] *= al;
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
          const __nv_bfloat162 r01 = *reinterpret_cast<const __nv_bfloat162*>(&rv[j].x);
          const __nv_bfloat162 r23 = *reinterpret_cast<const __nv_bfloat162*>(&rv[j].y);
          const float r0 = __low2float(r01), r1 = __high2float(r01), r2 = __low2float(r23), r3 = __high2float(r23);
#pragma unroll
          for (int g = 0; g < MG; ++g) {
            if (g < G) {
              const float pg = __half2float(*reinterpret_cast<const __half*>(ptile + sw128_off(g, prow, 2048)));
              acc[hx][g][0] = fmaf(pg, r0, acc[hx][g][0]);
              acc[hx][g][1] = fmaf(pg, r1, acc[hx][g][1]);
              acc[hx][g][2] = fmaf(pg, r2, acc[hx][g][2]);
              acc[hx][g][3] = fmaf(pg, r3, acc[hx][g][3]);
            }
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[RES_DONE]);
    }
  }
  if (!ok) {
    *abort_flag = 1;
    flag_error(a.err, LR_DEVERR_TIMEOUT);
  }
  if (bad && lane == 0) flag_error(a.err, bad);
  const int Hq = a.Hkv * G;
#pragma unroll
  for (int hx = 0; hx < 2; ++hx) {
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      if (g >= G) continue;
      float* part = a.partials + (((size_t)b * Hq + (ha + hx) * G + g) * a.n_split + split) * a.part_stride;
      *reinterpret_cast<float4*>(part + 4 + kHd + a.H + 4 * lane) =
          make_float4(acc[hx][g][0], acc[hx][g][1], acc[hx][g][2], acc[hx][g][3]);
    }
  }
}

template <int MG>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapW1,
                 const TcArgs a) {
  using L = Layout<MG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffMisc + 4);

  const int s = blockIdx.x, hp = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H, nh = a.H / 128, nk = a.r / kChunk, nw = 2 * nh;
  const int ha = 2 * hp;  // first KV head of the pair

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[FULL0 + i], 1);
      mbar_init(&bars[EMPTY0 + i], 1);
    }
    mbar_init(&bars[S1_FULL], 1);
    mbar_init(&bars[S1_FREE], kEpi);
    mbar_init(&bars[KT_READY], kEpi);
    mbar_init(&bars[KT_FREE], 1);
    mbar_init(&bars[U_FULL], 1);
    mbar_init(&bars[U_FREE], kEpi);
    mbar_init(&bars[G_READY], kEpi);
    mbar_init(&bars[G_FREE], 1);
    mbar_init(&bars[O3_FULL0], 1);
    mbar_init(&bars[O3_FULL1], 1);
    mbar_init(&bars[O3_FREE0], kEpi);
    mbar_init(&bars[O3_FREE1], kEpi);
    mbar_init(&bars[EPI_SYNC], kGrp);
    mbar_init(&bars[RES_READY], 1);
    mbar_init(&bars[RES_DONE], 1);
    mbar_init(&bars[DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapW1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  {  // b1 of both heads as fp16, zero p tile
    __half* b1s = reinterpret_cast<__half*>(sm + L::kOffB1);
    const size_t pseq = a.pred_per_seq ? (size_t)b : 0;
    for (int i = threadIdx.x; i < 2 * 256; i += kThreads) {
      const int hx = i / 256, c = i % 256;
      b1s[i] = __float2half_rn(
          c < H ? __bfloat162float(a.b1[((pseq * a.L + a.layer) * a.Hkv + ha + hx) * H + c]) : 0.f);
    }
    uint32_t* pz = reinterpret_cast<uint32_t*>(sm + L::kOffP);
    for (int i = threadIdx.x; i < 1024; i += kThreads) pz[i] = 0u;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // The setup above overlaps the end of the prep grid (programmatic dependent launch);
  // its outputs (schedule, Qhat, fp16 W1) are read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_tiles = tile_count(a, b, hp);
  const int t_begin = (int)((long long)s * n_tiles / a.n_split);
  const int t_end = (int)((long long)(s + 1) * n_tiles / a.n_split);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      const int rowB = (a.layer * a.Hkv + ha) * kHd;
      const int rowQ = (b * a.n_hp + hp) * (int)L::kQRows;
      const int w1seq = a.pred_per_seq ? b : 0;
      for (int ti = t_begin; ti < t_end && ok; ++ti) {
        const TileInfo t = tile_info(a, b, hp, ti);
        const int row0 = t.blk[0] >= 0 ? t.blk[0] * kBlock : a.T;
        const int row1 = t.blk[1] >= 0 ? t.blk[1] * kBlock : a.T;
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait(&bars[EMPTY0 + st], ph ^ 1, abort_flag))) break;
          uint8_t* dst = sm + L::kOffRing + st * L::kStageBytes;
          mbar_arrive_expect_tx(&bars[FULL0 + st], L::kStageBytes);
          tma_load_3d(dst, &mapA, &bars[FULL0 + st], kc * kChunk, row0, b);
          tma_load_3d(dst + 8192, &mapA, &bars[FULL0 + st], kc * kChunk, row1, b);
          tma_load_3d(dst + 16384, &mapB, &bars[FULL0 + st], kc * kChunk, rowB, b);
          tma_load_3d(dst + 32768, &mapB, &bars[FULL0 + st], kc * kChunk, rowB + kHd, b);
          tma_load_2d(dst + 49152, &mapQ, &bars[FULL0 + st], kc * kChunk, rowQ);
        }
        for (int j = 0; j < nw && ok; ++j, ++it) {
          const int hx = j / nh, half = j % nh;
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait(&bars[EMPTY0 + st], ph ^ 1, abort_flag))) break;
          uint8_t* dst = sm + L::kOffRing + st * L::kStageBytes;
          const int wrow = ((w1seq * a.Hkv + ha + hx) * H) + half * 128;
          mbar_arrive_expect_tx(&bars[FULL0 + st], 32768);
          tma_load_2d(dst, &mapW1, &bars[FULL0 + st], 0, wrow);
          tma_load_2d(dst + 16384, &mapW1, &bars[FULL0 + st], 64, wrow);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(a.err, LR_DEVERR_TIMEOUT);
      }
      // drain: every load issued has landed before the CTA may exit
      for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait_drain(&bars[FULL0 + j % kStages], (j / kStages) & 1, kWaitCycles / 4);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s1 = idesc_bf16_f32(128, 256, false, false);
      const uint32_t id_sc = idesc_bf16_f32(128, L::kQRows, false, false);
      const uint32_t id_u = idesc_f16_f32(128, 128, false, false);
      const uint32_t id_o3 = idesc_f16_f32(128, 16, true, false);
      const uint32_t kt = smem_u32(sm + L::kOffKt), gt = smem_u32(sm + L::kOffG), pt = smem_u32(sm + L::kOffP);
      uint32_t it = 0;
      bool ok = true;
      int tl = 0;
      for (int ti = t_begin; ti < t_end && ok; ++ti, ++tl) {
        if (!(ok = mbar_wait(&bars[S1_FREE], (tl & 1) ^ 1, abort_flag))) break;
        tc_fence_after();
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait(&bars[FULL0 + st], ph, abort_flag))) break;
          tc_fence_after();
          const uint32_t base = smem_u32(sm + L::kOffRing + st * L::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t adesc = sw128_desc(base + ks * 32, 16, 1024);
            mma_f16_ss(tmem + kColS1, adesc, sw128_desc(base + 16384 + ks * 32, 16, 1024), id_s1, (kc | ks) != 0);
            mma_f16_ss(tmem + kColSC, adesc, sw128_desc(base + 49152 + ks * 32, 16, 1024), id_sc, (kc | ks) != 0);
          }
          mma_commit(&bars[EMPTY0 + st]);
        }
        if (!ok) break;
        mma_commit(&bars[S1_FULL]);
        for (int hx = 0; hx < 2 && ok; ++hx) {
          const int n_kt = 2 * tl + hx;
          if (!(ok = mbar_wait(&bars[KT_READY], n_kt & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&bars[O3_FREE0 + hx], (tl & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          // sum p k~ needs only the key and p tiles: issue it ahead of the GELU branch
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_f16_ss(tmem + kColO3 + hx * 48, sw128_desc(kt + ks * 2048, 16384, 1024),
                       sw128_desc(pt + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024), id_o3, ks != 0);
          for (int half = 0; half < nh && ok; ++half, ++it) {
            const int j = n_kt * nh + half;
            const uint32_t st = it % kStages, ph = (it / kStages) & 1;
            if (!(ok = mbar_wait(&bars[FULL0 + st], ph, abort_flag))) break;
            if (!(ok = mbar_wait(&bars[U_FREE], (j & 1) ^ 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t wb = smem_u32(sm + L::kOffRing + st * L::kStageBytes);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
              mma_f16_ss(tmem + kColU, sw128_desc(kt + off, 16, 1024), sw128_desc(wb + off, 16, 1024), id_u,
                         ks != 0);
            }
            mma_commit(&bars[EMPTY0 + st]);
            mma_commit(&bars[U_FULL]);
          }
          for (int half = 0; half < nh && ok; ++half) {
            const int j = n_kt * nh + half;
            if (!(ok = mbar_wait(&bars[G_READY], j & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_f16_ss(tmem + kColO3 + hx * 48 + 16 + half * 16, sw128_desc(gt + ks * 2048, 16384, 1024),
                         sw128_desc(pt + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024), id_o3, ks != 0);
            mma_commit(&bars[G_FREE]);
          }
          if (!ok) break;
          mma_commit(&bars[KT_FREE]);
          mma_commit(&bars[O3_FULL0 + hx]);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_error(a.err, LR_DEVERR_TIMEOUT);
      }
      // every MMA issued has completed before TMEM is released
      mma_commit(&bars[DRAIN]);
      mbar_wait_drain(&bars[DRAIN], 0, kWaitCycles / 4);
    }
  } else if (warp == 10) {
    // ---------------------------------------------------------------- residual rows
    residual_warp<MG>(a, sm, bars, abort_flag, b, hp, s, t_begin, t_end);
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-9)
    Epi<MG> e(a, sm, bars, abort_flag, warp, lane, tmem);
    bool ok = true;
    for (int i = 0; t_begin + i < t_end && ok; ++i) ok = e.tile(i, tile_info(a, b, hp, t_begin + i));
    if (!ok) {
      *abort_flag = 1;
      flag_error(a.err, LR_DEVERR_TIMEOUT);
    }
    e.write_partials(b, s, ha);
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Prep work of one decode call, one launch:
//   blocks [0, n_w1)             the layer's W1 as fp16 (bf16 -> fp16 is exact except below
//                                2^-14 or above 65504, where values saturate)
//   blocks [n_w1, n_w1 + n_q)    Qhat = scale * B_l^h q for every query head, stored as bf16
//                                hi + lo rows (hi = bf16(x), lo = bf16(x - hi)); one block per
//                                (64 rank columns, KV head, sequence)
//   blocks [n_w1 + n_q, ...)     selective mode: per (sequence, head pair) the union of the two
//                                block lists with a 2-bit head mask (bit 0: first head); entries
//                                out of range or not strictly ascending are skipped and flagged
template <int MG>
__global__ void __launch_bounds__(256) decode_tc_prep_kernel(TcArgs a, int n_w1, int n_q, const int* blocks,
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
    // one block per (64 rank columns, KV head, sequence): thread (dg, c) sums 32 of the 128
    // key dims for column c, all loads of a thread in flight at once; then a 4-way reduction
    __shared__ float qs[8][kHd];
    __shared__ float part[4][64][MG];
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
    float acc[MG];
#pragma unroll
    for (int g = 0; g < MG; ++g) acc[g] = 0.f;
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
        for (int g = 0; g < MG; ++g) acc[g] = fmaf(v[d], qs[g][dg * 32 + d], acc[g]);
    }
#pragma unroll
    for (int g = 0; g < MG; ++g) part[dg][c][g] = acc[g];
    __syncthreads();
    if (dg != 0 || j >= a.r) return;
    const int hp = h >> 1, hx = h & 1;
    __nv_bfloat16* out = a.qhat + ((size_t)(b * a.n_hp + hp) * (4 * MG) + hx * 2 * MG) * a.r + j;
#pragma unroll
    for (int g = 0; g < MG; ++g) {
      const float x = part[0][c][g] + part[1][c][g] + part[2][c][g] + part[3][c][g];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      out[(size_t)g * a.r] = hi;
      out[(size_t)(MG + g) * a.r] = lo;
    }
    return;
  }
  if (tid != 0) return;
  const int q = bid - n_w1 - n_q;
  const int hp = q % a.n_hp, b = q / a.n_hp;
  const int* la = blocks + ((size_t)b * a.Hkv + 2 * hp) * n_sel;
  const int* lb = la + n_sel;
  int* out = const_cast<int*>(a.sched) + ((size_t)b * a.n_hp + hp) * a.sched_stride;
  int i = 0, j = 0, n = 0, prev_a = -1, prev_b = -1, bits = 0;
  auto next = [&](const int* l, int& k, int& prev) -> int {
    while (k < n_sel) {
      const int v = l[k];
      const bool bad_range = v < 0 || v >= a.nblk;
      const bool bad_order = k > 0 && l[k - 1] >= v;
      if (bad_range) bits |= LR_DEVERR_BLOCK_RANGE;
      if (bad_order) bits |= LR_DEVERR_BLOCK_ORDER;
      if (!bad_range && !bad_order && v > prev) return v;
      ++k;
    }
    return -1;
  };
  int va = next(la, i, prev_a), vb = next(lb, j, prev_b);
  while (va >= 0 || vb >= 0) {
    int v, m;
    if (vb < 0 || (va >= 0 && va < vb)) { v = va; m = 1; prev_a = va; ++i; }
    else if (va < 0 || vb < va) { v = vb; m = 2; prev_b = vb; ++j; }
    else { v = va; m = 3; prev_a = va; prev_b = vb; ++i; ++j; }
    out[1 + n++] = v | (m << 28);
    va = next(la, i, prev_a);
    vb = next(lb, j, prev_b);
  }
  out[0] = n;
  if (bits) flag_error(a.err, bits);
}

template <int MG>
cudaError_t launch_mg(const TcArgs& a, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mQ,
                      const CUtensorMap& mW1, const int* blocks, int n_sel, cudaStream_t st) {
  const size_t n_w1_vec = (size_t)a.w1_seqs * a.Hkv * a.H * kHd / 4;
  const int n_w1 = (int)((n_w1_vec + 255) / 256 < 512 ? (n_w1_vec + 255) / 256 : 512);
  const int n_q = ((a.r + 63) / 64) * a.Hkv * a.B;
  const int n_s = a.sched ? a.n_hp * a.B : 0;
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_prep_kernel<MG>, a, n_w1, n_q, blocks, n_sel);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_tc_kernel<MG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Layout<MG>::kSmemBytes);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(a.n_split, a.n_hp, a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Layout<MG>::kSmemBytes;
  e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<MG>, mA, mB, mQ, mW1, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int qhat_rows(int G) { return G <= 4 ? 16 : 32; }

cudaError_t launch_decode_tc(const TcArgs& a, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mQ,
                             const CUtensorMap& mW1, const int* blocks, int n_sel, cudaStream_t st) {
  return a.G <= 4 ? launch_mg<4>(a, mA, mB, mQ, mW1, blocks, n_sel, st)
                  : launch_mg<8>(a, mA, mB, mQ, mW1, blocks, n_sel, st);
}

}  // namespace tc
}  // namespace lr
