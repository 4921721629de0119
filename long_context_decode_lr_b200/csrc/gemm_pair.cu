// Persistent tensor-core GEMM on CTA pairs (bf16 operands, fp32 accumulation, sm_100a):
//   C[b, m, n] = sum_k Aop[b, m, k] * Bop[b, n, k]
// Aop is K-major ([B, M, K], rows of K); Bop is K-major ([B, N, K]) or MN-major
// ([B, K, N], rows of N). The packer uses it for its two dense contractions:
//   projection  A  = K_group . Bt       (Bop = Bt read MN-major; "LowRAM" project page,
//                                        Figure 3: the shared per-token factor)
//   key rebuild K~ = A . Bt^T           (Bop = Bt read K-major: every layer and KV head of
//                                        the group at once, k~ = A . B_l^h)
// A 2-CTA cluster owns 256 x BN output tiles and walks them with a stride of the cluster
// count. CTA r holds rows 128 r .. 128 r + 127 of the A tile and half of the BN columns of
// the B tile; CTA 0 issues the tcgen05 MMAs for both (M = 256). Warp roles per CTA: warp 0
// streams A and B chunks of 64 along K through a ring with TMA (the bytes of both CTAs
// count on CTA 0's barrier); warp 1 allocates TMEM and (CTA 0) issues the MMAs into one of
// two accumulator buffers; warps 2-5 drain their CTA's 128 rows from TMEM, round them to
// the output type and store 32 x 64 tiles through shared memory with TMA, while the next
// tile accumulates in the other buffer. Every wait is bounded: a timeout raises the abort
// flag of both CTAs and sets LR_DEVERR_TIMEOUT in the error word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lr_common.cuh"
#include "lr_gemm.h"
#include "sm100.cuh"

namespace lr {
namespace tc {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRingBytes = 196608;     // operand ring (192 KB)
constexpr int kStageOutBytes = 4096;   // one 32 x 64 output tile (16-bit)

template <int BN, bool kBmn>
struct GemmLayout {
  static constexpr int kABytes = 128 * 64 * 2;           // this CTA's 128 rows x 64 K
  static constexpr int kBBytes = (BN / 2) * 64 * 2;      // this CTA's BN/2 columns x 64 K
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = kRingBytes / kStageBytes;
  static constexpr int kOffOut = kStages * kStageBytes;  // 4 warps x 2 output buffers
  static constexpr int kOffBar = kOffOut + 8 * kStageOutBytes;
  static constexpr int kOffMisc = kOffBar + 8 * (2 * kStages + 6);
  static constexpr int kSmemBytes = kOffMisc + 64;
  static constexpr uint32_t kTmemCols = 2 * BN;
};

enum GBar { G_FULL0 = 0 };  // FULL[s], EMPTY[s], then TFULL[2], TEMPTY[2], DRAIN, spare

template <int BN, bool kBmn>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                 const __grid_constant__ CUtensorMap mapC, const GemmArgs g) {
  using L = GemmLayout<BN, kBmn>;
  constexpr int S = L::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  if (smem_u32(sm) & 1023u) {
    if (threadIdx.x == 0) flag_error(g.err, LR_DEVERR_LAUNCH);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* FULL = bars;
  uint64_t* EMPTY = bars + S;
  uint64_t* TFULL = bars + 2 * S;
  uint64_t* TEMPTY = bars + 2 * S + 2;
  uint64_t* DRAIN = bars + 2 * S + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffMisc + 4);

  const uint32_t rank = cluster_cta_rank();
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (g.M + 255) / 256, nt = g.N / BN, nk = g.K / 64;
  const int n_tiles = g.B * mt * nt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&FULL[i], 1);
      mbar_init(&EMPTY[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&TFULL[i], 1);
      mbar_init(&TEMPTY[i], 8);  // one arrival per epilogue warp of both CTAs (CTA 0's copy)
    }
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
    tma_prefetch_desc(&mapC);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  auto tile_coords = [&](int t, int& b, int& m0, int& n0) {
    n0 = (t % nt) * BN;
    const int r = t / nt;
    m0 = (r % mt) * 256;
    b = r / mt;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = cluster; t < n_tiles && ok; t += n_clusters) {
        int b, m0, n0;
        tile_coords(t, b, m0, n0);
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % S, ph = (it / S) & 1;
          if (!(ok = mbar_wait_cl(&EMPTY[st], ph ^ 1, abort_flag))) break;
          uint8_t* dst = sm + st * L::kStageBytes;
          const uint32_t cf = mapa_shared(&FULL[st], 0);
          if (rank == 0) mbar_arrive_expect_tx(&FULL[st], 2u * L::kStageBytes);
          tma_load_3d_pair(dst, &mapA, cf, kc * 64, m0 + 128 * (int)rank, b);
          if (kBmn) {
#pragma unroll
            for (int i = 0; i < BN / 128; ++i)
              tma_load_3d_pair(dst + L::kABytes + i * 8192, &mapB, cf, n0 + (BN / 2) * (int)rank + 64 * i, kc * 64, b);
          } else {
            tma_load_3d_pair(dst + L::kABytes, &mapB, cf, kc * 64, n0 + (BN / 2) * (int)rank, b);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        st_cluster_u32(mapa_shared(sm + L::kOffMisc + 4, rank ^ 1u), 1u);
        flag_error(g.err, LR_DEVERR_TIMEOUT);
      }
      if (rank == 0)  // the loads of the last stages have landed
        for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
          mbar_wait_cl_drain(&FULL[j % S], (j / S) & 1, kWaitCycles / 4);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (CTA 0)
    if (rank == 0 && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, BN, false, kBmn);
      uint32_t it = 0;
      bool ok = true;
      int i = 0;
      for (int t = cluster; t < n_tiles && ok; t += n_clusters, ++i) {
        const int buf = i & 1;
        if (i >= 2 && !(ok = mbar_wait_cl(&TEMPTY[buf], ((i >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t dcol = tmem + buf * BN;
        for (int kc = 0; kc < nk && ok; ++kc, ++it) {
          const uint32_t st = it % S, ph = (it / S) & 1;
          if (!(ok = mbar_wait_cl(&FULL[st], ph, abort_flag))) break;
          tc_fence_after();
          const uint32_t a = smem_u32(sm + st * L::kStageBytes);
          const uint32_t bb = a + L::kABytes;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = kBmn ? sw128_desc(bb + ks * 2048, 8192, 1024) : sw128_desc(bb + ks * 32, 16, 1024);
            mma_f16_pair(dcol, sw128_desc(a + ks * 32, 16, 1024), bd, idesc, (kc | ks) != 0);
          }
          mma_commit_pair_mc(&EMPTY[st], 3);
        }
        if (ok) mma_commit_pair_mc(&TFULL[buf], 3);
      }
      if (!ok) {
        *abort_flag = 1;
        st_cluster_u32(mapa_shared(sm + L::kOffMisc + 4, 1u), 1u);
        flag_error(g.err, LR_DEVERR_TIMEOUT);
      }
      mma_commit_pair_mc(DRAIN, 1);
      mbar_wait_cl_drain(DRAIN, 0, kWaitCycles / 4);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    uint8_t* out0 = sm + L::kOffOut + (warp - 2) * 2 * kStageOutBytes;
    const uint32_t c_tempty = mapa_shared(&TEMPTY[0], 0);
    bool ok = true;
    int i = 0, ob = 0;
    for (int t = cluster; t < n_tiles && ok; t += n_clusters, ++i) {
      int b, m0, n0;
      tile_coords(t, b, m0, n0);
      const int buf = i & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait_cl(&TFULL[buf], (i >> 1) & 1, abort_flag)))) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 64; ++c, ob ^= 1) {
        uint32_t v0[32], v1[32];
        tmem_ld32(trow + buf * BN + c * 64, v0);
        tmem_ld32(trow + buf * BN + c * 64 + 32, v1);
        tmem_ld_wait();
        if (c == BN / 64 - 1) {  // this warp is done with the accumulator buffer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(c_tempty + 8u * buf);
        }
        uint8_t* ob_ptr = out0 + ob * kStageOutBytes;
        if (lane == 0) bulk_wait_read_le1();  // the store that last read this buffer is done with it
        __syncwarp();
        uint8_t* rowp = ob_ptr + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t* src = j < 4 ? &v0[8 * j] : &v1[8 * (j - 4)];
          uint4 w;
          if (g.out_f16) {
            w.x = pack_f16x2_sat(__uint_as_float(src[0]), __uint_as_float(src[1]));
            w.y = pack_f16x2_sat(__uint_as_float(src[2]), __uint_as_float(src[3]));
            w.z = pack_f16x2_sat(__uint_as_float(src[4]), __uint_as_float(src[5]));
            w.w = pack_f16x2_sat(__uint_as_float(src[6]), __uint_as_float(src[7]));
          } else {
            w.x = pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1]));
            w.y = pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3]));
            w.z = pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5]));
            w.w = pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7]));
          }
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = m0 + 128 * (int)rank + 32 * q;
          if (y < g.M) tma_store_3d(&mapC, ob_ptr, n0 + c * 64, y, b);  // rows past M are clipped by TMA
          bulk_commit_group();
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      st_cluster_u32(mapa_shared(sm + L::kOffMisc + 4, rank ^ 1u), 1u);
      flag_error(g.err, LR_DEVERR_TIMEOUT);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // no CTA frees TMEM or exits while the pair's MMAs or loads may touch it
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem, L::kTmemCols);
  }
}

template <int BN, bool kBmn>
int max_clusters_for() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev]) return cached[dev];
  using L = GemmLayout<BN, kBmn>;
  if (cudaFuncSetAttribute(gemm_pair_kernel<BN, kBmn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::kSmemBytes) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<BN, kBmn>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cached[dev] = n;
  return n;
}

template <int BN, bool kBmn>
cudaError_t launch_t(const GemmArgs& g, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC,
                     cudaStream_t st) {
  using L = GemmLayout<BN, kBmn>;
  static_assert(L::kSmemBytes <= 232448, "shared memory budget");
  static_assert(L::kOffOut % 1024 == 0 && L::kStageBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  const int n_tiles = g.B * ((g.M + 255) / 256) * (g.N / BN);
  if (n_tiles == 0) return cudaSuccess;
  int clusters = max_clusters_for<BN, kBmn>();
  if (clusters <= 0) return cudaErrorInvalidConfiguration;
  if (clusters > n_tiles) clusters = n_tiles;
  cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<BN, kBmn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kSmemBytes);
  if (e != cudaSuccess) return e;
  gemm_pair_kernel<BN, kBmn><<<2 * clusters, kThreads, L::kSmemBytes, st>>>(mA, mB, mC, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_pair(const GemmArgs& g, const CUtensorMap& mA, const CUtensorMap& mB, const CUtensorMap& mC,
                             cudaStream_t st) {
  if (g.K % 64 || g.N % g.bn || (g.bn != 128 && g.bn != 256)) return cudaErrorInvalidValue;
  if (g.bn == 256) return g.b_mn_major ? launch_t<256, true>(g, mA, mB, mC, st) : launch_t<256, false>(g, mA, mB, mC, st);
  return g.b_mn_major ? launch_t<128, true>(g, mA, mB, mC, st) : launch_t<128, false>(g, mA, mB, mC, st);
}

}  // namespace tc
}  // namespace lr
