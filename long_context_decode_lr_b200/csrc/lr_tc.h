// Internal interface of the tensor-core decode kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace lr {
namespace tc {

// Pair kernel (2-CTA clusters, one KV head per pair; see decode_pair.cu).
struct PairArgs {
  int B, T, L, Hkv, G, H, r;
  int layer, k, nblk, pred_per_seq;
  int n_pairs;       // CTA pairs per (sequence, KV head); each CTA writes its own split
  float scale;
  const __nv_bfloat16* q;        // [B, Hq, 128]
  const __nv_bfloat16* b1;       // [(B,) L, Hkv, H]
  const __nv_bfloat16* Bt;       // [B, D, r]
  __nv_bfloat16* qhat;           // workspace: [B, Hkv, 16, r] scale * B_l^h q, bf16 hi rows then lo rows
  const __nv_bfloat16* W1;       // [(B,) L, Hkv, H, 128]
  __half* W1h;                   // workspace: [(B,) Hkv, H, 128] fp16 copy of the layer's W1
  int w1_seqs;                   // 1, or B when each sequence has its own predictor
  const int* res_idx;            // [B, L, Hkv, k]
  const __nv_bfloat16* res_val;  // [B, L, Hkv, k, 128] (null with 2-bit rows)
  const uint8_t* res_codes;      // 2-bit rows: [B, L, Hkv, k, 32] codes, else null
  const float* res_lo;           // 2-bit rows: [B, L, Hkv, k] row minimum
  const float* res_step;         // 2-bit rows: [B, L, Hkv, k] level step
  const int* res_ptr;            // [B, L, Hkv, nblk + 1] or null
  int* sched;                    // selective mode: [B, Hkv, 1 + n_sel] valid blocks; null in full mode
  int sched_stride;              // 1 + n_sel
  float* partials;               // [B, Hq, 2 * n_pairs, part_stride]
  int part_stride;
  int* err;
};

constexpr int kPairQRows = 16;  // Qhat rows per KV head: hi parts of 8 query heads, then lo parts

// Largest number of 2-CTA clusters of the pair kernel that can be resident at once.
int pair_max_clusters();
cudaError_t launch_decode_pair(const PairArgs& a, const CUtensorMap& mA, const CUtensorMap& mB0,
                               const CUtensorMap& mB1, const CUtensorMap& mQ, const CUtensorMap& mW1,
                               const int* blocks, int n_sel, cudaStream_t st);

}  // namespace tc
}  // namespace lr
