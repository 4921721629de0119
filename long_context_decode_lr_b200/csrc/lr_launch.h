// Host-side launch functions of the LowRAM kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "lowram.h"

namespace lr {

struct DecodeArgs;
struct PackArgs;
struct SelectArgs;

// General CUDA-core decode path (any supported shape, fp32 or bf16 storage).
size_t decode_general_smem_bytes(int hd, int H, int G);
size_t decode_combine_smem_bytes(int hd, int H, int G, int n_split, int elem_bytes, int n_tail);
cudaError_t launch_decode_general(const DecodeArgs& a, lr_dtype dt, cudaStream_t st);
cudaError_t launch_decode_combine(const DecodeArgs& a, lr_dtype dt, cudaStream_t st);

// Packer steps.
cudaError_t launch_pack_project_general(const PackArgs& a, lr_dtype dt, cudaStream_t st);
cudaError_t launch_pack_predict_general(const PackArgs& a, lr_dtype dt, cudaStream_t st);
cudaError_t launch_pack_gather(const PackArgs& a, lr_dtype dt, cudaStream_t st);

// 2-bit residual rows: codes, row minimum and level step of every row.
cudaError_t launch_quantize_rows(const void* rows, lr_dtype dt, long long n_rows, int hd, uint8_t* codes, float* lo,
                                 float* step, cudaStream_t st);

// Top-k token selection (radix select) and residual block pointers.
cudaError_t launch_topk(const float* err, int n_seg, int T, int k, int* idx_out, cudaStream_t st);
cudaError_t launch_block_ptr(const int* idx, int n_seg, int k, int T, int* ptr_out, cudaStream_t st);

// Block selection: block means of A (once per packed cache), mean-key block scores and
// their top-n_sel per (sequence, KV head).
cudaError_t launch_block_means(const void* A, int B, int T, int r, lr_dtype dt, float* abar, cudaStream_t st);
int select_rank_splits(int r);
cudaError_t launch_select_blocks(const SelectArgs& a, lr_dtype dt, cudaStream_t st);

}  // namespace lr
