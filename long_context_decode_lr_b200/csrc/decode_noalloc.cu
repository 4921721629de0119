// lr_decode_attn_noalloc: the decode step for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: code that runs where a cudaMalloc
// would be unsafe or forbidden (inside an allocator or memory-pool callback, in a
// runtime that owns every allocation and hands out only fixed buffers, or in a
// real-time path where an allocation could block or fail). For them this entry point
// runs the same decode on a scratch area that is part of the loaded library: a
// file-scope device array of a fixed size. It allocates nothing and frees nothing.
//
// The array lives on every GPU that loads the library until the process exits, and all
// calls on a device share it. The first call on a device looks up the array's device
// address with cudaGetSymbolAddress (host code cannot use the array's name as a device
// pointer); make that first call before any stream capture. The address is kept for the
// life of the process, so the entry point must not be used on a device after
// cudaDeviceReset there. Calls that overlap on the GPU (different streams, or host threads
// without ordering) race on the array. lr_get_device_error with a NULL workspace reads the
// array's error word (that of the last call on the current device).
#include <atomic>

#include <cuda_runtime.h>

#include "lowram.h"

namespace lr {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kScratchBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// The decode workspace of this entry point. Each call clears the first 256 bytes (the
// device error word) and overwrites everything else it reads, so stale contents from
// the previous call are never consumed.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];

}  // namespace

namespace lr {
// Device address of the current device's scratch array (looked up once per device).
lr_status noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LR_ERR_CUDA;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return LR_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return LR_OK;
}
}  // namespace lr

extern "C" lr_status lr_decode_attn_noalloc(const lr_cache_shape* shape, int32_t layer, int32_t n_q_heads,
                                            const void* q, const void* A, const void* Bt,
                                            const lr_predictor* predictor, const int32_t* res_idx,
                                            const void* res_val, const int32_t* res_blk_ptr, int32_t k,
                                            const int32_t* block_list, int32_t n_sel, float scale, void* o,
                                            lr_stream_t stream) {
  const int32_t sel = block_list ? n_sel : 0;
  const size_t need = shape ? lr_decode_workspace_bytes(shape, n_q_heads, sel) : 0;
  if (need > kScratchBytes) {
    lr::set_last_error("lr_decode_attn_noalloc: this shape needs more scratch than the 16 MiB static area; "
                       "call lr_decode_attn with a caller workspace instead");
    return LR_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  const lr_status st = lr::noalloc_scratch_address(&ws);
  if (st != LR_OK) return st;
  return lr_decode_attn(shape, layer, n_q_heads, q, A, Bt, predictor, res_idx, res_val, res_blk_ptr, k, block_list,
                        n_sel, scale, o, ws, kScratchBytes, stream);
}
