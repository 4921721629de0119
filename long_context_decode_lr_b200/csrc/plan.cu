// Workspace layout and kernel choice for lr_decode_attn and lr_pack_prefill.
#include "lr_common.cuh"
#include "lr_launch.h"
#include "lr_plan.h"

namespace lr {

namespace {
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t elem_bytes(lr_dtype d) { return d == LR_BF16 ? 2 : 4; }
}  // namespace

DecodePlan plan_decode(const lr_cache_shape& s, int n_q_heads, int n_sel, int sm_count) {
  DecodePlan p{};
  p.path = DecodePath::General;
  const int nblk = ceil_div(s.T, LR_BLOCK_TOKENS);
  const int units = n_sel > 0 ? n_sel : nblk;
  const int per_row = s.batch * s.n_kv_heads;
  int n_split = per_row > 0 ? ceil_div(2 * sm_count, per_row) : 1;
  if (n_split > units) n_split = units;
  if (n_split > 1024) n_split = 1024;
  if (n_split < 1) n_split = 1;
  p.n_split = n_split;
  p.part_stride = 4 + 2 * s.head_dim + s.hidden;
  p.part_off = 256;
  const size_t part_bytes = (size_t)s.batch * n_q_heads * n_split * p.part_stride * sizeof(float);
  p.sched_off = align256(p.part_off + part_bytes);
  p.ws_bytes = p.sched_off;
  return p;
}

PackPlan plan_pack(const lr_cache_shape& s, int k) {
  (void)k;
  PackPlan p{};
  p.tensor = false;
  const size_t rows = (size_t)s.batch * s.n_layers * s.n_kv_heads * s.T;
  p.err_off = 256;
  p.diff_off = align256(p.err_off + rows * sizeof(float));
  p.ws_bytes = align256(p.diff_off + rows * s.head_dim * elem_bytes(s.dtype));
  return p;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodePlan& plan, lr_dtype dt, cudaStream_t st) {
  (void)plan;
  cudaError_t e = launch_decode_general(a, dt, st);
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, dt, st);
}

cudaError_t launch_pack(const PackArgs& a, const PackPlan& plan, lr_dtype dt, cudaStream_t st) {
  (void)plan;
  if (a.T == 0) return launch_block_ptr(a.res_idx, a.res_ptr ? a.B * a.L * a.Hkv : 0, a.k, a.T, a.res_ptr, st);
  cudaError_t e = launch_pack_project_general(a, dt, st);
  if (e != cudaSuccess) return e;
  if ((e = launch_pack_predict_general(a, dt, st)) != cudaSuccess) return e;
  const int n_seg = a.B * a.L * a.Hkv;
  if ((e = launch_topk(a.err, n_seg, a.T, a.k, a.res_idx, st)) != cudaSuccess) return e;
  if ((e = launch_pack_gather(a, dt, st)) != cudaSuccess) return e;
  if (a.res_ptr) return launch_block_ptr(a.res_idx, n_seg, a.k, a.T, a.res_ptr, st);
  return cudaSuccess;
}

}  // namespace lr
