// Combine ("Module glm5next_mlp", §One all-reduce for both EP and TP: the
// shared output and the routed slots are added in one combine kernel):
//   out[t] = bf16( shared[t] + sum_j c_j * y_perm[row_of[t*k + j]] ),
// fp32 sum in slot order.  One warp per token, 16-byte vectors.
#include "moe_internal.h"

namespace moe {

namespace {

__device__ __forceinline__ void add8(float (&a)[8], const uint4 v, float c) {
  a[0] = fmaf(c, bf16lo(v.x), a[0]);
  a[1] = fmaf(c, bf16hi(v.x), a[1]);
  a[2] = fmaf(c, bf16lo(v.y), a[2]);
  a[3] = fmaf(c, bf16hi(v.y), a[3]);
  a[4] = fmaf(c, bf16lo(v.z), a[4]);
  a[5] = fmaf(c, bf16hi(v.z), a[5]);
  a[6] = fmaf(c, bf16lo(v.w), a[6]);
  a[7] = fmaf(c, bf16hi(v.w), a[7]);
}

// One warp per (token, 256-element chunk of the hidden row): 8 warps per
// block, so even a handful of tokens spreads over many SMs.
__global__ void __launch_bounds__(256)
    combine_kernel(const __nv_bfloat16* __restrict__ y_perm, const int32_t* __restrict__ row_of,
                   const float* __restrict__ topk_w, const __nv_bfloat16* __restrict__ shared, int T, int k, int H,
                   int blocks_per_token, __nv_bfloat16* __restrict__ out) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x / blocks_per_token;
  const int chunk = (blockIdx.x - t * blocks_per_token) * 8 + warp;
  if (t >= T) return;
  const int c = chunk * 32 + lane;  // 16-byte column of the row
  if (chunk * 32 >= H / 8) return;  // whole warp past the row
  // slot rows and weights: one load per lane, then broadcast to every lane
  int my_row = 0;
  float my_c = 1.f;
  if (lane < k) {
    my_row = row_of[static_cast<size_t>(t) * k + lane];
    if (topk_w != nullptr) my_c = topk_w[static_cast<size_t>(t) * k + lane];
  }
  int rows[MOE_MAX_TOP_K];
  float cs[MOE_MAX_TOP_K];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    cs[j] = __shfl_sync(0xffffffffu, my_c, j);
  }
  if (c >= H / 8) return;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (shared != nullptr) add8(a, __ldg(reinterpret_cast<const uint4*>(shared + static_cast<size_t>(t) * H) + c), 1.f);
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j)
    if (j < k) add8(a, __ldg(reinterpret_cast<const uint4*>(y_perm + static_cast<size_t>(rows[j]) * H) + c), cs[j]);
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]);
  o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]);
  o.w = pack_bf16x2(a[6], a[7]);
  reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = o;
}

}  // namespace

cudaError_t launch_combine(const moe_config& cfg, const void* y_perm, const int32_t* row_of, const float* topk_w,
                           const void* shared_out, int T, void* out, cudaStream_t stream) {
  const int chunks = (cfg.hidden / 8 + 31) / 32;  // 256-element chunks per row
  const int bpt = (chunks + 7) / 8;
  combine_kernel<<<static_cast<unsigned>(T) * bpt, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(y_perm), row_of, topk_w, static_cast<const __nv_bfloat16*>(shared_out), T,
      cfg.top_k, cfg.hidden, bpt, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace moe
