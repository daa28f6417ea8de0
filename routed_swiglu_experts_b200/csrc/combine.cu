// Combine ("Module glm5next_mlp", §One all-reduce for both EP and TP: the
// shared output and the routed slots are added in one combine kernel):
//   out[t] = bf16( shared[t] + sum_j c_j * y_perm[row_of[t*k + j]] ),
// fp32 sum in slot order (the shared row first).  One warp per token,
// 16-byte vectors.
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

// One warp per token (per column slice of its row when there are too few
// tokens to fill the GPU: blockIdx.y picks the slice): lane j < k reads slot
// j's routed row and weight once,
// the warp shares them with shuffles, then walks the hidden row four 16-byte
// vectors per lane at a time, so every lane keeps (k + 1) x 4 loads in flight
// (two per lane measured 10% slower on the skewed layer, the same on the mid
// one) and the index work is paid once per token.  Routed rows outside [lo, hi)
// (when `range` is given: range[0] = lo, range[e1 - e0] = hi, the rows of this
// rank's experts) are left out: expert parallelism's partial combine.
constexpr int kCombineWarps = 8;
constexpr int kVecPerLane = 4;

__global__ void __launch_bounds__(kCombineWarps * 32)
    combine_kernel(const __nv_bfloat16* __restrict__ y_perm, const int32_t* __restrict__ row_of,
                   const float* __restrict__ topk_w, const __nv_bfloat16* __restrict__ shared, int T, int k, int H,
                   const int32_t* __restrict__ range, int range_len, __nv_bfloat16* __restrict__ out) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kCombineWarps + warp;
  if (t >= T) return;
  int lo = 0, hi = 0x7fffffff;
  if (range != nullptr) {
    lo = __ldg(range);
    hi = __ldg(range + range_len);
  }
  // slot rows and weights: one load per lane, then broadcast to every lane;
  // `used` marks the slots whose row is in [lo, hi)
  int my_row = 0;
  float my_c = 1.f;
  bool mine = false;
  if (lane < k) {
    my_row = __ldg(row_of + static_cast<size_t>(t) * k + lane);
    mine = my_row >= lo && my_row < hi;
    if (topk_w != nullptr) my_c = __ldg(topk_w + static_cast<size_t>(t) * k + lane);
  }
  const uint32_t used = __ballot_sync(0xffffffffu, mine);
  int rows[MOE_MAX_TOP_K];
  float cs[MOE_MAX_TOP_K];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    cs[j] = __shfl_sync(0xffffffffu, my_c, j);
  }
  const int n16 = H / 8;  // 16-byte vectors per row
  // this warp's columns: slice blockIdx.y of gridDim.y, whole 64-vector steps
  const int step = 32 * kVecPerLane;
  const int per = (n16 + step * gridDim.y - 1) / (step * gridDim.y) * step;
  const int c_end = min(n16, per * static_cast<int>(blockIdx.y + 1));
  const uint4* srow = shared != nullptr ? reinterpret_cast<const uint4*>(shared + static_cast<size_t>(t) * H) : nullptr;
  uint4* orow = reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H);
  for (int c0 = per * static_cast<int>(blockIdx.y) + lane; c0 < c_end; c0 += step) {
    float a[kVecPerLane][8];
#pragma unroll
    for (int v = 0; v < kVecPerLane; ++v)
#pragma unroll
      for (int q = 0; q < 8; ++q) a[v][q] = 0.f;
    if (srow != nullptr) {
#pragma unroll
      for (int v = 0; v < kVecPerLane; ++v) {
        const int c = c0 + 32 * v;
        if (c < c_end) add8(a[v], __ldg(srow + c), 1.f);
      }
    }
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
      if ((used >> j) & 1u) {
        const uint4* yr = reinterpret_cast<const uint4*>(y_perm + static_cast<size_t>(rows[j]) * H);
#pragma unroll
        for (int v = 0; v < kVecPerLane; ++v) {
          const int c = c0 + 32 * v;
          if (c < c_end) add8(a[v], __ldg(yr + c), cs[j]);
        }
      }
    }
#pragma unroll
    for (int v = 0; v < kVecPerLane; ++v) {
      const int c = c0 + 32 * v;
      if (c < c_end) {
        uint4 o;
        o.x = pack_bf16x2(a[v][0], a[v][1]);
        o.y = pack_bf16x2(a[v][2], a[v][3]);
        o.z = pack_bf16x2(a[v][4], a[v][5]);
        o.w = pack_bf16x2(a[v][6], a[v][7]);
        orow[c] = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config& cfg, const void* y_perm, const int32_t* row_of, const float* topk_w,
                           const void* shared_out, int T, void* out, const int32_t* range, int range_len,
                           cudaStream_t stream) {
  // few tokens: split each row into column slices so that about 2048 warps run
  const int n16 = cfg.hidden / 8;
  constexpr int step = 32 * kVecPerLane;  // 16-byte vectors a warp covers per pass
  const int slices = std::max(1, std::min((n16 + step - 1) / step, (2048 + T - 1) / std::max(T, 1)));
  const dim3 grid(static_cast<unsigned>((T + kCombineWarps - 1) / kCombineWarps), static_cast<unsigned>(slices));
  return launch_kernel(combine_kernel, grid, dim3(kCombineWarps * 32), 0, stream,
                               static_cast<const __nv_bfloat16*>(y_perm), row_of, topk_w,
                               static_cast<const __nv_bfloat16*>(shared_out), T, cfg.top_k, cfg.hidden, range,
                               range_len, static_cast<__nv_bfloat16*>(out));
}

}  // namespace moe
