// Shared expert for a handful of tokens (T <= 32).  With so few tokens the
// shared expert ("Module glm5next_mlp", FFN_MODULE: the dense SwiGLU FFN also
// serves the shared expert) is bound by reading its bf16 weights once from
// HBM, and a tile per 256 weight rows would leave most SMs idle.  So each
// projection is a split-K tensor-core GEMM (splitk_gemm.cu) whose K slices
// spread the weight stream over every SM, followed by a kernel that adds the
// slices in a fixed order (deterministic) and applies the epilogue:
//   gate/up: h_s[t, f] = bf16( silu(min(G, L)) * clamp(U, -L, L) )
//            (§Numerics: asymmetric clamp; G = columns [0, I_s), U = [I_s, 2 I_s)
//             of the fused [gate; up] weight)
//   down:    out[t, j] = bf16( sum_f h_s[t, f] W_d[j, f] )   (unscaled)
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kMmaN = 256;

// part[s][T][ncols]; gate/up reads gate at column f and up at column Is + f.
// One thread per (token, 4 consecutive output columns); slices are added in
// ascending order.
__global__ void __launch_bounds__(256)
    dense_small_finish_kernel(const float* __restrict__ part, int S, int T, int ncols, int gate_up, int cols,
                              float L, __nv_bfloat16* __restrict__ out) {
  const int c4 = cols / 4;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // over T * cols / 4
  if (idx >= T * c4) return;
  const int tok = idx / c4, f = (idx - tok * c4) * 4;
  const size_t slice = static_cast<size_t>(T) * ncols;
  const float* p = part + static_cast<size_t>(tok) * ncols + f;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll 4
  for (int s = 0; s < S; ++s) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p + s * slice));
    a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    if (gate_up) {
      const float4 u = __ldg(reinterpret_cast<const float4*>(p + s * slice + cols));
      b.x += u.x; b.y += u.y; b.z += u.z; b.w += u.w;
    }
  }
  float v[4] = {a.x, a.y, a.z, a.w};
  if (gate_up) {
    const float u[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float gv = fminf(v[j], L);
      const float uv = fminf(fmaxf(u[j], -L), L);
      v[j] = __fdividef(gv, 1.f + __expf(-gv)) * uv;
    }
  }
  *reinterpret_cast<uint2*>(out + static_cast<size_t>(tok) * cols + f) =
      make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// K slices so that (column tiles x slices) fills the SMs in one wave, each
// slice at least 4 k-blocks of 64.
int splits_for(int N, int K, int T, int num_sms) {
  const int n_tiles = (N + kMmaN - 1) / kMmaN;
  int s = std::max(1, num_sms / n_tiles);
  s = std::min(s, kDenseSmallMaxSplits);
  s = std::min(s, std::max(1, (K / 64) / 4));
  return splitk_actual_splits(K, 1, kMmaN, T, s);
}

}  // namespace

bool dense_small_ok(int T, int H, int Is) {
  return T >= 1 && T <= kDenseSmallMaxTokens && H % 8 == 0 && Is % 8 == 0;
}

size_t dense_small_part_floats(int H, int Is) {
  return static_cast<size_t>(kDenseSmallMaxSplits) * std::max(2 * Is, H) * kDenseSmallMaxTokens;
}

cudaError_t launch_dense_small_ffn(const void* x, int T, int H, int Is, const void* w_gu, const void* w_d, float L,
                                   float* part, void* h_s, void* out, int32_t* err, int num_sms, cudaStream_t stream) {
  // gate/up: [T, H] x [2 I_s, H]^T
  int S = splits_for(2 * Is, H, T, num_sms);
  cudaError_t e = launch_splitk_gemm(x, T, H, w_gu, 1, 2 * Is, kMmaN, S, part, err, num_sms, stream);
  if (e != cudaSuccess) return e;
  e = launch_kernel(dense_small_finish_kernel, dim3((T * Is / 4 + 255) / 256), dim3(256), 0, stream,
                            static_cast<const float*>(part), S, T, 2 * Is, 1, Is, L, static_cast<__nv_bfloat16*>(h_s));
  if (e != cudaSuccess) return e;
  // down: [T, I_s] x [H, I_s]^T
  S = splits_for(H, Is, T, num_sms);
  e = launch_splitk_gemm(h_s, T, Is, w_d, 1, H, kMmaN, S, part, err, num_sms, stream);
  if (e != cudaSuccess) return e;
  return launch_kernel(dense_small_finish_kernel, dim3((T * H / 4 + 255) / 256), dim3(256), 0, stream,
                               static_cast<const float*>(part), S, T, H, 0, H, 0.f, static_cast<__nv_bfloat16*>(out));
}

}  // namespace moe
