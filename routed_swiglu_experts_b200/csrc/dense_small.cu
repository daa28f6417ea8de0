// Shared expert for a handful of tokens (T <= 32): a weight-streaming
// split-K kernel.  With so few tokens the shared expert is bound by reading
// its bf16 weights once from HBM; a 128-row tcgen05 tile would leave most
// SMs idle (only I_s/128 tiles), so here every warp streams 16 weight rows
// over one K slice through a cp.async ring and uses mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) as the dot-product engine; a second kernel adds the K
// slices in a fixed order (deterministic) and applies the SwiGLU clamp
// ("Module glm5next_mlp" §Numerics; the shared expert is added unscaled).
//
// m16 tile rows: gate/up mode puts gate rows f0..f0+7 in tile rows 0..7 and
// up rows f0..f0+7 in tile rows 8..15, so each thread holds a gate and an up
// value of the same feature; down mode takes 16 consecutive rows.
// Thread (g = lane/4, t = lane%4) loads 8 consecutive k of its rows and of
// its token per 32-wide step: MMA 1 takes the first four (slots 2t, 2t+1,
// 2t+8, 2t+9), MMA 2 the last four -- the same slot order for A and B.
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kDsWarps = 8;
constexpr int kDsTok = 32;  // tokens per call (4 n8 tiles)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 and4(uint4 v, uint32_t m) { return make_uint4(v.x & m, v.y & m, v.z & m, v.w & m); }

// Per-thread cp.async ring (same scheme as the W4A16 kernels): each 32-wide
// k step a thread copies its two weight words and its four token words into
// its own slots, kDsStages - 1 steps ahead of the MMAs.
constexpr int kDsStages = 4;
constexpr int kDsSlots = 6;
constexpr size_t kDsSmem = static_cast<size_t>(kDsWarps) * kDsStages * kDsSlots * 32 * sizeof(uint4);

// part[s][tile][16][32]: K-slice s of tile `tile` (blockIdx.x * 8 + warp).
__global__ void __launch_bounds__(kDsWarps * 32)
    dense_small_kernel(const __nv_bfloat16* __restrict__ w, int K, int tiles, int gate_up, int half_rows,
                       const __nv_bfloat16* __restrict__ act, int T, int kslice, float* __restrict__ part) {
  extern __shared__ __align__(16) uint4 ds_ring[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x * kDsWarps + warp;
  const int s = blockIdx.y;
  if (tile >= tiles) return;
  const int k0 = s * kslice, k1 = min(K, k0 + kslice);
  const int steps = (k1 - k0) / 32;
  // weight rows of tile rows g and g+8
  int ra, rb;
  if (gate_up) {
    ra = tile * 8 + g;
    rb = half_rows + tile * 8 + g;
  } else {
    ra = tile * 16 + g;
    rb = ra + 8;
  }
  const __nv_bfloat16* pa = w + static_cast<size_t>(ra) * K + k0 + 8 * t;
  const __nv_bfloat16* pb = w + static_cast<size_t>(rb) * K + k0 + 8 * t;
  const __nv_bfloat16* px[4];
  uint32_t keep[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int tok = g + 8 * n;
    keep[n] = tok < T ? 0xffffffffu : 0u;
    px[n] = act + static_cast<size_t>(tok < T ? tok : 0) * K + k0 + 8 * t;
  }
  uint4* ring = ds_ring + static_cast<size_t>(warp) * kDsStages * kDsSlots * 32 + lane;
  auto issue = [&](int i) {
    uint4* st = ring + (i % kDsStages) * kDsSlots * 32;
    cp_async16(st, pa + 32 * i);
    cp_async16(st + 32, pb + 32 * i);
#pragma unroll
    for (int n = 0; n < 4; ++n) cp_async16(st + (2 + n) * 32, px[n] + 32 * i);
  };
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;
#pragma unroll
  for (int i = 0; i < kDsStages - 1; ++i) {
    if (i < steps) issue(i);
    cp_async_commit();
  }
  for (int i = 0; i < steps; ++i) {
    cp_async_wait<kDsStages - 2>();
    if (i + kDsStages - 1 < steps) issue(i + kDsStages - 1);
    cp_async_commit();
    const uint4* st = ring + (i % kDsStages) * kDsSlots * 32;
    const uint4 a = st[0], b = st[32];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const uint4 xv = and4(st[(2 + n) * 32], keep[n]);
      mma_bf16_16816(acc[n], a.x, b.x, a.y, b.y, xv.x, xv.y);
      mma_bf16_16816(acc[n], a.z, b.z, a.w, b.w, xv.z, xv.w);
    }
  }
  cp_async_wait<0>();
  // C fragment: acc[n][0..1] row g, tokens 8n + 2t, +1; acc[n][2..3] row g+8
  float* out = part + (static_cast<size_t>(s) * tiles + tile) * 16 * kDsTok;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int tok = 8 * n + 2 * t;
    *reinterpret_cast<float2*>(out + g * kDsTok + tok) = make_float2(acc[n][0], acc[n][1]);
    *reinterpret_cast<float2*>(out + (g + 8) * kDsTok + tok) = make_float2(acc[n][2], acc[n][3]);
  }
}

// gate/up: h[tok, f] = bf16(silu(min(G, L)) * clamp(U, -L, L)), G/U summed
// over the S slices in order.  down: out[tok, j] = bf16(sum).
__global__ void __launch_bounds__(256)
    dense_small_finish_kernel(const float* __restrict__ part, int S, int tiles, int gate_up, int cols, int T,
                              float L, __nv_bfloat16* __restrict__ out) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // over T * cols
  if (idx >= T * cols) return;
  const int tok = idx / cols, f = idx - tok * cols;
  int tile, r;
  if (gate_up) {
    tile = f / 8;
    r = f % 8;
  } else {
    tile = f / 16;
    r = f % 16;
  }
  float a = 0.f, b = 0.f;
  for (int s = 0; s < S; ++s) {
    const float* p = part + (static_cast<size_t>(s) * tiles + tile) * 16 * kDsTok;
    a += p[r * kDsTok + tok];
    if (gate_up) b += p[(r + 8) * kDsTok + tok];
  }
  float v;
  if (gate_up) {
    const float gv = fminf(a, L);
    const float uv = fminf(fmaxf(b, -L), L);
    v = __fdividef(gv, 1.f + __expf(-gv)) * uv;
  } else {
    v = a;
  }
  out[static_cast<size_t>(tok) * cols + f] = __float2bfloat16_rn(v);
}

int splits_for(int tiles, int K) {
  int s = std::max(1, (kDsWarps * 148 + tiles - 1) / tiles);
  s = std::min(s, kDenseSmallMaxSplits);
  s = std::min(s, std::max(1, K / 256));
  return s;
}

}  // namespace

bool dense_small_ok(int T, int H, int Is) {
  return T >= 1 && T <= kDsTok && H % 32 == 0 && Is % 32 == 0 && Is % 8 == 0 && H % 16 == 0;
}

size_t dense_small_part_floats(int H, int Is) {
  return static_cast<size_t>(kDenseSmallMaxSplits) * std::max(2 * Is, H) * kDsTok;
}

cudaError_t launch_dense_small_ffn(const void* x, int T, int H, int Is, const void* w_gu, const void* w_d, float L,
                                   float* part, void* h_s, void* out, cudaStream_t stream) {
  // gate/up: I_s/8 tiles of (8 gate + 8 up) rows over K = H
  const int t_gu = Is / 8;
  int S = splits_for(t_gu, H);
  int kslice = ((H + S - 1) / S + 31) / 32 * 32;
  S = (H + kslice - 1) / kslice;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(dense_small_kernel), static_cast<int>(kDsSmem));
  if (e != cudaSuccess) return e;
  dense_small_kernel<<<dim3((t_gu + kDsWarps - 1) / kDsWarps, S), kDsWarps * 32, kDsSmem, stream>>>(
      static_cast<const __nv_bfloat16*>(w_gu), H, t_gu, 1, Is, static_cast<const __nv_bfloat16*>(x), T, kslice,
      part);
  dense_small_finish_kernel<<<(T * Is + 255) / 256, 256, 0, stream>>>(part, S, t_gu, 1, Is, T, L,
                                                                      static_cast<__nv_bfloat16*>(h_s));
  // down: H/16 tiles of 16 rows over K = I_s
  const int t_d = H / 16;
  S = splits_for(t_d, Is);
  kslice = ((Is + S - 1) / S + 31) / 32 * 32;
  S = (Is + kslice - 1) / kslice;
  dense_small_kernel<<<dim3((t_d + kDsWarps - 1) / kDsWarps, S), kDsWarps * 32, kDsSmem, stream>>>(
      static_cast<const __nv_bfloat16*>(w_d), Is, t_d, 0, 0, static_cast<const __nv_bfloat16*>(h_s), T, kslice,
      part);
  dense_small_finish_kernel<<<(T * H + 255) / 256, 256, 0, stream>>>(part, S, t_d, 0, H, T, 0.f,
                                                                     static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace moe
