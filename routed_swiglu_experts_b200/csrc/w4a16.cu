// W4A16 routed expert projections for small token counts ("Module
// glm5next_mlp", W4A16_GEMV_MODULE: its GEMV kernels run every routed-expert
// projection except the grouped prefill GEMM).  HBM-bound: every weight byte
// is read once per (expert, 8-token chunk), dequantised in registers and fed
// to mma.sync m16n8k16 (bf16 in, fp32 accumulate), which keeps the per-code
// ALU work to one shift + one LOP3 + half a bf16x2 subtract.
//
// Weight format: uint8 [N, K/2], the code of k = 2c in the low nibble of byte
// c and k = 2c+1 in the high nibble; w = (code - 8) * scale[n, k / 128].
//
// Mapping: the MMA reduces over 16 "slots"; any bijection of physical k onto
// slots is valid as long as A (weights) and B (activations) use the same one.
// Thread (group g = lane/4, t = lane%4) loads 16 contiguous code bytes of a
// row per 128-wide scale group (k in [128q + 32t, 128q + 32t + 32)); each
// 32-bit word (8 codes, physical offsets 0..7) feeds two MMAs:
//   first : slots {2t, 2t+1} <- offsets {0, 4};  slots {2t+8, 2t+9} <- {1, 5}
//   second: slots {2t, 2t+1} <- offsets {2, 6};  slots {2t+8, 2t+9} <- {3, 7}
// so (w >> 4i) & 0x000F000F | 0x43004300 is directly the bf16x2 pair
// {128 + q_i, 128 + q_{i+4}}; subtracting 136 gives the exact (q - 8) values.
// The activations get the same order with two byte-permutes per 16 bytes.
// The per-group scale multiplies each group's fp32 partial sum.
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kW4Warps = 8;
constexpr int kTok = 8;  // tokens per pass (the MMA's N)

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t codes_pair(uint32_t w, int shift) {
  // {128 + q_lo, 128 + q_hi} as bf16x2, then minus {136, 136}
  const uint32_t b = ((w >> shift) & 0x000F000Fu) | 0x43004300u;
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(b), "r"(0x43084308u));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 128-wide scale group for rows (g, g+8) of one weight matrix:
// acc += scale * sum_k W[row, k] x[tok, k].  wr0 / wr8: 16 code bytes of
// rows g and g+8; xv[i]: 8 bf16 activations for word i (already zero for
// absent tokens).
__device__ __forceinline__ void group_mma(float (&acc)[4], const uint4 wr0, const uint4 wr8, const uint4 (&xv)[4],
                                          float s0, float s8) {
  float t[4] = {0.f, 0.f, 0.f, 0.f};
  const uint32_t w0[4] = {wr0.x, wr0.y, wr0.z, wr0.w};
  const uint32_t w8[4] = {wr8.x, wr8.y, wr8.z, wr8.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = xv[i];
    const uint32_t b04 = __byte_perm(u.x, u.z, 0x5410), b15 = __byte_perm(u.x, u.z, 0x7632);
    const uint32_t b26 = __byte_perm(u.y, u.w, 0x5410), b37 = __byte_perm(u.y, u.w, 0x7632);
    mma_bf16_16816(t, codes_pair(w0[i], 0), codes_pair(w8[i], 0), codes_pair(w0[i], 4), codes_pair(w8[i], 4), b04,
                   b15);
    mma_bf16_16816(t, codes_pair(w0[i], 8), codes_pair(w8[i], 8), codes_pair(w0[i], 12), codes_pair(w8[i], 12), b26,
                   b37);
  }
  acc[0] = fmaf(t[0], s0, acc[0]);
  acc[1] = fmaf(t[1], s0, acc[1]);
  acc[2] = fmaf(t[2], s8, acc[2]);
  acc[3] = fmaf(t[3], s8, acc[3]);
}

__device__ __forceinline__ uint4 and4(uint4 v, uint32_t m) { return make_uint4(v.x & m, v.y & m, v.z & m, v.w & m); }

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// gate/up + clamped SwiGLU for one expert (blockIdx.y) and 128 intermediate
// columns (blockIdx.x); each warp owns 16 columns.
__global__ void __launch_bounds__(kW4Warps * 32)
    w4a16_gateup_kernel(const __nv_bfloat16* __restrict__ x_perm, const int32_t* __restrict__ offsets,
                        const uint8_t* __restrict__ q_gu, const __nv_bfloat16* __restrict__ s_gu, int H, int I,
                        float L, __nv_bfloat16* __restrict__ h) {
  const int e = blockIdx.y;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  if (r1 <= r0) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * (kW4Warps * 16) + warp * 16;
  if (n0 >= I) return;
  const int groups = H / 128;
  const size_t row_bytes = static_cast<size_t>(H) / 2;
  const uint8_t* qe = q_gu + static_cast<size_t>(e) * 2 * I * row_bytes;
  const __nv_bfloat16* se = s_gu + static_cast<size_t>(e) * 2 * I * groups;
  const uint8_t* qg0 = qe + static_cast<size_t>(n0 + g) * row_bytes + 16 * t;
  const uint8_t* qg8 = qg0 + 8 * row_bytes;
  const uint8_t* qu0 = qe + static_cast<size_t>(I + n0 + g) * row_bytes + 16 * t;
  const uint8_t* qu8 = qu0 + 8 * row_bytes;
  const __nv_bfloat16* sg0 = se + static_cast<size_t>(n0 + g) * groups;
  const __nv_bfloat16* sg8 = sg0 + 8 * groups;
  const __nv_bfloat16* su0 = se + static_cast<size_t>(I + n0 + g) * groups;
  const __nv_bfloat16* su8 = su0 + 8 * groups;

  for (int tc = r0; tc < r1; tc += kTok) {
    __syncwarp();
    const int ntok = min(kTok, r1 - tc);
    const uint32_t keep = g < ntok ? 0xffffffffu : 0u;  // zero the activations of absent tokens
    const __nv_bfloat16* xr = x_perm + static_cast<size_t>(tc + (g < ntok ? g : 0)) * H + 32 * t;
    float ag[4] = {0.f, 0.f, 0.f, 0.f}, au[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
    for (int q = 0; q < groups; ++q) {
      const size_t cb = static_cast<size_t>(q) * 64;
      const uint4 wg0 = ld_stream16(qg0 + cb), wg8 = ld_stream16(qg8 + cb);
      const uint4 wu0 = ld_stream16(qu0 + cb), wu8 = ld_stream16(qu8 + cb);
      uint4 xv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xv[i] = and4(__ldg(reinterpret_cast<const uint4*>(xr + 128 * q + 8 * i)), keep);
      group_mma(ag, wg0, wg8, xv, bf16_at(sg0 + q), bf16_at(sg8 + q));
      group_mma(au, wu0, wu8, xv, bf16_at(su0 + q), bf16_at(su8 + q));
    }
    // acc[0..1]: row g, tokens 2t, 2t+1; acc[2..3]: row g+8, same tokens
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = 2 * t + (j & 1);
      const int col = n0 + g + (j >> 1) * 8;
      if (tok < ntok) {
        const float gv = fminf(ag[j], L);
        const float uv = fminf(fmaxf(au[j], -L), L);
        h[static_cast<size_t>(tc + tok) * I + col] = __float2bfloat16_rn(__fdividef(gv, 1.f + __expf(-gv)) * uv);
      }
    }
  }
}

// down projection for one expert (blockIdx.y) and 128 hidden columns
// (blockIdx.x): y_perm[r, j] = bf16( w_perm[r] * sum_i W_d[j, i] h[r, i] ).
__global__ void __launch_bounds__(kW4Warps * 32)
    w4a16_down_kernel(const __nv_bfloat16* __restrict__ h, const int32_t* __restrict__ offsets,
                      const uint8_t* __restrict__ q_d, const __nv_bfloat16* __restrict__ s_d,
                      const float* __restrict__ w_perm, int H, int I, __nv_bfloat16* __restrict__ y_perm) {
  const int e = blockIdx.y;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  if (r1 <= r0) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * (kW4Warps * 16) + warp * 16;
  if (n0 >= H) return;
  const int groups = I / 128;
  const size_t row_bytes = static_cast<size_t>(I) / 2;
  const uint8_t* qe = q_d + static_cast<size_t>(e) * H * row_bytes;
  const __nv_bfloat16* se = s_d + static_cast<size_t>(e) * H * groups;
  const uint8_t* q0 = qe + static_cast<size_t>(n0 + g) * row_bytes + 16 * t;
  const uint8_t* q8 = q0 + 8 * row_bytes;
  const __nv_bfloat16* s0 = se + static_cast<size_t>(n0 + g) * groups;
  const __nv_bfloat16* s8 = s0 + 8 * groups;

  for (int tc = r0; tc < r1; tc += kTok) {
    __syncwarp();
    const int ntok = min(kTok, r1 - tc);
    const uint32_t keep = g < ntok ? 0xffffffffu : 0u;
    const __nv_bfloat16* hr = h + static_cast<size_t>(tc + (g < ntok ? g : 0)) * I + 32 * t;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int q = 0; q < groups; ++q) {
      const size_t cb = static_cast<size_t>(q) * 64;
      const uint4 w0 = ld_stream16(q0 + cb), w8 = ld_stream16(q8 + cb);
      uint4 xv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xv[i] = and4(__ldg(reinterpret_cast<const uint4*>(hr + 128 * q + 8 * i)), keep);
      group_mma(a, w0, w8, xv, bf16_at(s0 + q), bf16_at(s8 + q));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = 2 * t + (j & 1);
      const int col = n0 + g + (j >> 1) * 8;
      if (tok < ntok) {
        const int r = tc + tok;
        const float sc = w_perm != nullptr ? w_perm[r] : 1.f;
        y_perm[static_cast<size_t>(r) * H + col] = __float2bfloat16_rn(a[j] * sc);
      }
    }
  }
}

}  // namespace

cudaError_t launch_w4a16_gateup(const moe_config& cfg, const moe_weights& w, const void* x_perm,
                                const int32_t* offsets, void* h, cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  const dim3 grid((I + kW4Warps * 16 - 1) / (kW4Warps * 16), E);
  w4a16_gateup_kernel<<<grid, kW4Warps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x_perm), offsets, static_cast<const uint8_t*>(w.w_gate_up),
      static_cast<const __nv_bfloat16*>(w.s_gate_up), H, I, cfg.swiglu_limit, static_cast<__nv_bfloat16*>(h));
  return cudaGetLastError();
}

cudaError_t launch_w4a16_down(const moe_config& cfg, const moe_weights& w, const void* h, const int32_t* offsets,
                              const float* w_perm, void* y_perm, cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  const dim3 grid((H + kW4Warps * 16 - 1) / (kW4Warps * 16), E);
  w4a16_down_kernel<<<grid, kW4Warps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(h), offsets, static_cast<const uint8_t*>(w.w_down),
      static_cast<const __nv_bfloat16*>(w.s_down), w_perm, H, I, static_cast<__nv_bfloat16*>(y_perm));
  return cudaGetLastError();
}

}  // namespace moe
