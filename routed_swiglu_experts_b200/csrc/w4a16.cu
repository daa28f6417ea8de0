// W4A16 routed expert projections for small token counts ("Module
// glm5next_mlp", W4A16_GEMV_MODULE: its GEMV kernels run every routed-expert
// projection except the grouped prefill GEMM).  HBM-bound: every weight byte
// is read once per (expert, 8-token chunk) with streaming 16-byte loads,
// dequantised in registers and fed to mma.sync m16n8k16 (fp16 in, fp32
// accumulate), which keeps the ALU work per 8 codes to one shift and four
// LOP3s.
//
// Weight format: uint8 [N, K/2], the code of k = 2c in the low nibble of byte
// c and k = 2c+1 in the high nibble; w = (code - 8) * scale[n, k / 128].
//
// Dequantisation without a subtract.  For a 32-bit word w of 8 codes
// (nibble i = physical offset i), OR-ing the fp16 exponent of 1024 gives
//   P0 = (w      & 0x000F000F) | 0x64006400 = {1024 + q0,    1024 + q4}
//   P1 = (w      & 0x00F000F0) | 0x64006400 = {1024 + 16 q1, 1024 + 16 q5}
//   P2 = (w >> 8 & 0x000F000F) | 0x64006400 = {1024 + q2,    1024 + q6}
//   P3 = (w >> 8 & 0x00F000F0) | 0x64006400 = {1024 + 16 q3, 1024 + 16 q7}
// all exact fp16 integers.  The MMA reduces over 16 slots; any bijection of
// physical k onto slots works if activations use the same one.  Thread
// (g = lane / 4, t = lane % 4) owns k in [128 q + 32 t, 128 q + 32 t + 32)
// of each 128-wide scale group q; each word feeds two MMAs:
//   first : slots {2t, 2t+1} <- P0 (x0, x4);  slots {2t+8, 2t+9} <- P1 (x1/16, x5/16)
//   second: slots {2t, 2t+1} <- P2 (x2, x6);  slots {2t+8, 2t+9} <- P3 (x3/16, x7/16)
// The activations are pre-arranged once per call in exactly that order as
// fp16 (x/16 in the "16 q" slots, an exact power-of-two scaling), so
//   MMA = sum_q (q x) + 1024 * sum(xA) + 1024 * sum(xB')
// and the wanted  sum (q - 8) x  = MMA - corr,  corr = 1032 sum(xA) + 1152
// sum(xB'), with xA the activations in the plain slots and xB' = x/16 the
// scaled ones (fp32 sums of the fp16 values actually used).  Each group's
// fp32 result is multiplied by its bf16 scale.
#include <cuda_fp16.h>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kW4Warps = 8;
constexpr int kTok = 8;       // tokens per pass (the MMA's N)
constexpr int kRowsPerWarp = 32;  // output rows per warp (two m16 tiles)

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Dequantised slot pairs of one code word (see the file comment).
struct Pairs {
  uint32_t p0, p1, p2, p3;
};
__device__ __forceinline__ Pairs code_pairs(uint32_t w) {
  const uint32_t w8 = w >> 8;
  Pairs r;
  r.p0 = (w & 0x000F000Fu) | 0x64006400u;
  r.p1 = (w & 0x00F000F0u) | 0x64006400u;
  r.p2 = (w8 & 0x000F000Fu) | 0x64006400u;
  r.p3 = (w8 & 0x00F000F0u) | 0x64006400u;
  return r;
}

// One 128-wide group, one m16 tile (rows g and g+8 of the tile): 8 MMAs.
// c0 / c8: 16 code bytes of rows g and g+8; act: the thread's 4 words of
// pre-arranged fp16 activations (token g).
__device__ __forceinline__ void tile_group(float (&t)[4], const uint4 c0, const uint4 c8, const uint4 (&act)[4]) {
  const uint32_t r0[4] = {c0.x, c0.y, c0.z, c0.w};
  const uint32_t r8[4] = {c8.x, c8.y, c8.z, c8.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const Pairs a = code_pairs(r0[i]);
    const Pairs b = code_pairs(r8[i]);
    mma_f16_16816(t, a.p0, b.p0, a.p1, b.p1, act[i].x, act[i].y);
    mma_f16_16816(t, a.p2, b.p2, a.p3, b.p3, act[i].z, act[i].w);
  }
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ uint4 and4(uint4 v, uint32_t m) { return make_uint4(v.x & m, v.y & m, v.z & m, v.w & m); }

// Activations in MMA slot order.  One thread per 8 consecutive values of a
// row: in {x0..x7} -> out fp16 {x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16};
// corr[row, group] = 1032 * sum(plain) + 1152 * sum(scaled) over the group's
// 128 values (16 threads, reduced with shuffles).
__global__ void __launch_bounds__(256)
    w4a16_prep_kernel(const __nv_bfloat16* __restrict__ act, int rows, int K, uint4* __restrict__ act16,
                      float* __restrict__ corr) {
  const int chunks = K / 8;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // rows * chunks threads (K % 128 == 0)
  const bool ok = idx < rows * chunks;
  const int r = ok ? idx / chunks : 0, c = ok ? idx % chunks : 0;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (ok) v = __ldg(reinterpret_cast<const uint4*>(act + static_cast<size_t>(r) * K) + c);
  const float x0 = bf16lo(v.x), x1 = bf16hi(v.x), x2 = bf16lo(v.y), x3 = bf16hi(v.y);
  const float x4 = bf16lo(v.z), x5 = bf16hi(v.z), x6 = bf16lo(v.w), x7 = bf16hi(v.w);
  const __half2 a04 = __floats2half2_rn(x0, x4), b15 = __floats2half2_rn(x1 * 0.0625f, x5 * 0.0625f);
  const __half2 a26 = __floats2half2_rn(x2, x6), b37 = __floats2half2_rn(x3 * 0.0625f, x7 * 0.0625f);
  float sa = __low2float(a04) + __high2float(a04) + __low2float(a26) + __high2float(a26);
  float sb = __low2float(b15) + __high2float(b15) + __low2float(b37) + __high2float(b37);
  float cv = 1032.f * sa + 1152.f * sb;
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) cv += __shfl_xor_sync(0xffffffffu, cv, off);
  if (ok) {
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a04);
    o.y = *reinterpret_cast<const uint32_t*>(&b15);
    o.z = *reinterpret_cast<const uint32_t*>(&a26);
    o.w = *reinterpret_cast<const uint32_t*>(&b37);
    act16[idx] = o;
    if ((c & 15) == 0) corr[static_cast<size_t>(r) * (K / 128) + c / 16] = cv;
  }
}

// out rows [n0, n0+32) of one weight matrix for the tokens of one pass:
// acc[tile][4] += scale * (MMA - corr), tile in {0,1}; rows of tile j are
// n0 + 16 j + {g, g+8}.  q: codes of the matrix, s: its scales.
__device__ __forceinline__ void stream_rows(float (&acc)[2][4], const uint8_t* __restrict__ q,
                                            const __nv_bfloat16* __restrict__ s, int n0, int K, int g, int t,
                                            const uint4* __restrict__ a16, const float* __restrict__ corr_lo,
                                            const float* __restrict__ corr_hi, uint32_t keep) {
  const int groups = K / 128;
  const size_t row_bytes = static_cast<size_t>(K) / 2;
  const uint8_t* q00 = q + static_cast<size_t>(n0 + g) * row_bytes + 16 * t;
  const uint8_t* q08 = q00 + 8 * row_bytes;
  const uint8_t* q10 = q00 + 16 * row_bytes;
  const uint8_t* q18 = q00 + 24 * row_bytes;
  const __nv_bfloat16* s00 = s + static_cast<size_t>(n0 + g) * groups;
  const __nv_bfloat16* s08 = s00 + 8 * groups;
  const __nv_bfloat16* s10 = s00 + 16 * groups;
  const __nv_bfloat16* s18 = s00 + 24 * groups;
#pragma unroll 2
  for (int gq = 0; gq < groups; ++gq) {
    const size_t cb = static_cast<size_t>(gq) * 64;
    const uint4 c00 = ld_stream16(q00 + cb), c08 = ld_stream16(q08 + cb);
    const uint4 c10 = ld_stream16(q10 + cb), c18 = ld_stream16(q18 + cb);
    uint4 act[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) act[i] = and4(__ldg(a16 + gq * 16 + i), keep);
    float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
    tile_group(t0, c00, c08, act);
    tile_group(t1, c10, c18, act);
    const float cl = corr_lo[gq], ch = corr_hi[gq];
    const float sc00 = bf16_at(s00 + gq), sc08 = bf16_at(s08 + gq);
    const float sc10 = bf16_at(s10 + gq), sc18 = bf16_at(s18 + gq);
    acc[0][0] = fmaf(sc00, t0[0] - cl, acc[0][0]);
    acc[0][1] = fmaf(sc00, t0[1] - ch, acc[0][1]);
    acc[0][2] = fmaf(sc08, t0[2] - cl, acc[0][2]);
    acc[0][3] = fmaf(sc08, t0[3] - ch, acc[0][3]);
    acc[1][0] = fmaf(sc10, t1[0] - cl, acc[1][0]);
    acc[1][1] = fmaf(sc10, t1[1] - ch, acc[1][1]);
    acc[1][2] = fmaf(sc18, t1[2] - cl, acc[1][2]);
    acc[1][3] = fmaf(sc18, t1[3] - ch, acc[1][3]);
  }
}

// gate/up + clamped SwiGLU for one expert (blockIdx.y) and 256 intermediate
// columns (blockIdx.x); each warp owns 32 columns (32 gate + 32 up rows).
__global__ void __launch_bounds__(kW4Warps * 32)
    w4a16_gateup_kernel(const uint4* __restrict__ x16, const float* __restrict__ xcorr,
                        const int32_t* __restrict__ offsets, const uint8_t* __restrict__ q_gu,
                        const __nv_bfloat16* __restrict__ s_gu, int H, int I, float L, __nv_bfloat16* __restrict__ h) {
  const int e = blockIdx.y;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  if (r1 <= r0) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * (kW4Warps * kRowsPerWarp) + warp * kRowsPerWarp;
  if (n0 >= I) return;
  const int groups = H / 128;
  const uint8_t* qe = q_gu + static_cast<size_t>(e) * 2 * I * (H / 2);
  const __nv_bfloat16* se = s_gu + static_cast<size_t>(e) * 2 * I * groups;
  const uint8_t* qgate = qe;
  const uint8_t* qup = qe + static_cast<size_t>(I) * (H / 2);
  const __nv_bfloat16* sgate = se;
  const __nv_bfloat16* sup = se + static_cast<size_t>(I) * groups;

  for (int tc = r0; tc < r1; tc += kTok) {
    __syncwarp();
    const int ntok = min(kTok, r1 - tc);
    const uint32_t keep = g < ntok ? 0xffffffffu : 0u;
    const int rg = tc + (g < ntok ? g : 0);                       // B row of this thread
    const int tlo = tc + min(2 * t, ntok - 1), thi = tc + min(2 * t + 1, ntok - 1);  // C columns
    const uint4* a16 = x16 + static_cast<size_t>(rg) * (H / 8) + 4 * t;
    float ag[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float au[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    stream_rows(ag, qgate, sgate, n0, H, g, t, a16, xcorr + static_cast<size_t>(tlo) * groups,
                xcorr + static_cast<size_t>(thi) * groups, keep);
    stream_rows(au, qup, sup, n0, H, g, t, a16, xcorr + static_cast<size_t>(tlo) * groups,
                xcorr + static_cast<size_t>(thi) * groups, keep);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = 2 * t + (c & 1);
        const int col = n0 + 16 * j + g + (c >> 1) * 8;
        if (tok < ntok) {
          const float gv = fminf(ag[j][c], L);
          const float uv = fminf(fmaxf(au[j][c], -L), L);
          h[static_cast<size_t>(tc + tok) * I + col] = __float2bfloat16_rn(__fdividef(gv, 1.f + __expf(-gv)) * uv);
        }
      }
    }
  }
}

// down projection for one expert (blockIdx.y) and 256 hidden columns
// (blockIdx.x): y_perm[r, j] = bf16( w_perm[r] * sum_i W_d[j, i] h[r, i] ).
__global__ void __launch_bounds__(kW4Warps * 32)
    w4a16_down_kernel(const uint4* __restrict__ h16, const float* __restrict__ hcorr,
                      const int32_t* __restrict__ offsets, const uint8_t* __restrict__ q_d,
                      const __nv_bfloat16* __restrict__ s_d, const float* __restrict__ w_perm, int H, int I,
                      __nv_bfloat16* __restrict__ y_perm) {
  const int e = blockIdx.y;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  if (r1 <= r0) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * (kW4Warps * kRowsPerWarp) + warp * kRowsPerWarp;
  if (n0 >= H) return;
  const int groups = I / 128;
  const uint8_t* qe = q_d + static_cast<size_t>(e) * H * (I / 2);
  const __nv_bfloat16* se = s_d + static_cast<size_t>(e) * H * groups;

  for (int tc = r0; tc < r1; tc += kTok) {
    __syncwarp();
    const int ntok = min(kTok, r1 - tc);
    const uint32_t keep = g < ntok ? 0xffffffffu : 0u;
    const int rg = tc + (g < ntok ? g : 0);
    const int tlo = tc + min(2 * t, ntok - 1), thi = tc + min(2 * t + 1, ntok - 1);
    const uint4* a16 = h16 + static_cast<size_t>(rg) * (I / 8) + 4 * t;
    float a[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    stream_rows(a, qe, se, n0, I, g, t, a16, hcorr + static_cast<size_t>(tlo) * groups,
                hcorr + static_cast<size_t>(thi) * groups, keep);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = 2 * t + (c & 1);
        const int col = n0 + 16 * j + g + (c >> 1) * 8;
        if (tok < ntok) {
          const int r = tc + tok;
          const float sc = w_perm != nullptr ? w_perm[r] : 1.f;
          y_perm[static_cast<size_t>(r) * H + col] = __float2bfloat16_rn(a[j][c] * sc);
        }
      }
    }
  }
}

cudaError_t launch_prep(const void* act, int rows, int K, void* act16, float* corr, cudaStream_t stream) {
  const long long threads = static_cast<long long>(rows) * (K / 8);
  w4a16_prep_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(act), rows, K, static_cast<uint4*>(act16), corr);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16_gateup(const moe_config& cfg, const moe_weights& w, const void* x_perm,
                                const int32_t* offsets, int rows, void* act16, float* corr, void* h,
                                cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  cudaError_t e = launch_prep(x_perm, rows, H, act16, corr, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid((I + kW4Warps * kRowsPerWarp - 1) / (kW4Warps * kRowsPerWarp), E);
  w4a16_gateup_kernel<<<grid, kW4Warps * 32, 0, stream>>>(
      static_cast<const uint4*>(act16), corr, offsets, static_cast<const uint8_t*>(w.w_gate_up),
      static_cast<const __nv_bfloat16*>(w.s_gate_up), H, I, cfg.swiglu_limit, static_cast<__nv_bfloat16*>(h));
  return cudaGetLastError();
}

cudaError_t launch_w4a16_down(const moe_config& cfg, const moe_weights& w, const void* h, const int32_t* offsets,
                              int rows, void* act16, float* corr, const float* w_perm, void* y_perm,
                              cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  cudaError_t e = launch_prep(h, rows, I, act16, corr, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid((H + kW4Warps * kRowsPerWarp - 1) / (kW4Warps * kRowsPerWarp), E);
  w4a16_down_kernel<<<grid, kW4Warps * 32, 0, stream>>>(
      static_cast<const uint4*>(act16), corr, offsets, static_cast<const uint8_t*>(w.w_down),
      static_cast<const __nv_bfloat16*>(w.s_down), w_perm, H, I, static_cast<__nv_bfloat16*>(y_perm));
  return cudaGetLastError();
}

}  // namespace moe
