// W4A16 routed expert projections for small token counts ("Module
// glm5next_mlp", W4A16_GEMV_MODULE: its GEMV kernels run every routed-expert
// projection except the grouped prefill GEMM).  HBM-bound: every weight byte
// is read once per (expert, 8-token chunk) through a per-warp cp.async ring,
// dequantised in registers and fed to mma.sync m16n8k16 (fp16 in, fp32
// accumulate) as a dot-product engine, which keeps the ALU work per 8 codes
// to one shift, four LOP3s and four fp16x2 subtractions.
//
// Weight format: uint8 [N, K/2], the code of k = 2c in the low nibble of byte
// c and k = 2c+1 in the high nibble; w = (code - 8) * scale[n, k / 128].
//
// Dequantisation: the exponent-OR ("magic number") integer-to-fp16
// conversion of mixed-input GEMM kernels (Kim et al., "Who Says Elephants
// Can't Run: Bringing Large Scale MoE Models into Cloud Scale Production",
// 2022; the Marlin kernels, Frantar et al., 2024).  For a 32-bit word w of 8
// codes (nibble i = physical offset i), OR-ing the fp16 exponent of 1024 and
// subtracting the offset with one sub.f16x2 gives exact fp16 pairs:
//   P0 = ((w      & 0x000F000F) | 0x64006400) - 1032 = {q0 - 8,       q4 - 8}
//   P1 = ((w      & 0x00F000F0) | 0x64006400) - 1152 = {16 (q1 - 8),  16 (q5 - 8)}
//   P2 = ((w >> 8 & 0x000F000F) | 0x64006400) - 1032 = {q2 - 8,       q6 - 8}
//   P3 = ((w >> 8 & 0x00F000F0) | 0x64006400) - 1152 = {16 (q3 - 8),  16 (q7 - 8)}
// The MMA reduces over 16 slots; any bijection of physical k onto slots
// works if activations use the same one.  Thread (g = lane / 4, t = lane % 4)
// owns k in [128 q + 32 t, 128 q + 32 t + 32) of each 128-wide scale group
// q; each word feeds two MMAs:
//   first : slots {2t, 2t+1} <- P0 (x0, x4);  slots {2t+8, 2t+9} <- P1 (x1/16, x5/16)
//   second: slots {2t, 2t+1} <- P2 (x2, x6);  slots {2t+8, 2t+9} <- P3 (x3/16, x7/16)
// The activations are pre-arranged once per call in exactly that order as
// fp16 (x/16 in the slots of the 16-times codes: an exact power-of-two
// scaling), so each group's MMA sum is exactly sum_k (q_k - 8) x_k up to the
// fp32 accumulation; it is then multiplied by the group's bf16 scale.
//
// NVFP4 experts (FP4 E2M1 codes packed the same way, an FP8 E4M3 scale per
// 16 of K, an fp32 scale per expert tensor) run the same kernels with
// FP4 = true.  A thread's 32 k of a group are two whole 16-wide scale
// blocks, and in each MMA its slots hold k of one block only, so it decodes
// a word into the same slot pairs (e2m1_word_pairs: {k0, k4}, {k1, k5},
// {k2, k6}, {k3, k7}, no 16-times pairs, activations not divided by 16) and
// multiplies them by its row's block scale before the MMA -- exact in fp16
// (e2m1 * e4m3: at most 6 significant bits, magnitude 0 or within
// [2^-10, 2688]).  The MMAs then accumulate across groups directly, and the
// tensor scale multiplies the fp32 sum at the store.
#include <cuda_fp16.h>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kTok = 8;  // tokens per work item (the MMA's N)

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Dequantised slot pairs of one code word (see the file comment).
struct Pairs {
  uint32_t p0, p1, p2, p3;
};
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ Pairs code_pairs(uint32_t w) {
  const uint32_t w8 = w >> 8;
  Pairs r;
  r.p0 = hsub2((w & 0x000F000Fu) | 0x64006400u, 0x64086408u);   // - {1032, 1032}
  r.p1 = hsub2((w & 0x00F000F0u) | 0x64006400u, 0x64806480u);   // - {1152, 1152}
  r.p2 = hsub2((w8 & 0x000F000Fu) | 0x64006400u, 0x64086408u);
  r.p3 = hsub2((w8 & 0x00F000F0u) | 0x64006400u, 0x64806480u);
  return r;
}

// D = A B (C = 0): the first MMA of a group starts its sum without zeroing
// the accumulator registers every group.
__device__ __forceinline__ void mma_f16_16816_zc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
  const float z = 0.f;
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
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
    if (i == 0)
      mma_f16_16816_zc(t, a.p0, b.p0, a.p1, b.p1, act[i].x, act[i].y);
    else
      mma_f16_16816(t, a.p0, b.p0, a.p1, b.p1, act[i].x, act[i].y);
    mma_f16_16816(t, a.p2, b.p2, a.p3, b.p3, act[i].z, act[i].w);
  }
}

// NVFP4: one 128-wide group of one m16 tile, accumulating into d.  The
// weights of rows g and g + 8 are decoded and multiplied by their E4M3 block
// scales (sa*, sb*: (s, s) of the thread's first and second 16 of k) before
// the MMAs, so no per-group scale follows.
__device__ __forceinline__ void tile_group_fp4(float (&d)[4], const uint4 c0, const uint4 c8, const uint4 (&act)[4],
                                               uint32_t sa0, uint32_t sb0, uint32_t sa8, uint32_t sb8) {
  const uint32_t r0[4] = {c0.x, c0.y, c0.z, c0.w};
  const uint32_t r8[4] = {c8.x, c8.y, c8.z, c8.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t s0 = i < 2 ? sa0 : sb0, s8 = i < 2 ? sa8 : sb8;
    const uint4 a = e2m1_word_pairs(r0[i]);
    const uint4 b = e2m1_word_pairs(r8[i]);
    mma_f16_16816(d, hmul2_bits(a.x, s0), hmul2_bits(b.x, s8), hmul2_bits(a.y, s0), hmul2_bits(b.y, s8), act[i].x,
                  act[i].y);
    mma_f16_16816(d, hmul2_bits(a.z, s0), hmul2_bits(b.z, s8), hmul2_bits(a.w, s0), hmul2_bits(b.w, s8), act[i].z,
                  act[i].w);
  }
}

// Activations in MMA slot order.  One block per row, one thread per 8
// consecutive values: in {x0..x7} -> out fp16 {x0, x4, x1/16, x5/16, x2, x6,
// x3/16, x7/16} (NVFP4, FP4 = true: {x0, x4, x1, x5, x2, x6, x3, x7}).
// gsrc != NULL: row r of the output is token row gsrc[r] / gk of act (the
// permutation's gather, done here instead of in a separate copy).
template <bool FP4>
__global__ void __launch_bounds__(128)
    w4a16_prep_kernel(const __nv_bfloat16* __restrict__ act, int k8, const int32_t* __restrict__ gsrc, int gk,
                      uint4* __restrict__ act16) {
  constexpr float m = FP4 ? 1.f : 0.0625f;  // weight of the odd slots
  const int r = blockIdx.x;
  const int in_row = gsrc != nullptr ? __ldg(gsrc + r) / gk : r;
  const uint4* in = reinterpret_cast<const uint4*>(act) + static_cast<size_t>(in_row) * k8;
  uint4* out = act16 + static_cast<size_t>(r) * k8;
  for (int c = threadIdx.x; c < k8; c += blockDim.x) {
    const uint4 v = __ldg(in + c);
    const __half2 a04 = __floats2half2_rn(bf16lo(v.x), bf16lo(v.z));
    const __half2 b15 = __floats2half2_rn(bf16hi(v.x) * m, bf16hi(v.z) * m);
    const __half2 a26 = __floats2half2_rn(bf16lo(v.y), bf16lo(v.w));
    const __half2 b37 = __floats2half2_rn(bf16hi(v.y) * m, bf16hi(v.w) * m);
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a04);
    o.y = *reinterpret_cast<const uint32_t*>(&b15);
    o.z = *reinterpret_cast<const uint32_t*>(&a26);
    o.w = *reinterpret_cast<const uint32_t*>(&b37);
    out[c] = o;
  }
}

// Down-projection activations: the clamped SwiGLU of the fp32 gate/up
// projection ("Module glm5next_mlp" §Numerics), rounded to bf16 like the
// bf16 path's h, then laid out in MMA slot order as above.  gu: fp32
// [rows, 2I] (gate columns [0, I), up columns [I, 2I)); one thread per 8
// consecutive features of a row.
// Shared expert (when gus != NULL): its fp32 gate/up [Ts, 2 I_s] from the
// gate/up launch becomes h_s = bf16(silu(min(G, L)) * clamp(U, -L, L)) [Ts, I_s],
// row-major, for the bf16 GEMV of its down projection (indices past n8).
__device__ __forceinline__ float swiglu_clamped_f(float g, float u, float L) {
  const float gc = fminf(g, L);
  const float uc = fminf(fmaxf(u, -L), L);
  return __fdividef(gc, 1.f + __expf(-gc)) * uc;
}

template <bool FP4>
__global__ void __launch_bounds__(256)
    w4a16_prep_swiglu_kernel(const float* __restrict__ gu, int I, long long n8, float L, uint4* __restrict__ act16,
                             const float* __restrict__ gus, int Is, long long n8s, __nv_bfloat16* __restrict__ hs) {
  constexpr float m = FP4 ? 1.f : 0.0625f;  // weight of the odd slots (see w4a16_prep_kernel)
  long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n8) {
    idx -= n8;
    if (gus == nullptr || idx >= n8s) return;
    const int is8 = Is / 8;
    const long long r = idx / is8;
    const int f = static_cast<int>(idx - r * is8) * 8;
    const float* gp = gus + r * 2 * Is + f;
    float h[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = swiglu_clamped_f(__ldg(gp + j), __ldg(gp + Is + j), L);
    uint4 o;
    o.x = pack_bf16x2(h[0], h[1]);
    o.y = pack_bf16x2(h[2], h[3]);
    o.z = pack_bf16x2(h[4], h[5]);
    o.w = pack_bf16x2(h[6], h[7]);
    *reinterpret_cast<uint4*>(hs + r * Is + f) = o;
    return;
  }
  const int i8 = I / 8;
  const long long r = idx / i8;
  const int f = static_cast<int>(idx - r * i8) * 8;
  const float* gp = gu + r * 2 * I + f;
  const float4 g0 = __ldg(reinterpret_cast<const float4*>(gp)), g1 = __ldg(reinterpret_cast<const float4*>(gp + 4));
  const float4 u0 = __ldg(reinterpret_cast<const float4*>(gp + I)), u1 = __ldg(reinterpret_cast<const float4*>(gp + I + 4));
  const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
  float h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) h[j] = __bfloat162float(__float2bfloat16_rn(swiglu_clamped_f(gv[j], uv[j], L)));
  const __half2 a04 = __floats2half2_rn(h[0], h[4]);
  const __half2 b15 = __floats2half2_rn(h[1] * m, h[5] * m);
  const __half2 a26 = __floats2half2_rn(h[2], h[6]);
  const __half2 b37 = __floats2half2_rn(h[3] * m, h[7] * m);
  uint4 o;
  o.x = *reinterpret_cast<const uint32_t*>(&a04);
  o.y = *reinterpret_cast<const uint32_t*>(&b15);
  o.z = *reinterpret_cast<const uint32_t*>(&a26);
  o.w = *reinterpret_cast<const uint32_t*>(&b37);
  act16[idx] = o;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The shared expert's bf16 projection for up to 32 tokens, run by the
// blocks of blockIdx.y == 0 of the routed GEMV launches so that its weight
// stream (HBM-bound, no dequantisation) overlaps the routed experts' ALU-bound
// one instead of running before them.  One warp: rows [n0, n0 + 16) of
// W [N, K] against every token of act [T, K] (bf16, row-major), fp32
// accumulation, out [T, N] (fp32, or bf16 when !F32OUT).
// Each thread loads 8 consecutive k of its rows g and g + 8 and of its tokens
// per 32-wide K step and feeds two m16n8k16 MMAs per 8 tokens; the MMA reduces
// over its 16 slots, so physical k = k0 + 8t + j goes to slot 2t + {0, 1, 8, 9}
// (j = 0..3) of the first MMA and the same slots of the second (j = 4..7),
// for weights and activations alike.
template <bool F32OUT>
__device__ __noinline__ void shared_gemv_warp(const __nv_bfloat16* __restrict__ W, const __nv_bfloat16* __restrict__ act,
                                              int N, int K, int T, int n0, void* __restrict__ out, int lane) {
  const int g = lane >> 2, t = lane & 3;
  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const bool r0 = n0 + g < N, r8 = n0 + g + 8 < N;
  const uint4* w0 = reinterpret_cast<const uint4*>(W + static_cast<size_t>(r0 ? n0 + g : 0) * K + 8 * t);
  const uint4* w8 = reinterpret_cast<const uint4*>(W + static_cast<size_t>(r8 ? n0 + g + 8 : 0) * K + 8 * t);
  const uint4 z = make_uint4(0, 0, 0, 0);
  // the weight rows of the next K step are loaded before this step's MMAs
  // (two steps of weights in flight per thread)
  auto load_w = [&](int k0, uint4& a, uint4& b) {
    const bool kin = k0 < K && k0 + 8 * t < K;  // K % 8 == 0: the 8 values are all in or all out
    a = (r0 && kin) ? __ldcs(w0 + k0 / 8) : z;
    b = (r8 && kin) ? __ldcs(w8 + k0 / 8) : z;
  };
  uint4 na, nb;
  load_w(0, na, nb);
  for (int k0 = 0; k0 < K; k0 += 32) {
    const bool kin = k0 + 8 * t < K;
    const uint4 wa = na, wb = nb;
    load_w(k0 + 32, na, nb);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = 8 * j + g;
      const uint4 av = (tok < T && kin)
                           ? __ldg(reinterpret_cast<const uint4*>(act + static_cast<size_t>(tok) * K + k0 + 8 * t))
                           : z;
      mma_bf16_16816(acc[j], wa.x, wb.x, wa.y, wb.y, av.x, av.y);
      mma_bf16_16816(acc[j], wa.z, wb.z, wa.w, wb.w, av.z, av.w);
    }
  }
  // acc[j][0..1]: row n0 + g, tokens 8j + 2t + {0, 1}; acc[j][2..3]: row n0 + g + 8
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = 8 * j + 2 * t + (c & 1);
      const int col = n0 + g + 8 * (c >> 1);
      if (tok < T && col < N) {
        const size_t o = static_cast<size_t>(tok) * N + col;
        if (F32OUT)
          static_cast<float*>(out)[o] = acc[j][c];
        else
          static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(acc[j][c]);
      }
    }
}

// Shared-expert projection riding along in a routed GEMV launch (NULL w: none).
struct SharedJob {
  const __nv_bfloat16* w;    // [N, K]
  const __nv_bfloat16* act;  // [T, K]
  void* out;                 // [T, N]: fp32 (gate/up) or bf16 (down)
  int N, K, T;
};

// Streaming GEMV.  One warp owns 16 output rows of one expert for one
// 8-token chunk and walks K one 128-wide scale group at a time.  The code
// stream is the latency problem: each thread copies its 16 code bytes of rows
// g and g+8 per group into its own slots of a per-warp shared-memory ring
// with cp.async, kGemvStages - 1 groups ahead of the MMAs, so every warp keeps
// several kilobytes in flight without spending registers on them (a thread
// only reads back what it copied itself: no barrier).  Per group a thread
// also loads its token's 64 activation bytes (lanes past the chunk's last
// token load that token: their output columns are never stored, and
// unconditional loads save the per-group zero fill, 3% of the kernel's time)
// and its two rows' bf16 scales, one 2-byte load each (cache-resident; holding
// a batch of 8 scales per row in registers instead cost 16 registers of the
// 72 and measured 2% slower).  A group's first MMA takes a zero accumulator
// operand instead of zeroed registers.  The gate/up projection runs as one matrix of 2I
// rows with fp32 output (the SwiGLU is applied when the down projection's
// activations are prepared: pairing each gate row with its up row in one
// MMA tile to apply it in registers measured 0.5% slower); the down projection writes bf16 scaled by the
// row's combine weight.  Groups are walked eight at a time, so the ring slot
// of every copy and read is a constant of the unrolled loop and the code
// and activation addresses are constant offsets from a per-batch base: the
// ALU pipe, which the nibble conversion already keeps busy, spends nothing
// on ring bookkeeping (3% faster than computing the slot from the group
// index, same bits).  Seven blocks per SM hold the registers at 72.
constexpr int kGemvWarps = 4;
constexpr int kGemvRows = 16 * kGemvWarps;  // output rows per block
constexpr int kGemvStages = 4;
constexpr int kGemvBlocksPerSm = 7;
constexpr size_t kGemvSmem = static_cast<size_t>(kGemvWarps) * kGemvStages * 64 * sizeof(uint4);
static_assert(8 % kGemvStages == 0, "ring slots repeat within a batch of 8 groups");

template <bool F32OUT, bool FP4>
__global__ void __launch_bounds__(kGemvWarps * 32, kGemvBlocksPerSm)
    w4a16_gemv_kernel(const uint4* __restrict__ act16, const int32_t* __restrict__ offsets,
                      const uint8_t* __restrict__ q, const void* __restrict__ scales,
                      const float* __restrict__ tscale, int N, int K, const float* __restrict__ w_perm,
                      void* __restrict__ out, const SharedJob sj) {
  extern __shared__ uint4 gemv_ring[];
  constexpr int S = kGemvStages;
  // blocks of the first grid row take the shared expert (when there is one):
  // they start first, and their weight stream runs beside the routed blocks'
  int e = blockIdx.y;
  if (sj.w != nullptr) {
    if (e == 0) {
      const int n0s = blockIdx.x * kGemvRows + (threadIdx.x / 32) * 16;
      if (n0s < sj.N) shared_gemv_warp<F32OUT>(sj.w, sj.act, sj.N, sj.K, sj.T, n0s, sj.out, threadIdx.x % 32);
      return;
    }
    --e;
  }
  const int r_begin = offsets[e], r_end = offsets[e + 1];
  if (r_end <= r_begin) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * kGemvRows + warp * 16;
  if (n0 >= N) return;
  const int groups = K / 128;
  const size_t rb = static_cast<size_t>(K) / 2;
  const size_t row0 = static_cast<size_t>(e) * N + n0 + g;
  const uint8_t* q0 = q + row0 * rb + 16 * t;  // row g; row g + 8 at + q8off
  const uint32_t q8off = 8u * static_cast<uint32_t>(rb);  // < 2^32: a bf16 row of K is < 2^31 bytes
  // int4: the bf16 scales of rows g and g + 8; NVFP4: their E4M3 block-scale
  // pairs (blocks 8 q + 2t and + 1 of group q, at 16-bit index 4 q)
  const __nv_bfloat16* s0p = FP4 ? nullptr : static_cast<const __nv_bfloat16*>(scales) + row0 * groups;
  const __nv_bfloat16* s8p = FP4 ? nullptr : s0p + 8 * groups;
  const unsigned short* f0p =
      FP4 ? reinterpret_cast<const unsigned short*>(static_cast<const uint8_t*>(scales) + row0 * (K / 16)) + t
          : nullptr;
  const unsigned short* f8p = FP4 ? f0p + 8 * (K / 32) : nullptr;
  const float ts = FP4 ? __ldg(tscale + e) : 1.f;
  uint4* ring = gemv_ring + warp * S * 64 + lane;
  // codes of group i (rows g and g + 8, 16 bytes each) from base qb into ring slot `slot`
  auto issue = [&](const uint8_t* qb, int i, int slot) {
    uint4* st = ring + slot * 64;
    cp_async16(st, qb + i * 64);
    cp_async16(st + 32, qb + q8off + i * 64);
  };

  for (int tc = r_begin; tc < r_end; tc += kTok) {
    const int ntok = min(kTok, r_end - tc);
    const uint4* ap = act16 + static_cast<size_t>(tc + min(g, ntok - 1)) * (K / 8) + 4 * t;
#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
      if (i < groups) issue(q0, i, i);
      cp_async_commit();
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};

    const uint8_t* qb = q0;  // codes of group g0
    const uint4* ab = ap;    // activations of group g0
    for (int g0 = 0; g0 < groups; g0 += 8, qb += 8 * 64, ab += 8 * 16) {
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int gq = g0 + jj;
        if (gq < groups) {
          uint4 act[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) act[i] = __ldg(ab + jj * 16 + i);
          cp_async_wait<S - 2>();  // group gq has landed
          if (gq + S - 1 < groups) issue(qb, jj + S - 1, (jj + S - 1) % S);  // g0 % S == 0
          cp_async_commit();
          const uint4* st = ring + (jj % S) * 64;
          const uint4 c0 = st[0], c8 = st[32];
          if (FP4) {
            const uint32_t v0 = e4m3x2_to_f16x2(__ldg(f0p + 4 * gq)), v8 = e4m3x2_to_f16x2(__ldg(f8p + 4 * gq));
            tile_group_fp4(acc, c0, c8, act, __byte_perm(v0, 0, 0x1010), __byte_perm(v0, 0, 0x3232),
                           __byte_perm(v8, 0, 0x1010), __byte_perm(v8, 0, 0x3232));
          } else {
            float tt[4];
            tile_group(tt, c0, c8, act);
            const float a0 = __bfloat162float(__ldg(s0p + gq)), a8 = __bfloat162float(__ldg(s8p + gq));
            acc[0] = fmaf(a0, tt[0], acc[0]);
            acc[1] = fmaf(a0, tt[1], acc[1]);
            acc[2] = fmaf(a8, tt[2], acc[2]);
            acc[3] = fmaf(a8, tt[3], acc[3]);
          }
        }
      }
    }
    cp_async_wait<0>();
    // acc[0..1]: row n0 + g, tokens 2t, 2t+1; acc[2..3]: row n0 + g + 8
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int tok = 2 * t + (cc & 1);
      const int col = n0 + g + 8 * (cc >> 1);
      if (tok < ntok) {
        const int r = tc + tok;
        const float a = FP4 ? acc[cc] * ts : acc[cc];
        if (F32OUT) {
          static_cast<float*>(out)[static_cast<size_t>(r) * N + col] = a;
        } else {
          const float v = a * (w_perm != nullptr ? w_perm[r] : 1.f);
          static_cast<__nv_bfloat16*>(out)[static_cast<size_t>(r) * N + col] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

template <bool FP4>
cudaError_t launch_prep(const void* act, int rows, int K, const int32_t* gsrc, int gk, void* act16,
                        cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  return launch_kernel(w4a16_prep_kernel<FP4>, dim3(rows), dim3(128), 0, stream,
                               static_cast<const __nv_bfloat16*>(act), K / 8, gsrc, gk, static_cast<uint4*>(act16));
}

template <bool F32OUT, bool FP4>
cudaError_t launch_gemv(const void* q, const void* scales, const float* tscale, int E, int N, int K,
                        const void* act16, const int32_t* offsets, const float* w_perm, void* out,
                        const SharedJob& sj, cudaStream_t stream) {
  const int nx = std::max(N, sj.w != nullptr ? sj.N : 0);
  const dim3 grid((nx + kGemvRows - 1) / kGemvRows, E + (sj.w != nullptr ? 1 : 0));
  if (grid.y == 0) return cudaSuccess;  // no routed expert and no shared expert in this call
  return launch_kernel(w4a16_gemv_kernel<F32OUT, FP4>, grid, dim3(kGemvWarps * 32), kGemvSmem, stream,
                       static_cast<const uint4*>(act16), offsets, static_cast<const uint8_t*>(q), scales, tscale, N,
                       K, w_perm, out, sj);
}

}  // namespace

bool w4a16_shared_fusable(int T, int Is) { return Is > 0 && T >= 1 && T <= kW4a16SharedMaxTokens; }

cudaError_t launch_w4a16_gateup(const moe_config& cfg, const moe_weights& w, const void* x_rows,
                                const int32_t* gather_src, const int32_t* offsets, int rows, void* act16, float* gu,
                                const void* x_shared, int T, float* gu_shared, cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  const bool fp4 = cfg.expert_format == MOE_W_NVFP4;
  cudaError_t e = fp4 ? launch_prep<true>(x_rows, rows, H, gather_src, cfg.top_k, act16, stream)
                      : launch_prep<false>(x_rows, rows, H, gather_src, cfg.top_k, act16, stream);
  if (e != cudaSuccess) return e;
  SharedJob sj{};
  if (x_shared != nullptr)  // shared gate/up [2 I_s, H] x tokens [T, H] -> fp32 [T, 2 I_s]
    sj = SharedJob{static_cast<const __nv_bfloat16*>(w.shared_w_gate_up), static_cast<const __nv_bfloat16*>(x_shared),
                   gu_shared, 2 * cfg.shared_inter, H, T};
  // W_gu [E, 2I, H/2]: one matrix of 2I rows per expert (gate rows, then up rows)
  if (fp4)
    return launch_gemv<true, true>(w.w_gate_up, w.s_gate_up, w.g_gate_up, E, 2 * I, H, act16, offsets, nullptr, gu,
                                   sj, stream);
  return launch_gemv<true, false>(w.w_gate_up, w.s_gate_up, nullptr, E, 2 * I, H, act16, offsets, nullptr, gu, sj,
                                  stream);
}

cudaError_t launch_w4a16_down(const moe_config& cfg, const moe_weights& w, const float* gu, const int32_t* offsets,
                              int rows, void* act16, const float* w_perm, void* y_perm, const float* gu_shared,
                              int T, void* h_shared, void* shared_out, cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts, Is = cfg.shared_inter;
  const bool fp4 = cfg.expert_format == MOE_W_NVFP4;
  const long long n8 = static_cast<long long>(rows) * (I / 8);
  const long long n8s = gu_shared != nullptr ? static_cast<long long>(T) * (Is / 8) : 0;
  if (n8 + n8s > 0) {
    const dim3 grid(static_cast<unsigned>((n8 + n8s + 255) / 256));
    cudaError_t e =
        fp4 ? launch_kernel(w4a16_prep_swiglu_kernel<true>, grid, dim3(256), 0, stream, gu, I, n8, cfg.swiglu_limit,
                            static_cast<uint4*>(act16), gu_shared, Is, n8s, static_cast<__nv_bfloat16*>(h_shared))
            : launch_kernel(w4a16_prep_swiglu_kernel<false>, grid, dim3(256), 0, stream, gu, I, n8, cfg.swiglu_limit,
                            static_cast<uint4*>(act16), gu_shared, Is, n8s, static_cast<__nv_bfloat16*>(h_shared));
    if (e != cudaSuccess) return e;
  }
  SharedJob sj{};
  if (gu_shared != nullptr)  // shared down [H, I_s] x h_s [T, I_s] -> bf16 [T, H], unscaled
    sj = SharedJob{static_cast<const __nv_bfloat16*>(w.shared_w_down), static_cast<const __nv_bfloat16*>(h_shared),
                   shared_out, H, Is, T};
  if (fp4)
    return launch_gemv<false, true>(w.w_down, w.s_down, w.g_down, E, H, I, act16, offsets, w_perm, y_perm, sj, stream);
  return launch_gemv<false, false>(w.w_down, w.s_down, nullptr, E, H, I, act16, offsets, w_perm, y_perm, sj, stream);
}

}  // namespace moe
