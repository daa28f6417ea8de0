// Grouped W4A16 expert FFN GEMMs for many tokens per expert, on CTA pairs
// (tcgen05.mma.cta_group::2, fp16 operands, fp32 accumulate).
//
// "Module glm5next_mlp", W4A16 grouped prefill GEMM (MOE_GROUPED_MODULE with
// int4 group-128 weights, w = (q - 8) * scale): one launch per projection
// for all experts, driven by the expert row offsets.
//   gate/up:  h[t, f] = silu(min(G, L)) * clamp(U, -L, L), rounded to bf16
//             (§Numerics: asymmetric clamp), stored as fp16 for the down MMA
//   down:     y[t, n] = bf16( row_scale[t] * sum_i W_d[n, i] h[t, i] )
//
// Same tile and roles as the bf16 CTA-pair kernel (weights = M, 256 rows per
// pair; tokens = N rounded to 16; two 256-column TMEM accumulators), plus a
// code producer and eight dequantisation warps per CTA: TMA copies the int4
// codes of the CTA's 128 weight rows (128 bytes per row: four 64-deep K
// steps per copy) into a two-stage staging ring; two threads per weight row
// turn its 32 codes per K step into fp16 weights
//   (q - 8) * scale   -- exact in fp16: a 4-bit integer times a bf16 scale
// (within the fp16 range moe.h states for the W4A16 format) and write them,
// 128-byte swizzled, into the MMA's A stage, then each warp arrives on the
// pair's full barrier.  The code-to-fp16 step is the exponent-OR ("magic
// number") conversion of mixed-input GEMM kernels -- OR a nibble into the
// mantissa of fp16 1024.0, subtract 1024 + 8 -- as described by Kim et al.,
// "Who Says Elephants Can't Run: Bringing Large Scale MoE Models into Cloud
// Scale Production" (2022), and used by the Marlin kernels (Frantar et al.,
// 2024).  Within every aligned 8 of K the weights sit in the order
// {0, 4, 1, 5, 2, 6, 3, 7} (how four LOP3s split a 32-bit code word); the
// tokens are prepared in the same order, and the gate/up epilogue writes h
// in it, so the K sum is unchanged.
// NVFP4 experts (the module summary's routed NVFP4 MoE) run on the same
// kernel with FP4 = true: the codes are FP4 E2M1 values packed the same way,
// each 16 of K share one FP8 E4M3 scale, and each expert's weight tensor has
// one fp32 scale.  The dequantisation warps form e2m1 * e4m3 in fp16 --
// exact: at most 6 significant bits, magnitude 0 or within [2^-10, 2688] --
// with the sm_100a conversions cvt.rn.f16x2.e2m1x2 and .e4m3x2, and the
// epilogues multiply the fp32 accumulators by the tensor scale.  The activations stay 16-bit: the
// pages state no activation quantisation, so the block-scaled fp4 x fp4 MMA
// (which would quantise the tokens too) is not used.
// Tiles are handed out from a queue in the workspace header as in the bf16
// kernel.  Every mbarrier wait is bounded (MOE_ERR_DEVICE_TIMEOUT on expiry).
#include <cstring>

#include <cuda_fp16.h>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BK = 64;
constexpr int ROWS = 128;                    // weight rows per CTA
constexpr int TOK = 256;                     // tokens per pair tile
constexpr int STAGES = 5;                    // A (dequantised) and B (token) stages
constexpr int CKB = 4;                       // 64-deep K steps per code copy (128-byte code rows)
constexpr int CSTAGES = 2;                   // code stages
constexpr int A_BYTES = ROWS * BK * 2;       // 16 KB fp16 weights (dequantised)
constexpr int B_BYTES = (TOK / 2) * BK * 2;  // 16 KB fp16 tokens (this CTA's half)
constexpr int C_BYTES = ROWS * CKB * BK / 2; // 16 KB int4 codes, 128-byte swizzled rows
constexpr int DQ_WARPS = 8;                  // dequantisation warps: two threads per weight row
constexpr int DQ_WARP0 = 7;                  // first dequantisation warp
constexpr int THREADS = (DQ_WARP0 + DQ_WARPS) * 32;  // 0-3 epilogue, 4 token TMA, 5 MMA, 6 code TMA, 7.. dequant
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr int HPITCH = 144;                  // bytes per token row of the staged gate/up output
constexpr int QD = 8;                        // tile-id ring depth
// readers of every tile id, per CTA: token TMA (second CTA) or MMA issuer
// (first CTA), code TMA, 8 dequantisation warps, 4 epilogue warps
constexpr uint32_t kTileReaders = 2 * (1 + 1 + DQ_WARPS + 4);

enum class Kind { GateUp, Down };

struct alignas(64) Int4Params {
  CUtensorMap tma_q;          // codes: gate/up {K/2, 8, 2, N/8, G} box {128, 8, 2, 8, 1}; down {K/2, N, G} box {128, 128, 1}
  CUtensorMap tma_x;          // fp16 tokens {K, rows} box {64, 128}, 128-byte swizzle
  const int32_t* offsets;     // [groups + 1]
  const void* scales;         // int4: bf16 gate/up [G, 2N, K/128], down [G, N, K/128];
                              // NVFP4: E4M3 bytes gate/up [G, 2N, K/16], down [G, N, K/16]
  const float* tscale;        // NVFP4: fp32 tensor scale per expert (nullptr for int4)
  void* out;                  // gate/up: fp16 h [rows, N]; down: bf16 y [rows, N]
  const float* row_scale;     // down: per token row (or nullptr)
  int32_t groups;
  int32_t rows;
  int32_t n_out;              // N: I (gate/up) or H (down)
  int32_t K;
  int32_t k_blocks;
  int32_t f_tiles;
  float limit;
  int32_t* err;
  int32_t* queue;             // {next tile, pairs retired}: zero at launch, left zero at exit
  uint64_t wait_ns;           // limit of every wait on another role's progress
  int32_t test_withhold;      // test hook: never signal the first tile's accumulator to the epilogue
};

struct Ctl {
  uint64_t full[STAGES];      // pair's first CTA: the dequantisation warps of both CTAs
  uint64_t tok_full[STAGES];  // pair's first CTA: token bytes of both CTAs
  uint64_t empty[STAGES];
  uint64_t code_full[CSTAGES];   // this CTA's codes landed
  uint64_t code_empty[CSTAGES];  // this CTA's dequantisation warps read them
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint64_t tq_full[QD];       // tile id published (one arrive)
  uint64_t tq_empty[QD];      // first CTA: every reader has taken it
  int32_t tq[QD];             // tile ids; -1 = no more tiles
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t tiles;
  int32_t off[MOE_MAX_EXPERTS + 1];
  int32_t tp[MOE_MAX_EXPERTS + 1];
  uint4 obuf[512];
};

constexpr size_t kSmem = 1024 + STAGES * (A_BYTES + B_BYTES) + CSTAGES * C_BYTES + sizeof(Ctl);
static_assert(kSmem <= 232448, "fits the 227 KB opt-in shared memory");

struct Tile {
  int g, fidx, row0, ntok, nmma;
};

__device__ __forceinline__ Tile decode(const Int4Params& P, const Ctl& c, int t) {
  Tile ti;
  const int nf = P.f_tiles;
  const int u = t / nf;
  int lo = 0, hi = P.groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (c.tp[mid] <= u) lo = mid; else hi = mid;
  }
  ti.g = lo;
  const int tm = c.tp[lo + 1] - c.tp[lo];
  const int local = t - c.tp[lo] * nf;
  ti.fidx = local / tm;
  const int tmi = local - ti.fidx * tm;
  ti.row0 = c.off[lo] + tmi * TOK;
  ti.ntok = min(TOK, c.off[lo + 1] - ti.row0);
  ti.nmma = (ti.ntok + 15) / 16 * 16;
  return ti;
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// One code word (8 codes, k = 0..7 of an aligned 8) -> four fp16x2 weights in
// the order {k0, k4}, {k1, k5}, {k2, k6}, {k3, k7}.  The fp16 exponent OR
// gives 1024 + q (low nibble of each half) or 1024 + 16 q (high nibble);
// subtracting 1032 or 1152 leaves q - 8 or 16 (q - 8) exactly, and the scale
// (s, or s / 16 for the 16-times values) makes the weight; every step is
// exact in fp16.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t s2, uint32_t s2_16) {
  const uint32_t w8 = w >> 8;
  uint4 r;
  r.x = hmul2_u(hsub2_u((w & 0x000F000Fu) | 0x64006400u, 0x64086408u), s2);
  r.y = hmul2_u(hsub2_u((w & 0x00F000F0u) | 0x64006400u, 0x64806480u), s2_16);
  r.z = hmul2_u(hsub2_u((w8 & 0x000F000Fu) | 0x64006400u, 0x64086408u), s2);
  r.w = hmul2_u(hsub2_u((w8 & 0x00F000F0u) | 0x64006400u, 0x64806480u), s2_16);
  return r;
}

// One word of FP4 E2M1 codes -> four fp16x2 weights in the same {k0, k4},
// {k1, k5}, {k2, k6}, {k3, k7} order as dequant_word (e2m1_word_pairs),
// each times its block's E4M3 scale s2 = (s, s).  Every product is exact in
// fp16 (see the file comment).
__device__ __forceinline__ uint4 dequant_word_fp4(uint32_t w, uint32_t s2) {
  uint4 r = e2m1_word_pairs(w);
  r.x = hmul2_u(r.x, s2);  // k0, k4
  r.y = hmul2_u(r.y, s2);  // k1, k5
  r.z = hmul2_u(r.z, s2);  // k2, k6
  r.w = hmul2_u(r.w, s2);  // k3, k7
  return r;
}

// Reader side of the tile-id ring: wait until slot q holds the next id (it
// may have been stored by the other CTA of the pair: cluster-scope acquire).
__device__ __forceinline__ bool wait_tile(Ctl& c, int q, uint32_t qph, volatile int32_t* abort, uint64_t limit_ns,
                                          int& t) {
  if (!mbar_wait_bounded<true>(&c.tq_full[q], qph, abort, limit_ns)) return false;
  t = c.tq[q];
  return true;
}
__device__ __forceinline__ void release_tile(Ctl& c, int q) { mbar_arrive_cluster(leader_bar(&c.tq_empty[q])); }
__device__ __forceinline__ void next_slot(int& q, uint32_t& qph) {
  if (++q == QD) {
    q = 0;
    qph ^= 1u;
  }
}

// Position of feature f inside its aligned 8 after the {0,4,1,5,2,6,3,7} order.
__device__ __forceinline__ int slot_of(int f) {
  const int j = f & 7;
  return (f & ~7) | ((j & 3) * 2 + (j >> 2));
}

template <Kind KIND, bool FP4>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    ffn_int4_pair_kernel(const __grid_constant__ Int4Params P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* smem_a = smem;
  unsigned char* smem_b = smem + STAGES * A_BYTES;
  unsigned char* smem_c = smem_b + STAGES * B_BYTES;
  Ctl& c = *reinterpret_cast<Ctl*>(smem_c + CSTAGES * C_BYTES);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&c.full[s], 2 * DQ_WARPS);
      mbar_init(&c.tok_full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int s = 0; s < CSTAGES; ++s) {
      mbar_init(&c.code_full[s], 1);
      mbar_init(&c.code_empty[s], DQ_WARPS);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&c.tmem_full[a], 1);
      mbar_init(&c.tmem_empty[a], 2 * 4);
    }
    mbar_init(&c.mma_done, 1);
    for (int i = 0; i < QD; ++i) {
      mbar_init(&c.tq_full[i], 1);
      mbar_init(&c.tq_empty[i], kTileReaders);
    }
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&P.tma_q);
    tma_prefetch_desc(&P.tma_x);
  }
  if (warp == 0) {  // offsets + token-tile prefix per expert
    const int G = P.groups;
    const int per = (G + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      const int g = lane * per + j;
      if (g < G) {
        const int o0 = P.offsets[g], o1 = P.offsets[g + 1];
        c.off[g] = o0;
        local += (o1 - o0 + TOK - 1) / TOK;
      }
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int j = 0; j < per; ++j) {
      const int g = lane * per + j;
      if (g < G) {
        c.tp[g] = run;
        run += (P.offsets[g + 1] - P.offsets[g] + TOK - 1) / TOK;
      }
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
      c.off[G] = P.offsets[G];
      c.tp[G] = total;
      c.tiles = total * P.f_tiles;
    }
  }
  if (warp == 5) tmem_alloc_pair(&c.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();

  const uint32_t tmem_base = c.tmem_base;
  const int total_tiles = c.tiles;
  volatile int32_t* abort_flag = &c.abort_flag;
  auto fail = [&](int detail) {
    *abort_flag = 1;
    report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, detail);
  };

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      int q = 0;
      uint32_t qph = 0;
      int t_next = -2;  // next queue position, once fetched
      for (;;) {
        // Next tile: this thread of the first CTA takes it from the launch's
        // queue and publishes it to every role of both CTAs.
        int t;
        if (leader) {
          if (!mbar_wait_bounded<true>(&c.tq_empty[q], qph ^ 1u, abort_flag, P.wait_ns)) {
            fail(50);
            break;
          }
          if (t_next == -2) t_next = atomicAdd(P.queue, 1);
          t = t_next < total_tiles ? t_next : -1;
          t_next = -2;
          c.tq[q] = t;
          st_cluster_u32(map_to_rank(smem_u32(&c.tq[q]), 1), static_cast<uint32_t>(t));
          mbar_arrive_cluster(map_to_rank(smem_u32(&c.tq_full[q]), 1));
          mbar_arrive(&c.tq_full[q]);
        } else {
          if (!wait_tile(c, q, qph, abort_flag, P.wait_ns, t)) {
            fail(51);
            break;
          }
          release_tile(c, q);
        }
        next_slot(q, qph);
        if (t < 0) break;
        const Tile ti = decode(P, c, t);
        const int xrow = ti.row0 + static_cast<int>(rank) * (ti.nmma / 2);
        const int kpre = P.k_blocks > 3 ? P.k_blocks - 3 : 0;  // fetch the next id a few copies early
        for (int kb = 0; kb < P.k_blocks; ++kb) {
          if (!mbar_wait_bounded(&c.empty[stage], phase ^ 1u, abort_flag, P.wait_ns)) {
            fail(41);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&c.tok_full[stage], 2 * B_BYTES);
          tma_load_2d_pair(smem_b + stage * B_BYTES, &P.tma_x, kb * BK, xrow, leader_bar(&c.tok_full[stage]));
          if (leader && kb == kpre) t_next = atomicAdd(P.queue, 1);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (leader) {
        // retire from the queue; the last pair of the launch resets it
        __threadfence();
        if (atomicAdd(P.queue + 1, 1) == npairs - 1) {
          __threadfence();
          atomicExch(P.queue, 0);
          atomicExch(P.queue + 1, 0);
        }
      }
      // drain (first CTA): the last token copies of both CTAs complete on
      // its tok_full barriers
      const int nst = issued < STAGES ? issued : STAGES;
      for (int j = 0; j < nst; ++j) {
        const int i = issued - 1 - j;
        volatile int32_t never = 0;
        if (leader && !mbar_wait_bounded(&c.tok_full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1), &never,
                                         kTimeoutNs))
          report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 48);
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------- MMA issuer (first CTA) --
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, first = true;
      int q = 0;
      uint32_t qph = 0;
      for (;;) {
        int t;
        if (!wait_tile(c, q, qph, abort_flag, P.wait_ns, t)) {
          fail(52);
          break;
        }
        release_tile(c, q);
        next_slot(q, qph);
        if (t < 0) break;
        const Tile ti = decode(P, c, t);
        const uint32_t idesc = umma_idesc_f16(2 * ROWS, ti.nmma);
        if (!mbar_wait_bounded(&c.tmem_empty[acc], acc_phase ^ 1u, abort_flag, P.wait_ns)) {
          fail(42);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < P.k_blocks; ++kb) {
          if (!mbar_wait_bounded(&c.tok_full[stage], phase, abort_flag, P.wait_ns) ||
              !mbar_wait_bounded(&c.full[stage], phase, abort_flag, P.wait_ns)) {
            fail(43);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem_a + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(smem_b + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                           (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair(&c.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (!(P.test_withhold && first)) umma_commit_pair(&c.tmem_full[acc]);
        first = false;
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      umma_commit_pair_leader(&c.mma_done);
      volatile int32_t never = 0;
      if (!mbar_wait_bounded(&c.mma_done, 0, &never, kTimeoutNs)) report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 47);
    }
  } else if (warp == 6) {
    // ------------------------------------------------- code TMA producer --
    if (lane == 0) {
      int cs = 0, issued = 0;
      uint32_t cphase = 0;
      bool ok = true;
      const int ncb = (P.k_blocks + CKB - 1) / CKB;
      int q = 0;
      uint32_t qph = 0;
      for (;;) {
        int t;
        if (!wait_tile(c, q, qph, abort_flag, P.wait_ns, t)) {
          fail(53);
          break;
        }
        release_tile(c, q);
        next_slot(q, qph);
        if (t < 0) break;
        const Tile ti = decode(P, c, t);
        for (int cb = 0; cb < ncb; ++cb) {
          if (!mbar_wait_bounded(&c.code_empty[cs], cphase ^ 1u, abort_flag, P.wait_ns)) {
            fail(46);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&c.code_full[cs], C_BYTES);
          unsigned char* sc = smem_c + cs * C_BYTES;
          if (KIND == Kind::GateUp) {
            const int fb = ti.fidx * 16 + static_cast<int>(rank) * 8;  // first 8-feature block
            tma_load_5d(sc, &P.tma_q, cb * (CKB * BK / 2), 0, 0, fb, ti.g, &c.code_full[cs]);
          } else {
            const int n = ti.fidx * 256 + static_cast<int>(rank) * 128;
            tma_load_3d(sc, &P.tma_q, cb * (CKB * BK / 2), n, ti.g, &c.code_full[cs]);
          }
          ++issued;
          if (++cs == CSTAGES) {
            cs = 0;
            cphase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // drain: the last code copy of each stage
      const int nst = issued < CSTAGES ? issued : CSTAGES;
      for (int j = 0; j < nst; ++j) {
        const int i = issued - 1 - j;
        volatile int32_t never = 0;
        if (!mbar_wait_bounded(&c.code_full[i % CSTAGES], static_cast<uint32_t>((i / CSTAGES) & 1), &never,
                               kTimeoutNs))
          report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 49);
      }
    }
  } else if (warp >= DQ_WARP0) {
    // ------------------------------------- dequantisation (warps 7 .. 14) --
    // thread -> (weight row i of this CTA's 128, half of the row's 64 codes)
    const int dq = threadIdx.x - DQ_WARP0 * 32;
    const int i = dq & (ROWS - 1), half = dq / ROWS;
    const int groups = P.K / 128;
    const bool batch8 = (groups & 7) == 0;  // the row's scales come 8 groups per 16-byte load
    const uint32_t full_leader = leader_bar(&c.full[0]);
    int stage = 0, cs = 0;
    uint32_t phase = 0, cphase = 0;
    int q = 0;
    uint32_t qph = 0;
    for (;;) {
      int t = -1;
      const bool gotq = wait_tile(c, q, qph, abort_flag, P.wait_ns, t);
      if (!__all_sync(0xffffffffu, gotq)) {
        if (lane == 0) fail(54);
        break;
      }
      __syncwarp();
      if (lane == 0) release_tile(c, q);
      next_slot(q, qph);
      if (t < 0) break;
      const Tile ti = decode(P, c, t);
      // this row of the scale arrays (-1: past the end of the matrix, codes are zero-filled)
      int64_t srow = -1;
      if (KIND == Kind::GateUp) {
        const int f = ti.fidx * 128 + static_cast<int>(rank) * 64 + (i >> 4) * 8 + (i & 7);
        const int u = (i >> 3) & 1;
        if (f < P.n_out) srow = (static_cast<int64_t>(ti.g) * 2 + u) * P.n_out + f;
      } else {
        const int n = ti.fidx * 256 + static_cast<int>(rank) * 128 + i;
        if (n < P.n_out) srow = static_cast<int64_t>(ti.g) * P.n_out + n;
      }
      const __nv_bfloat16* sp =
          (!FP4 && srow >= 0) ? static_cast<const __nv_bfloat16*>(P.scales) + srow * groups : nullptr;
      // NVFP4: this thread's two E4M3 block scales per K step (blocks 4 kb + 2 half, + 1),
      // loaded one step ahead
      const unsigned short* sp8 =
          (FP4 && srow >= 0)
              ? reinterpret_cast<const unsigned short*>(static_cast<const unsigned char*>(P.scales) +
                                                        srow * (P.K / 16)) + half
              : nullptr;
      unsigned short s8_next = (sp8 != nullptr && P.k_blocks > 0) ? __ldg(sp8) : 0;
      uint4 sv = make_uint4(0, 0, 0, 0), sn = sv;
      if (!FP4 && batch8 && sp != nullptr) {
        sv = __ldg(reinterpret_cast<const uint4*>(sp));
        if (groups > 8) sn = __ldg(reinterpret_cast<const uint4*>(sp + 8));
      }
      bool ok = true;
      for (int kb = 0; kb < P.k_blocks; ++kb) {
        const int gq = kb >> 1;
        if (!FP4 && batch8 && (kb & 15) == 0 && kb > 0) {  // next batch of 8 groups
          sv = sn;
          if (sp != nullptr && gq + 8 < groups) sn = __ldg(reinterpret_cast<const uint4*>(sp + gq + 8));
        }
        float sf = 0.f;
        if (sp != nullptr) {
          if (batch8) {
            const int j = gq & 7;
            const uint32_t wv = (j >> 1) == 0 ? sv.x : (j >> 1) == 1 ? sv.y : (j >> 1) == 2 ? sv.z : sv.w;
            sf = (j & 1) ? bf16hi(wv) : bf16lo(wv);
          } else {
            sf = __bfloat162float(sp[gq]);
          }
        }
        const __half2 s2h = __floats2half2_rn(sf, sf);
        const __half2 s16h = __floats2half2_rn(sf * 0.0625f, sf * 0.0625f);
        const uint32_t s2 = *reinterpret_cast<const uint32_t*>(&s2h);
        const uint32_t s2_16 = *reinterpret_cast<const uint32_t*>(&s16h);
        uint32_t s2a = 0, s2b = 0;  // NVFP4: (s, s) of the thread's first and second 16 of K
        if (FP4) {
          const unsigned short s8 = s8_next;
          if (sp8 != nullptr && kb + 1 < P.k_blocks) s8_next = __ldg(sp8 + 2 * (kb + 1));
          const uint32_t both = e4m3x2_to_f16x2(s8);
          s2a = __byte_perm(both, 0, 0x1010);
          s2b = __byte_perm(both, 0, 0x3232);
        }
        // codes landed (first K step of a copy), and the MMAs have released this A stage
        const int sub = kb % CKB;
        const bool got = (sub != 0 || mbar_wait_bounded(&c.code_full[cs], cphase, abort_flag, P.wait_ns)) &&
                         mbar_wait_bounded(&c.empty[stage], phase ^ 1u, abort_flag, P.wait_ns);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) fail(45);
          ok = false;
          break;
        }
        // row i of the copy: 128 bytes, 16-byte chunk k at position k ^ (i % 8)
        const int chunk = sub * 2 + half;
        const uint4 q = *reinterpret_cast<const uint4*>(smem_c + cs * C_BYTES + i * 128 + ((chunk ^ (i & 7)) << 4));
        if (sub == CKB - 1 || kb == P.k_blocks - 1) {  // last K step of this copy
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.code_empty[cs]);
          if (++cs == CSTAGES) {
            cs = 0;
            cphase ^= 1u;
          }
        }
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
        unsigned char* dst = smem_a + stage * A_BYTES + i * 128;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = half * 4 + jj;  // 16-byte chunk of the 128-byte row
          *reinterpret_cast<uint4*>(dst + ((j ^ (i & 7)) << 4)) =
              FP4 ? dequant_word_fp4(qw[jj], jj < 2 ? s2a : s2b) : dequant_word(qw[jj], s2, s2_16);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_peer(full_leader + static_cast<uint32_t>(stage * sizeof(uint64_t)));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------- epilogue (warps 0 .. 3) --
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t empty_leader = map_to_rank(smem_u32(&c.tmem_empty[0]), 0);
    int q = 0;
    uint32_t qph = 0;
    for (;;) {
      int t = -1;
      const bool gotq = wait_tile(c, q, qph, abort_flag, P.wait_ns, t);
      if (!named_barrier_and(1, 128, gotq)) {
        if (lane == 0 && !gotq) fail(55);
        break;
      }
      __syncwarp();
      if (lane == 0) release_tile(c, q);
      next_slot(q, qph);
      if (t < 0) break;
      const Tile ti = decode(P, c, t);
      const int N = P.n_out;
      const bool got = mbar_wait_bounded(&c.tmem_full[acc], acc_phase, abort_flag, P.wait_ns);
      if (!named_barrier_and(1, 128, got)) {
        if (lane == 0 && !got) fail(44);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * 256);
      const int nch = ti.nmma / 32 + ((ti.nmma & 31) ? 1 : 0);
      if (KIND == Kind::GateUp) {
        // gate/up rows interleave as (b, u, r): a 16x256b load gives a thread
        // the gate and the up value of one feature (as in the bf16 kernel)
        const int f0 = ti.fidx * 128 + static_cast<int>(rank) * 64;
        const float L = P.limit;
        const float ts = FP4 ? __ldg(P.tscale + ti.g) : 1.f;
        unsigned char* hb = reinterpret_cast<unsigned char*>(c.obuf);
        __half* outh = static_cast<__half*>(P.out);
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
          uint32_t v[2][16];
          __syncwarp();
          tmem_ld16x256b_x4(tbase + ch * 32, v[0]);
          tmem_ld16x256b_x4(tbase + (16u << 16) + ch * 32, v[1]);
          tmem_ld_wait();
          named_barrier_sync(1, 128);  // previous chunk's staging reads done
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int fl = slot_of((2 * warp + h) * 8 + (lane >> 2));  // stored in the K order of the down MMA
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int tok = 8 * q + 2 * (lane & 3) + e;
                const float graw = __uint_as_float(v[h][4 * q + e]);
                const float uraw = __uint_as_float(v[h][4 * q + 2 + e]);
                const float gv = fminf(FP4 ? graw * ts : graw, L);
                const float uv = fminf(fmaxf(FP4 ? uraw * ts : uraw, -L), L);
                const float hv = __bfloat162float(__float2bfloat16_rn(__fdividef(gv, 1.f + __expf(-gv)) * uv));
                *reinterpret_cast<__half*>(hb + tok * HPITCH + fl * 2) = __float2half_rn(hv);
              }
          }
          named_barrier_sync(1, 128);  // staging complete
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int idx = threadIdx.x + 128 * r;
            const int row = idx >> 3, c16 = idx & 7;
            const int col = ch * 32 + row;
            const int f = f0 + c16 * 8;
            if (col < ti.ntok && f < N)
              *reinterpret_cast<uint4*>(outh + static_cast<size_t>(ti.row0 + col) * N + f) =
                  *reinterpret_cast<const uint4*>(hb + row * HPITCH + c16 * 16);
          }
        }
      } else {
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(c.obuf);
        __nv_bfloat16* outb = static_cast<__nv_bfloat16*>(P.out);
        const int nl = warp * 32 + lane;
        const int n0 = ti.fidx * 256 + static_cast<int>(rank) * 128;
        const float* rs = P.row_scale;
        const float ts = FP4 ? __ldg(P.tscale + ti.g) : 1.f;
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + ch * 32, v);
          tmem_ld_wait();
          const int mycol = ch * 32 + lane;
          const float rsv = (rs != nullptr && mycol < ti.ntok) ? rs[ti.row0 + mycol] : 1.f;
          const float my_sc = FP4 ? rsv * ts : rsv;
          named_barrier_sync(1, 128);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sc = __shfl_sync(0xffffffffu, my_sc, j);
            ob[j * 128 + nl] = __float2bfloat16_rn(__uint_as_float(v[j]) * sc);
          }
          named_barrier_sync(1, 128);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int idx = threadIdx.x + 128 * r;
            const int row = idx >> 4, c16 = idx & 15;
            const int col = ch * 32 + row;
            const int n = n0 + c16 * 8;
            if (col < ti.ntok && n < N)
              *reinterpret_cast<uint4*>(outb + static_cast<size_t>(ti.row0 + col) * N + n) = c.obuf[idx];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_leader + static_cast<uint32_t>(acc * sizeof(uint64_t)));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, remote arrives and copies are done
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Tokens for the gate/up MMA: fp16, each aligned 8 of K in the order
// {0, 4, 1, 5, 2, 6, 3, 7}.  One block per row, one thread per 8 values.
// gsrc != NULL: row r is token row gsrc[r] / gk of x (the permutation's
// gather).
__global__ void __launch_bounds__(128)
    int4_tokens_prep_kernel(const __nv_bfloat16* __restrict__ x, int k8, const int32_t* __restrict__ gsrc, int gk,
                            uint4* __restrict__ out) {
  const int r = blockIdx.x;
  const int in_row = gsrc != nullptr ? __ldg(gsrc + r) / gk : r;
  const uint4* in = reinterpret_cast<const uint4*>(x) + static_cast<size_t>(in_row) * k8;
  uint4* o = out + static_cast<size_t>(r) * k8;
  for (int c = threadIdx.x; c < k8; c += blockDim.x) {
    const uint4 v = __ldg(in + c);
    const __half2 p0 = __floats2half2_rn(bf16lo(v.x), bf16lo(v.z));  // x0, x4
    const __half2 p1 = __floats2half2_rn(bf16hi(v.x), bf16hi(v.z));  // x1, x5
    const __half2 p2 = __floats2half2_rn(bf16lo(v.y), bf16lo(v.w));  // x2, x6
    const __half2 p3 = __floats2half2_rn(bf16hi(v.y), bf16hi(v.w));  // x3, x7
    uint4 w;
    w.x = *reinterpret_cast<const uint32_t*>(&p0);
    w.y = *reinterpret_cast<const uint32_t*>(&p1);
    w.z = *reinterpret_cast<const uint32_t*>(&p2);
    w.w = *reinterpret_cast<const uint32_t*>(&p3);
    o[c] = w;
  }
}

bool encode_codes_gu(CUtensorMap* m, const void* q, int groups, int N, int K) {
  // codes [G][2][N][K/2] bytes seen as {K/2, r = 8, u = 2, b = N/8, G}
  const uint64_t row = static_cast<uint64_t>(K) / 2;
  const uint64_t dims[5] = {row, 8, 2, static_cast<uint64_t>(N / 8), static_cast<uint64_t>(groups)};
  const uint64_t strides[4] = {row, row * N, row * 8, row * N * 2};
  const uint32_t box[5] = {CKB * BK / 2, 8, 2, 8, 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_codes_d(CUtensorMap* m, const void* q, int groups, int N, int K) {
  const uint64_t row = static_cast<uint64_t>(K) / 2;
  const uint64_t dims[3] = {row, static_cast<uint64_t>(N), static_cast<uint64_t>(groups)};
  const uint64_t strides[2] = {row, row * N};
  const uint32_t box[3] = {CKB * BK / 2, 128, 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_tokens16(CUtensorMap* m, const void* base, int rows, int K) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t box[2] = {BK, TOK / 2};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <Kind KIND, bool FP4>
int resident_pairs_int4() {
  static int cached[64];
  static bool known[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!known[dev]) {
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof(lc));
    lc.gridDim = dim3(2);
    lc.blockDim = dim3(THREADS);
    lc.dynamicSmemBytes = kSmem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, ffn_int4_pair_kernel<KIND, FP4>, &lc) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cached[dev] = n;
    known[dev] = true;
  }
  return cached[dev];
}

template <Kind KIND, bool FP4>
cudaError_t launch_int4_pair(const void* tokens16, int rows, const int32_t* offsets, int groups, const void* q,
                             const void* scales, const float* tscale, int N, int K, void* out,
                             const float* row_scale, float limit, int32_t* err, int32_t* queue, int num_sms,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (queue == nullptr) return cudaErrorInvalidValue;
  Int4Params P;
  memset(&P, 0, sizeof(P));
  if (!encode_tokens16(&P.tma_x, tokens16, rows, K)) return cudaErrorInvalidValue;
  const bool okq = KIND == Kind::GateUp ? encode_codes_gu(&P.tma_q, q, groups, N, K)
                                        : encode_codes_d(&P.tma_q, q, groups, N, K);
  if (!okq) return cudaErrorInvalidValue;
  P.offsets = offsets;
  P.scales = scales;
  P.tscale = tscale;
  P.out = out;
  P.row_scale = row_scale;
  P.groups = groups;
  P.rows = rows;
  P.n_out = N;
  P.K = K;
  P.k_blocks = K / BK;
  P.f_tiles = KIND == Kind::GateUp ? (N + 127) / 128 : (N + 255) / 256;
  P.limit = limit;
  P.err = err;
  P.queue = queue;
  P.wait_ns = kTimeoutNs;
  cudaError_t e =
      ensure_smem_attr(reinterpret_cast<const void*>(ffn_int4_pair_kernel<KIND, FP4>), static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  int grid = std::max(2, num_sms / 2 * 2);
  const int pairs = resident_pairs_int4<KIND, FP4>();
  if (pairs > 0) grid = std::min(grid, 2 * pairs);
  return launch_kernel(ffn_int4_pair_kernel<KIND, FP4>, dim3(grid), dim3(THREADS), kSmem, stream, P);
}

}  // namespace

// Test hook: one tiny int4 gate/up problem (16 tokens, 64 features, K = 256;
// zero codes, scales and tokens in `scratch`, one expert of 16 rows) on one
// CTA pair whose first (only) accumulator is never signalled to the
// epilogue, with every wait on another role limited to 20 ms.  Both CTAs'
// epilogue waits run out and record MOE_ERR_DEVICE_TIMEOUT (detail 44); the
// token and code producers, the dequantisation warps, the MMA issuer and the
// pair's final cluster barrier finish on their normal paths.
cudaError_t launch_int4_pair_timeout_selftest(void* scratch, int32_t* err, int32_t* queue, cudaStream_t stream) {
  static const int32_t kOffsets[2] = {0, 16};
  unsigned char* base = static_cast<unsigned char*>(scratch);
  void* tokens16 = base + 1024;                             // fp16 [16, 256]
  void* q = base + 10240;                                   // uint8 [1, 2 x 64, 128]
  void* scales = base + 26624;                              // bf16 [1, 2 x 64, 2]
  int32_t* offsets = reinterpret_cast<int32_t*>(base + 27136);  // [0, 16]
  void* h16 = base + 28672;                                 // fp16 [16, 64]
  cudaError_t e = cudaMemcpyAsync(offsets, kOffsets, sizeof(kOffsets), cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return e;
  Int4Params P;
  memset(&P, 0, sizeof(P));
  if (!encode_tokens16(&P.tma_x, tokens16, 16, 256) || !encode_codes_gu(&P.tma_q, q, 1, 64, 256))
    return cudaErrorInvalidValue;
  P.offsets = offsets;
  P.scales = scales;
  P.out = h16;
  P.groups = 1;
  P.rows = 16;
  P.n_out = 64;
  P.K = 256;
  P.k_blocks = 256 / BK;
  P.f_tiles = 1;
  P.limit = 7.f;
  P.err = err;
  P.queue = queue;
  P.wait_ns = 20000000ull;
  P.test_withhold = 1;
  e = ensure_smem_attr(reinterpret_cast<const void*>(ffn_int4_pair_kernel<Kind::GateUp, false>),
                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  ffn_int4_pair_kernel<Kind::GateUp, false><<<2, THREADS, kSmem, stream>>>(P);
  return cudaGetLastError();
}

bool int4_prefill_preferred(int rows, int E) { return rows >= kInt4PrefillRowsPerExpert * E; }

cudaError_t launch_int4_ffn_prefill(const moe_config& cfg, const moe_weights& w, const void* x_rows,
                                    const int32_t* gather_src, const int32_t* offsets, int rows, void* tokens16,
                                    void* h16, const float* w_perm, void* y_perm, int32_t* err, int32_t* queues,
                                    int num_sms, cudaStream_t stream) {
  const int I = cfg.expert_inter, H = cfg.hidden, E = cfg.num_experts;
  if (rows <= 0) return cudaSuccess;
  cudaError_t e = launch_kernel(int4_tokens_prep_kernel, dim3(rows), dim3(128), 0, stream,
                                        static_cast<const __nv_bfloat16*>(x_rows), H / 8, gather_src, cfg.top_k,
                                        static_cast<uint4*>(tokens16));
  if (e != cudaSuccess) return e;
  if (cfg.expert_format == MOE_W_NVFP4) {
    e = launch_int4_pair<Kind::GateUp, true>(tokens16, rows, offsets, E, w.w_gate_up, w.s_gate_up, w.g_gate_up, I, H,
                                             h16, nullptr, cfg.swiglu_limit, err, queues, num_sms, stream);
    if (e != cudaSuccess) return e;
    return launch_int4_pair<Kind::Down, true>(h16, rows, offsets, E, w.w_down, w.s_down, w.g_down, H, I, y_perm,
                                              w_perm, 0.f, err, queues + 2, num_sms, stream);
  }
  e = launch_int4_pair<Kind::GateUp, false>(tokens16, rows, offsets, E, w.w_gate_up, w.s_gate_up, nullptr, I, H, h16,
                                            nullptr, cfg.swiglu_limit, err, queues, num_sms, stream);
  if (e != cudaSuccess) return e;
  return launch_int4_pair<Kind::Down, false>(h16, rows, offsets, E, w.w_down, w.s_down, nullptr, H, I, y_perm, w_perm,
                                             0.f, err, queues + 2, num_sms, stream);
}

}  // namespace moe
