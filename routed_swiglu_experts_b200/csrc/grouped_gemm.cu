// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Module glm5next_mlp", forward_prefill_gemm: one launch per projection for
// all experts, driven by per-expert tables over global expert ids.  Here the
// table is the expert row offsets produced by the permute; the weights of
// expert g are slice g of one stacked tensor, addressed by a 3-D TMA map.
//
// Three kernels share one persistent, warp-specialised design:
//   gate/up:  h = bf16( silu(min(X Wg^T, L)) * clamp(X Wu^T, -L, L) )
//             ("Module glm5next_mlp" §Numerics: asymmetric SwiGLU clamp;
//              "mstar.model.components.distributed.mlp" ParallelGatedMLP:
//              fused gate/up projection, gate = shard 0, up = shard 1)
//   down:     y = bf16( row_scale[r] * (H Wd^T) )   (combine weight fused)
//   router:   fp32 partial logits of x Wr^T with the fp32 router weight
//             split exactly into three bf16 parts (hi + mid + lo) that are
//             concatenated along K, so bf16 x bf16 products are exact and
//             the tensor core accumulates in fp32 ("bridge.models.beam.
//             modeling_beam" beam_router_gating_linear: fp32 operands);
//             K is split across CTAs for small token counts.
//
// Tile: 128 rows x 256 accumulator columns (gate/up: 128 gate + 128 up
// columns of the same intermediate slice; down: 256 hidden columns), K step
// 64 (one 128-byte swizzle atom).  Warps 0-3: epilogue (TMEM -> registers
// -> global), warp 4: TMA producer, warp 5: TMEM owner + MMA issuer.  A
// 4-stage smem ring (48 KB/stage) feeds the MMA; two 256-column TMEM
// accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
// Every mbarrier wait is bounded; on timeout the kernel records
// MOE_ERR_DEVICE_TIMEOUT in the workspace error word, drains its own
// in-flight copies and MMAs, frees TMEM and returns.
#include <cstring>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int MMA_N = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_BYTES = MMA_N * BK * 2;    // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;

enum class Mode { GateUp, Down, Router };

struct alignas(64) GemmParams {
  CUtensorMap tma_a[2];
  CUtensorMap tma_b[2];
  const int32_t* offsets[2];  // grouped problem: [groups+1]; else nullptr
  __nv_bfloat16* out[2];
  const float* row_scale[2];
  float* out_f32;             // router: partial logits [k_splits, rows, n_out]
  int32_t groups[2];
  int32_t rows[2];
  int32_t n_out[2];
  int32_t k_blocks[2];        // k-blocks of one pass over K (router: per part)
  int32_t k_parts[2];         // K repetitions with different B slices (router: 3)
  int32_t k_splits[2];        // tiles split along the (parts x k-blocks) range
  int32_t kb_per_split[2];
  int32_t n_tiles[2];         // output-column tiles x k_splits
  uint32_t idesc[2];          // MMA instruction descriptor (N per problem)
  int32_t b_bytes[2];         // bytes of one B stage
  int32_t nprob;
  float limit;
  int32_t* err;
};

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t tiles[2];
  int32_t off[MOE_MAX_EXPERTS + 1];
  int32_t mt[MOE_MAX_EXPERTS + 1];
};

constexpr size_t kSmemBytes = 1024 /*align slack*/ + STAGES * STAGE_BYTES + sizeof(SmemCtl);
static_assert(kSmemBytes <= 232448, "fits the 227 KB opt-in shared memory");

struct TileInfo {
  int p;        // problem
  int g;        // group (expert) inside the problem
  int row0;     // first A row of the tile
  int nrows;    // valid rows (<= BM)
  int nidx;     // output-column tile index
  int split;    // k-split index
};

// Tile order: problem 0 then problem 1; inside a problem, group by group;
// inside a group, output-column tile major, row tile minor (the row tiles of
// one weight slice run back to back and share it through L2).
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& P, const SmemCtl& c, int t) {
  TileInfo ti;
  ti.p = 0;
  if (t >= c.tiles[0]) {
    t -= c.tiles[0];
    ti.p = 1;
  }
  const int nt = P.n_tiles[ti.p];
  int m, r0, r1;
  if (P.offsets[ti.p] != nullptr) {
    const int G = P.groups[ti.p];
    const int u = t / nt;
    int lo = 0, hi = G;  // g with mt[g] <= u < mt[g+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (c.mt[mid] <= u) lo = mid; else hi = mid;
    }
    const int g = lo;
    const int mtg = c.mt[g + 1] - c.mt[g];
    const int local = t - c.mt[g] * nt;
    ti.nidx = local / mtg;
    m = local - ti.nidx * mtg;
    ti.g = g;
    r0 = c.off[g];
    r1 = c.off[g + 1];
  } else {
    const int mtg = (P.rows[ti.p] + BM - 1) / BM;
    ti.nidx = t / mtg;
    m = t - ti.nidx * mtg;
    ti.g = 0;
    r0 = 0;
    r1 = P.rows[ti.p];
  }
  ti.row0 = r0 + m * BM;
  ti.nrows = min(BM, r1 - ti.row0);
  const int ks = P.k_splits[ti.p];
  ti.split = ti.nidx % ks;
  ti.nidx /= ks;
  return ti;
}

// k-blocks [kb0, kb1) of the (parts x k-blocks) range a tile accumulates.
__device__ __forceinline__ void tile_k_range(const GemmParams& P, const TileInfo& ti, int& kb0, int& kb1) {
  const int total = P.k_blocks[ti.p] * P.k_parts[ti.p];
  kb0 = ti.split * P.kb_per_split[ti.p];
  kb1 = min(total, kb0 + P.kb_per_split[ti.p]);
}

template <Mode MODE>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* smem_a = smem;
  unsigned char* smem_b = smem + STAGES * A_BYTES;
  SmemCtl& c = *reinterpret_cast<SmemCtl*>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  constexpr int BN_OUT = MODE == Mode::GateUp ? 128 : 256;  // router: the problem's MMA N (<= 256)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&c.tmem_full[a], 1);
      mbar_init(&c.tmem_empty[a], 4 * 32);
    }
    mbar_init(&c.mma_done, 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tma_a[p]);
      tma_prefetch_desc(&P.tma_b[p]);
    }
  }
  // per-problem tile counts; grouped problems get (offsets, m-tile prefix)
  if (warp == 0) {
    for (int p = 0; p < 2; ++p) {
      int tiles = 0;
      if (p < P.nprob) {
        if (P.offsets[p] != nullptr) {
          const int G = P.groups[p];
          const int per = (G + 31) / 32;
          int local = 0;
          for (int j = 0; j < per; ++j) {
            const int g = lane * per + j;
            if (g < G) {
              const int o0 = P.offsets[p][g], o1 = P.offsets[p][g + 1];
              c.off[g] = o0;
              local += (o1 - o0 + BM - 1) / BM;
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
              c.mt[g] = run;
              run += (P.offsets[p][g + 1] - P.offsets[p][g] + BM - 1) / BM;
            }
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          if (lane == 0) {
            c.off[G] = P.offsets[p][G];
            c.mt[G] = total;
          }
          tiles = total * P.n_tiles[p];
        } else {
          tiles = ((P.rows[p] + BM - 1) / BM) * P.n_tiles[p];
        }
      }
      if (lane == 0) c.tiles[p] = tiles;
    }
  }
  if (warp == 5) tmem_alloc(&c.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = c.tmem_base;
  const int total_tiles = c.tiles[0] + c.tiles[1];
  volatile int32_t* abort_flag = &c.abort_flag;

  auto fail = [&](int detail) {
    *abort_flag = 1;
    report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, detail);
  };

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(P, c, t);
        const int p = ti.p;
        const int ncol0 = ti.nidx * (MODE == Mode::Router ? (P.b_bytes[p] / (BK * 2)) : BN_OUT);
        int kb0, kb1;
        tile_k_range(P, ti, kb0, kb1);
        const uint32_t stage_tx = static_cast<uint32_t>(A_BYTES + P.b_bytes[p]);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&c.empty[stage], phase ^ 1u, abort_flag, kTimeoutNs)) {
            fail(1);
            ok = false;
            break;
          }
          const int part = kb / P.k_blocks[p];
          const int kc = (kb - part * P.k_blocks[p]) * BK;
          mbar_arrive_expect_tx(&c.full[stage], stage_tx);
          tma_load_2d(smem_a + stage * A_BYTES, &P.tma_a[p], kc, ti.row0, &c.full[stage]);
          if (MODE == Mode::GateUp) {
            tma_load_3d(smem_b + stage * B_BYTES, &P.tma_b[p], kc, ncol0, 2 * ti.g, &c.full[stage]);
            tma_load_3d(smem_b + stage * B_BYTES + B_BYTES / 2, &P.tma_b[p], kc, ncol0, 2 * ti.g + 1,
                        &c.full[stage]);
          } else if (MODE == Mode::Down) {
            tma_load_3d(smem_b + stage * B_BYTES, &P.tma_b[p], kc, ncol0, ti.g, &c.full[stage]);
          } else {
            tma_load_3d(smem_b + stage * B_BYTES, &P.tma_b[p], kc, ncol0, part, &c.full[stage]);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // drain: wait (bounded) for the last copy issued to each stage
      const int nst = issued < STAGES ? issued : STAGES;
      for (int j = 0; j < nst; ++j) {
        const int i = issued - 1 - j;
        const int s = i % STAGES;
        const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
        volatile int32_t never = 0;
        if (!mbar_wait_bounded(&c.full[s], par, &never, kTimeoutNs)) report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 9);
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(P, c, t);
        const int p = ti.p;
        const uint32_t idesc = P.idesc[p];
        int kb0, kb1;
        tile_k_range(P, ti, kb0, kb1);
        if (!mbar_wait_bounded(&c.tmem_empty[acc], acc_phase ^ 1u, abort_flag, kTimeoutNs)) {
          fail(2);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MMA_N);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&c.full[stage], phase, abort_flag, kTimeoutNs)) {
            fail(3);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem_a + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(smem_b + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sw128_kmajor_desc(a_addr + kk * 32);
            const uint64_t bd = sw128_kmajor_desc(b_addr + kk * 32);
            umma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&c.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&c.tmem_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // drain every MMA this thread issued before TMEM is released
      umma_commit(&c.mma_done);
      volatile int32_t never = 0;
      if (!mbar_wait_bounded(&c.mma_done, 0, &never, kTimeoutNs)) report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 8);
    }
  } else {
    // ------------------------------------------- epilogue (warps 0 .. 3) --
    int acc = 0;
    uint32_t acc_phase = 0;
    const int row_in_tile = warp * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const TileInfo ti = decode_tile(P, c, t);
      const int p = ti.p;
      const int ncol0 = ti.nidx * (MODE == Mode::Router ? (P.b_bytes[p] / (BK * 2)) : BN_OUT);
      // every lane waits; the outcome is made warp-uniform before the
      // warp-collective TMEM loads
      const bool got = mbar_wait_bounded(&c.tmem_full[acc], acc_phase, abort_flag, kTimeoutNs);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) fail(4);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * MMA_N);
      const bool row_ok = row_in_tile < ti.nrows;
      const int N = P.n_out[p];
      __nv_bfloat16* orow = P.out[p] + static_cast<size_t>(ti.row0 + (row_ok ? row_in_tile : 0)) * N;
      if (MODE == Mode::GateUp) {
        const float L = P.limit;
#pragma unroll 1
        for (int ch = 0; ch < BN_OUT / 32; ++ch) {
          uint32_t g[32], u[32];
          __syncwarp();
          tmem_ld32(tbase + ch * 32, g);
          tmem_ld32(tbase + 128 + ch * 32, u);
          tmem_ld_wait();
          if (ch == BN_OUT / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&c.tmem_empty[acc]);
          }
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float h2[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float gv = __uint_as_float(g[2 * j + q]);
              float uv = __uint_as_float(u[2 * j + q]);
              gv = fminf(gv, L);
              uv = fminf(fmaxf(uv, -L), L);
              h2[q] = __fdividef(gv, 1.f + __expf(-gv)) * uv;
            }
            packed[j] = pack_bf16x2(h2[0], h2[1]);
          }
          const int col = ncol0 + ch * 32;
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (col + 8 * q < N)
                *reinterpret_cast<uint4*>(orow + col + 8 * q) =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          }
        }
      } else if (MODE == Mode::Down) {
        const float* rs = P.row_scale[p];
        const float scale = (rs != nullptr && row_ok) ? rs[ti.row0 + row_in_tile] : 1.f;
#pragma unroll 1
        for (int ch = 0; ch < BN_OUT / 32; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + ch * 32, v);
          tmem_ld_wait();
          if (ch == BN_OUT / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&c.tmem_empty[acc]);
          }
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            packed[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * scale, __uint_as_float(v[2 * j + 1]) * scale);
          const int col = ncol0 + ch * 32;
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (col + 8 * q < N)
                *reinterpret_cast<uint4*>(orow + col + 8 * q) =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          }
        }
      } else {
        // router: fp32 partial logits of this k-split
        const int n_mma = P.b_bytes[p] / (BK * 2);
        const int nch = (n_mma + 31) / 32;
        float* frow = P.out_f32 + (static_cast<size_t>(ti.split) * P.rows[p] + ti.row0 + (row_ok ? row_in_tile : 0)) * N;
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + ch * 32, v);
          tmem_ld_wait();
          if (ch == nch - 1) {
            tc_fence_before();
            mbar_arrive(&c.tmem_empty[acc]);
          }
          const int col = ncol0 + ch * 32;
          if (row_ok) {
            if ((N & 3) == 0) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (col + 4 * q < N)
                  *reinterpret_cast<uint4*>(frow + col + 4 * q) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2],
                                                                             v[4 * q + 3]);
            } else {
#pragma unroll
              for (int q = 0; q < 32; ++q)
                if (col + q < N) frow[col + q] = __uint_as_float(v[q]);
            }
          }
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host --

// 2-D bf16 map over [rows, K] (K innermost), box 64 x 128, 128-byte swizzle.
bool encode_a(CUtensorMap* m, const void* base, int rows, int K) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t box[2] = {BK, BM};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// 3-D bf16 map over [slices, N, K] (K innermost), box 64 x box_n x 1.
bool encode_b(CUtensorMap* m, const void* base, int slices, int N, int K, int box_n) {
  const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(slices)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * N * 2};
  const uint32_t box[3] = {BK, static_cast<uint32_t>(box_n), 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <Mode MODE>
cudaError_t launch_impl(const FfnProblem* routed, const FfnProblem* shared, float limit, int32_t* err, int num_sms,
                        cudaStream_t stream) {
  GemmParams P;
  memset(&P, 0, sizeof(P));
  const FfnProblem* probs[2];
  int np = 0;
  if (shared != nullptr && shared->rows > 0) probs[np++] = shared;  // longer tiles first
  if (routed != nullptr && routed->rows > 0) probs[np++] = routed;
  if (np == 0) return cudaSuccess;
  constexpr int BN_OUT = MODE == Mode::GateUp ? 128 : 256;
  for (int i = 0; i < np; ++i) {
    const FfnProblem& f = *probs[i];
    if (!encode_a(&P.tma_a[i], f.a, f.rows, f.K)) return cudaErrorInvalidValue;
    const bool okb = MODE == Mode::GateUp ? encode_b(&P.tma_b[i], f.w, 2 * f.groups, f.N, f.K, 128)
                                          : encode_b(&P.tma_b[i], f.w, f.groups, f.N, f.K, 256);
    if (!okb) return cudaErrorInvalidValue;
    P.offsets[i] = f.offsets;
    P.out[i] = static_cast<__nv_bfloat16*>(f.out);
    P.row_scale[i] = f.row_scale;
    P.groups[i] = f.groups;
    P.rows[i] = f.rows;
    P.n_out[i] = f.N;
    P.k_blocks[i] = (f.K + BK - 1) / BK;
    P.k_parts[i] = 1;
    P.k_splits[i] = 1;
    P.kb_per_split[i] = P.k_blocks[i];
    P.n_tiles[i] = (f.N + BN_OUT - 1) / BN_OUT;
    P.idesc[i] = umma_idesc_bf16(BM, MMA_N);
    P.b_bytes[i] = B_BYTES;
  }
  P.nprob = np;
  P.limit = limit;
  P.err = err;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(grouped_gemm_kernel<MODE>),
                                   static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  grouped_gemm_kernel<MODE><<<num_sms, THREADS, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_gemm(const void* x, int T, int H, const void* w_split, int E, int k_splits, float* part,
                               int32_t* err, int num_sms, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  GemmParams P;
  memset(&P, 0, sizeof(P));
  const int n_mma = router_mma_n(E);
  if (!encode_a(&P.tma_a[0], x, T, H)) return cudaErrorInvalidValue;
  if (!encode_b(&P.tma_b[0], w_split, 3, E, H, n_mma)) return cudaErrorInvalidValue;
  P.offsets[0] = nullptr;
  P.out_f32 = part;
  P.groups[0] = 1;
  P.rows[0] = T;
  P.n_out[0] = E;
  P.k_blocks[0] = (H + BK - 1) / BK;
  P.k_parts[0] = 3;
  const int total = 3 * P.k_blocks[0];
  const int kbps = (total + k_splits - 1) / k_splits;
  P.kb_per_split[0] = kbps;
  P.k_splits[0] = (total + kbps - 1) / kbps;
  P.n_tiles[0] = ((E + n_mma - 1) / n_mma) * P.k_splits[0];
  P.idesc[0] = umma_idesc_bf16(BM, n_mma);
  P.b_bytes[0] = n_mma * BK * 2;
  P.nprob = 1;
  P.err = err;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(grouped_gemm_kernel<Mode::Router>),
                                   static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int tiles = ((T + BM - 1) / BM) * P.n_tiles[0];
  grouped_gemm_kernel<Mode::Router><<<std::min(num_sms, tiles), THREADS, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

int router_actual_splits(int H, int k_splits) {
  const int total = 3 * ((H + BK - 1) / BK);
  const int kbps = (total + k_splits - 1) / k_splits;
  return (total + kbps - 1) / kbps;
}

cudaError_t launch_gemm_gateup(const FfnProblem* routed, const FfnProblem* shared, float limit, int32_t* err,
                               int num_sms, cudaStream_t stream) {
  return launch_impl<Mode::GateUp>(routed, shared, limit, err, num_sms, stream);
}

cudaError_t launch_gemm_down(const FfnProblem* routed, const FfnProblem* shared, int32_t* err, int num_sms,
                             cudaStream_t stream) {
  return launch_impl<Mode::Down>(routed, shared, 0.f, err, num_sms, stream);
}

}  // namespace moe
