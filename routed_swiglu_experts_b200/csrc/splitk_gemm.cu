// Split-K GEMM with fp32 partial outputs on the sm_100a tensor cores
// (tcgen05 + TMEM + TMA):  part[s][r][n] = sum over K-slice s of
// A[r, k] * B[p, n, k], where the K range is `parts` passes over the
// reduction length, pass p reading slice p of B.  Two users:
//  * router logits: the fp32 router weight split exactly into three bf16
//    parts (hi + mid + lo), so every bf16 x bf16 product is exact and the
//    tensor core accumulates in fp32 ("bridge.models.beam.modeling_beam"
//    beam_router_gating_linear: fp32 operands); parts = 3;
//  * the shared expert for a handful of tokens ("Module glm5next_mlp",
//    FFN_MODULE: the dense SwiGLU FFN also serves the shared expert): with so
//    few rows the projection is bound by streaming its bf16 weight once, so
//    K is split until every SM streams a slice; parts = 1.
// The caller sums the K slices in a fixed order (deterministic).
//
// Tile: 128 A rows x n_mma (<= 256) columns, K step 64 (one 128-byte
// swizzle atom); rows past the end of A are zero-filled by TMA and never
// stored.  Warps 0-3: epilogue (TMEM -> registers -> global fp32), warp 4:
// TMA producer, warp 5: TMEM owner + MMA issuer.  A shared-memory ring of as
// many stages as fit (up to 8) feeds the MMA: with a narrow B (the router's
// E columns) or few A rows (a handful of tokens) a stage is small, and what
// bounds the copy rate is the bytes in flight per SM, not the bytes per
// stage.  When the B slices are narrow (n_mma <= 128) one stage holds the A
// tile and the same K range of every B slice, so A is copied once for all
// passes instead of once per pass, and each slice accumulates into its own
// TMEM columns (the epilogue adds them, smallest first: for the router's
// three-way split of an fp32 weight the small parts keep their bits instead
// of being added into the large running sum).  Two TMEM accumulator sets,
// where they fit, let the epilogue of tile i overlap the MMAs of tile i+1.  Every mbarrier wait is bounded; on
// timeout the kernel records MOE_ERR_DEVICE_TIMEOUT in the workspace error
// word, drains its own in-flight copies and MMAs, frees TMEM and returns.
#include <cstring>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kMaxStages = 8;
constexpr int kRingBytes = 224 * 1024;     // shared-memory ring budget
constexpr int kMaxInnerStageBytes = 64 * 1024;  // B slices share a stage only while 3 stages fit
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct alignas(64) SplitKParams {
  CUtensorMap tma_a;          // A: {K, rows} box {64, 128}
  CUtensorMap tma_b;          // B: {K, N, parts} box {64, n_mma, 1}
  float* out_f32;             // partial logits [k_splits, rows, n_out]
  int32_t rows;
  int32_t n_out;
  int32_t n_mma;              // MMA N (columns of one tile)
  int32_t k_blocks;           // k-blocks of one pass over K
  int32_t parts;              // passes over K (slices of B)
  int32_t k_splits;           // tiles split along the (parts x k-blocks) range
  int32_t kb_per_split;       // K steps per split
  int32_t n_tiles;            // output-column tiles x k_splits
  int32_t stages;             // ring stages (<= kMaxStages)
  int32_t stage_bytes;        // A region + B slices of one stage (multiple of 1024)
  int32_t a_bytes;            // A region of a stage (multiple of 1024)
  int32_t b_bytes;            // one B slice of a stage: n_mma rows x 128 bytes
  int32_t parts_per_stage;    // 1: one B slice per K step; parts: every slice, each into its own accumulator
  int32_t acc_cols;           // TMEM columns of one tile's accumulators (parts_per_stage x n_mma)
  int32_t acc_bufs;           // accumulator sets in TMEM (2: epilogue overlaps the next tile)
  uint32_t idesc;             // MMA instruction descriptor
  int32_t* err;
  int32_t a_box_rows;         // rows per A copy: 128, or fewer when A has fewer rows
  uint64_t timeout_ns;        // limit of every wait on another role's progress
  int32_t test_withhold;      // test hook: never signal the first tile's accumulator
};

struct SmemCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
};

constexpr size_t kSmemMax = 1024 /*align slack*/ + kRingBytes + sizeof(SmemCtl);
static_assert(kSmemMax <= 232448, "fits the 227 KB opt-in shared memory");

struct TileInfo {
  int row0;     // first token row of the tile
  int nrows;    // valid rows (<= BM)
  int nidx;     // output-column tile index
  int split;    // k-split index
};

// Tile order: output-column tile (and k-split) major, row tile minor.
__device__ __forceinline__ TileInfo decode_tile(const SplitKParams& P, int t) {
  TileInfo ti;
  const int mtiles = (P.rows + BM - 1) / BM;
  int nidx = t / mtiles;
  const int m = t - nidx * mtiles;
  ti.row0 = m * BM;
  ti.nrows = min(BM, P.rows - ti.row0);
  ti.split = nidx % P.k_splits;
  ti.nidx = nidx / P.k_splits;
  return ti;
}

// K steps [kb0, kb1) a tile accumulates: of the (parts x k-blocks) range, or
// of the k-blocks alone when every B slice shares the stage.
__device__ __forceinline__ void tile_k_range(const SplitKParams& P, const TileInfo& ti, int& kb0, int& kb1) {
  const int total = P.parts_per_stage == 1 ? P.k_blocks * P.parts : P.k_blocks;
  kb0 = ti.split * P.kb_per_split;
  kb1 = min(total, kb0 + P.kb_per_split);
}

__global__ void __launch_bounds__(THREADS, 1) splitk_gemm_kernel(const __grid_constant__ SplitKParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  const int STAGES = P.stages;
  SmemCtl& c = *reinterpret_cast<SmemCtl*>(smem + STAGES * P.stage_bytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

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
    tma_prefetch_desc(&P.tma_a);
    tma_prefetch_desc(&P.tma_b);
  }
  if (warp == 5) tmem_alloc(&c.tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = c.tmem_base;
  const int total_tiles = ((P.rows + BM - 1) / BM) * P.n_tiles;
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
        const TileInfo ti = decode_tile(P, t);
        const int ncol0 = ti.nidx * P.n_mma;
        int kb0, kb1;
        tile_k_range(P, ti, kb0, kb1);
        // A rows past a_box_rows are not copied: the MMA reads whatever the
        // stage holds there (the B slices that follow A), which only feeds
        // accumulator rows that are never stored
        const int nps = P.parts_per_stage;
        const uint32_t stage_tx = static_cast<uint32_t>((P.a_box_rows + nps * P.n_mma) * BK * 2);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&c.empty[stage], phase ^ 1u, abort_flag, P.timeout_ns)) {
            fail(1);
            ok = false;
            break;
          }
          const int part = nps == 1 ? kb / P.k_blocks : 0;
          const int kc = (kb - part * P.k_blocks) * BK;
          unsigned char* st = smem + stage * P.stage_bytes;
          mbar_arrive_expect_tx(&c.full[stage], stage_tx);
          tma_load_2d(st, &P.tma_a, kc, ti.row0, &c.full[stage]);
          for (int q = 0; q < nps; ++q)
            tma_load_3d(st + P.a_bytes + q * P.b_bytes, &P.tma_b, kc, ncol0, part + q, &c.full[stage]);
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
        const TileInfo ti = decode_tile(P, t);
        const uint32_t idesc = P.idesc;
        int kb0, kb1;
        tile_k_range(P, ti, kb0, kb1);
        if (!mbar_wait_bounded(&c.tmem_empty[acc], acc_phase ^ 1u, abort_flag, P.timeout_ns)) {
          fail(2);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * P.acc_cols);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&c.full[stage], phase, abort_flag, P.timeout_ns)) {
            fail(3);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * P.stage_bytes);
          for (int q = 0; q < P.parts_per_stage; ++q) {
            const uint32_t b_addr = a_addr + static_cast<uint32_t>(P.a_bytes + q * P.b_bytes);
            const uint32_t d_q = d_tmem + static_cast<uint32_t>(q * P.n_mma);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = sw128_kmajor_desc(a_addr + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(b_addr + kk * 32);
              umma_bf16(d_q, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&c.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (!(P.test_withhold && t == static_cast<int>(blockIdx.x))) umma_commit(&c.tmem_full[acc]);
        if (++acc == P.acc_bufs) {
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
      const TileInfo ti = decode_tile(P, t);
      const int ncol0 = ti.nidx * P.n_mma;
      // every lane waits; the outcome is made warp-uniform before the
      // warp-collective TMEM loads
      const bool got = mbar_wait_bounded(&c.tmem_full[acc], acc_phase, abort_flag, P.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) fail(4);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * P.acc_cols);
      const bool row_ok = row_in_tile < ti.nrows;
      const int N = P.n_out;
      const int nch = (P.n_mma + 31) / 32;
      float* frow = P.out_f32 + (static_cast<size_t>(ti.split) * P.rows + ti.row0 + (row_ok ? row_in_tile : 0)) * N;
#pragma unroll 1
      for (int ch = 0; ch < nch; ++ch) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tbase + (P.parts_per_stage - 1) * P.n_mma + ch * 32, v);
        tmem_ld_wait();
        // per-slice accumulators (narrow B): add them from the last slice
        // (smallest terms of the router weight's split) to the first
        for (int q = P.parts_per_stage - 2; q >= 0; --q) {
          uint32_t u[32];
          tmem_ld32(tbase + q * P.n_mma + ch * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(u[j]));
        }
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
      if (++acc == P.acc_bufs) {
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
bool encode_a(CUtensorMap* m, const void* base, int rows, int K, int box_rows = BM) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t box[2] = {BK, static_cast<uint32_t>(box_rows)};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// 3-D bf16 map over [slices, N, K] (K innermost), box 64 x box_n x 1.
bool encode_b(CUtensorMap* m, const void* base, int slices, int N, int K, int box_n) {
  const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(slices)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * N * 2};
  const uint32_t box[3] = {BK, static_cast<uint32_t>(box_n), 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Ring geometry: A region of a_box_rows rows (rounded up to whole 8-row
// swizzle atoms), B slices of n_mma rows; all B slices in one stage when
// that keeps at least three stages, else one slice per stage.  Stage sizes
// are multiples of 1024 bytes (whole swizzle atoms at aligned addresses).
void set_geometry(SplitKParams& P, int n_mma, int parts, int a_box_rows) {
  P.a_bytes = (a_box_rows * BK * 2 + 1023) / 1024 * 1024;
  P.b_bytes = n_mma * BK * 2;
  const int inner = P.a_bytes + parts * P.b_bytes;
  P.parts_per_stage = (parts > 1 && inner <= kMaxInnerStageBytes) ? parts : 1;
  // the M = 128 MMA reads 128 rows of A (16 KB) from the start of a stage
  // whatever a_box_rows is: a stage is never shorter, so that read stays
  // inside the ring
  P.stage_bytes = std::max(P.a_bytes + P.parts_per_stage * P.b_bytes, BM * BK * 2);
  P.stages = std::min(kMaxStages, kRingBytes / P.stage_bytes);
  P.acc_cols = P.parts_per_stage * n_mma;
  P.acc_bufs = 2 * P.acc_cols <= static_cast<int>(TMEM_COLS) ? 2 : 1;
}

size_t smem_bytes(const SplitKParams& P) {
  return 1024 + static_cast<size_t>(P.stages) * P.stage_bytes + sizeof(SmemCtl);
}

}  // namespace

cudaError_t launch_splitk_gemm(const void* a, int rows, int K, const void* b, int parts, int N, int n_mma,
                               int k_splits, float* part, int32_t* err, int num_sms, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  if (n_mma < 16 || n_mma > 256 || n_mma % 16 != 0 || parts < 1) return cudaErrorInvalidValue;
  SplitKParams P;
  memset(&P, 0, sizeof(P));
  // a single row tile with few rows copies only a multiple of 8 rows of it
  const int a_box = rows < BM ? std::max(8, (rows + 7) / 8 * 8) : BM;
  if (!encode_a(&P.tma_a, a, rows, K, a_box)) return cudaErrorInvalidValue;
  P.a_box_rows = a_box;
  if (!encode_b(&P.tma_b, b, parts, N, K, n_mma)) return cudaErrorInvalidValue;
  P.out_f32 = part;
  P.rows = rows;
  P.n_out = N;
  P.n_mma = n_mma;
  P.k_blocks = (K + BK - 1) / BK;
  P.parts = parts;
  set_geometry(P, n_mma, parts, a_box);
  const int total = P.parts_per_stage == 1 ? parts * P.k_blocks : P.k_blocks;
  const int kbps = (total + k_splits - 1) / k_splits;
  P.kb_per_split = kbps;
  P.k_splits = (total + kbps - 1) / kbps;
  P.n_tiles = ((N + n_mma - 1) / n_mma) * P.k_splits;
  P.idesc = umma_idesc_bf16(BM, n_mma);
  P.err = err;
  P.timeout_ns = kTimeoutNs;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(splitk_gemm_kernel), static_cast<int>(kSmemMax));
  if (e != cudaSuccess) return e;
  const int tiles = ((rows + BM - 1) / BM) * P.n_tiles;
  return launch_kernel(splitk_gemm_kernel, dim3(std::min(num_sms, tiles)), dim3(THREADS), smem_bytes(P),
                               stream, P);
}

// Test hook: one 128 x 16 x 64 tile over zero operands in `scratch` whose
// MMA completion is never signalled to the epilogue, with a 20 ms wait limit.
// The epilogue's wait runs out, records MOE_ERR_DEVICE_TIMEOUT (detail 4) in
// *err, and every role leaves through the normal drain: the producer waits
// for its copy, the MMA issuer for its MMAs, TMEM is freed.
cudaError_t launch_splitk_timeout_selftest(void* scratch, int32_t* err, cudaStream_t stream) {
  unsigned char* base = static_cast<unsigned char*>(scratch);
  void* a = base + 1024;                   // bf16 [128, 64]
  void* b = base + 1024 + 128 * 64 * 2;    // bf16 [16, 64]
  float* part = reinterpret_cast<float*>(base + 1024 + 128 * 64 * 2 + 16 * 64 * 2);  // fp32 [128, 16]
  SplitKParams P;
  memset(&P, 0, sizeof(P));
  if (!encode_a(&P.tma_a, a, 128, 64)) return cudaErrorInvalidValue;
  P.a_box_rows = BM;
  if (!encode_b(&P.tma_b, b, 1, 16, 64, 16)) return cudaErrorInvalidValue;
  P.out_f32 = part;
  P.rows = 128;
  P.n_out = 16;
  P.n_mma = 16;
  P.k_blocks = 1;
  P.parts = 1;
  set_geometry(P, 16, 1, BM);
  P.kb_per_split = 1;
  P.k_splits = 1;
  P.n_tiles = 1;
  P.idesc = umma_idesc_bf16(BM, 16);
  P.err = err;
  P.timeout_ns = 20000000ull;
  P.test_withhold = 1;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(splitk_gemm_kernel), static_cast<int>(kSmemMax));
  if (e != cudaSuccess) return e;
  splitk_gemm_kernel<<<1, THREADS, smem_bytes(P), stream>>>(P);
  return cudaGetLastError();
}

int splitk_steps(int K, int parts, int n_mma, int rows) {
  SplitKParams P;
  memset(&P, 0, sizeof(P));
  set_geometry(P, n_mma, parts, rows < BM ? std::max(8, (rows + 7) / 8 * 8) : BM);
  const int kb = (K + BK - 1) / BK;
  return P.parts_per_stage == 1 ? parts * kb : kb;
}

int splitk_actual_splits(int K, int parts, int n_mma, int rows, int k_splits) {
  const int total = splitk_steps(K, parts, n_mma, rows);
  const int kbps = (total + k_splits - 1) / k_splits;
  return (total + kbps - 1) / kbps;
}

cudaError_t launch_router_gemm(const void* x, int T, int H, const void* w_split, int E, int k_splits, float* part,
                               int32_t* err, int num_sms, cudaStream_t stream) {
  return launch_splitk_gemm(x, T, H, w_split, 3, E, router_mma_n(E), k_splits, part, err, num_sms, stream);
}

int router_actual_splits(int T, int E, int H, int k_splits) {
  return splitk_actual_splits(H, 3, router_mma_n(E), T, k_splits);
}

}  // namespace moe
