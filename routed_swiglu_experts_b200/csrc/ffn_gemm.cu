// Grouped expert FFN GEMMs on CTA pairs (tcgen05.mma.cta_group::2), weights
// as the M operand and tokens as N ("swap AB").
//
// "Module glm5next_mlp", forward_prefill_gemm: one launch per projection for
// all experts; the expert row offsets from the permute drive the tiles.
//   gate/up:  h[t, f] = bf16( silu(min(G, L)) * clamp(U, -L, L) )
//             ("Module glm5next_mlp" §Numerics: asymmetric clamp;
//              "mstar.model.components.distributed.mlp" ParallelGatedMLP:
//              gate = shard 0, up = shard 1 of the fused projection)
//   down:     y[t, n] = bf16( row_scale[t] * sum_i W_d[n, i] h[t, i] )
//
// Why this shape.  A tile is 256 weight rows x up to 256 tokens of one
// expert, computed by a pair of CTAs on two SMs: each CTA loads its own 128
// weight rows (the A half) and half of the token rows (the B half) -- 32 KB
// per 64-wide K step for 2 MFLOP, half the shared-memory traffic per FLOP of
// a single-CTA 128 x 256 tile -- and the MMA issued by the pair's first CTA
// reads both halves.  Tokens are the N dimension, so a tile's token count is
// rounded up to 16 only: the ragged last tile of each expert wastes at most
// 15 token columns instead of up to 127 rows.
//
// Roles per CTA (192 threads): warps 0-3 epilogue (TMEM -> registers ->
// global), warp 4 TMA producer, warp 5 TMEM owner (+ MMA issuer in the first
// CTA).  3-stage ring of 64 KB, each stage two 64-deep K chunks of weights
// and tokens (one barrier round trip and one commit per 128 of K: the
// per-step handshake, not the bytes, is what a tile pays whatever its token
// count; 6 stages of 32 KB ran 2-4% slower); two 256-column fp32
// accumulators per CTA.
// Persistent: one pair per two SMs takes tiles from a queue (an atomic
// counter in the workspace header) in the fixed tile order below, so the
// pairs that draw ragged last tiles take more of them; a fixed round-robin
// split of the same order left whole pairs with only full tiles (an even
// pair count against an even tile count per expert).  The first CTA's
// producer takes each id and hands it to every role of both CTAs through a
// small ring of ids guarded by mbarriers.
// gate/up weight rows of a CTA cover 64 features, loaded through a 5-D view of
// the [gate; up] weight so that shared-memory row 16b + 8u + r is the gate
// (u = 0) or up (u = 1) row of feature 8b + r.  A 16-lane TMEM load then hands
// every thread the gate AND the up accumulator of one feature, and all four
// epilogue warps apply the SwiGLU without any exchange.
// Every mbarrier wait is bounded (MOE_ERR_DEVICE_TIMEOUT on expiry).
#include <cstring>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BK = 64;
constexpr int ROWS = 128;                  // weight rows per CTA (A half)
constexpr int TOK = 256;                   // tokens per pair tile (MMA N <= 256)
constexpr int KCH = 2;                     // 64-deep K chunks per pipeline stage
constexpr int STAGES = 6 / KCH;
constexpr int A_BYTES = ROWS * BK * 2;     // 16 KB per chunk
constexpr int B_BYTES = (TOK / 2) * BK * 2;  // 16 KB per chunk: this CTA's half of the tokens
constexpr int A_STAGE = KCH * A_BYTES;
constexpr int B_STAGE = KCH * B_BYTES;
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr int HPITCH = 144;                // bytes per token row of the staged gate/up output (64 bf16 + pad)
constexpr int QD = 8;                      // tile-id ring depth
// readers of every tile id: the MMA issuer and 4 epilogue warps of the first
// CTA, the TMA producer and 4 epilogue warps of the second
constexpr uint32_t kTileReaders = 1 + 4 + 1 + 4;

enum class Kind { GateUp, Down };

// Token boxes of 128, 64, 32, 16 and 8 rows: each CTA of a pair copies the
// smallest box that holds its nmma / 2 token rows, so a ragged last tile of
// an expert moves fewer bytes through L2 into shared memory (one copy per
// chunk either way).
constexpr int kTokBoxes = 5;
__host__ __device__ constexpr int tok_box_index(int rows_per_cta) {
  return rows_per_cta > 64 ? 0 : rows_per_cta > 32 ? 1 : rows_per_cta > 16 ? 2 : rows_per_cta > 8 ? 3 : 4;
}

struct alignas(64) PairParams {
  CUtensorMap tma_w[2];       // weights: gate/up {K, 8, 2, N/8, G} box {64, 8, 2, 8, 1}; down {K, N, G} box {64, 128, 1}
  CUtensorMap tma_x[2][kTokBoxes];  // tokens {K, rows} box {64, 128 >> i}: a tile copies only the rows it uses;
                                    // gathered problem: [0] only, {K, tokens} box {64, 1}
  const int32_t* offsets[2];  // grouped problem: [groups+1]; else nullptr
  const int32_t* gsrc[2];     // gathered problem: slot of each permuted row (token = slot / gk); else nullptr
  int32_t gk[2];              // slots per token of a gathered problem
  __nv_bfloat16* out[2];      // [rows, N]
  const float* row_scale[2];  // down: per token row (or nullptr)
  int32_t groups[2];
  int32_t rows[2];
  int32_t n_out[2];           // N: I (gate/up) or H (down)
  int32_t k_blocks[2];
  int32_t f_tiles[2];         // weight-row tiles per group (pair covers 128 features / 256 rows)
  int32_t nprob;
  float limit;
  int32_t* err;
  int32_t* queue;             // {next tile, pairs retired}: zero at launch, left zero at exit
  uint64_t wait_ns;           // limit of every wait on another role's progress
  int32_t test_withhold;      // test hook: never signal the first tile's accumulator to the epilogue
};

struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint64_t tq_full[QD];             // tile id published (one arrive)
  uint64_t tq_empty[QD];            // first CTA: every reader has taken it
  int32_t tq[QD];                   // tile ids; -1 = no more tiles
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t tiles[2];
  int32_t off[MOE_MAX_EXPERTS + 1];
  int32_t tp[MOE_MAX_EXPERTS + 1];  // token-tile prefix per group
  uint4 obuf[512];                  // one 32-token chunk of bf16 output, row-major
};

constexpr size_t kSmem = 1024 + STAGES * STAGE_BYTES + sizeof(Ctl);
static_assert(kSmem <= 232448, "fits the 227 KB opt-in shared memory");

struct Tile {
  int p, g, fidx, row0, ntok, nmma;
};

// Tile order: problem 0 then 1; group by group; inside a group weight-row
// tile major, token tile minor (the token tiles of one weight slice are
// handed out back to back, run at the same time on neighbouring pairs and
// share it through L2).
__device__ __forceinline__ Tile decode(const PairParams& P, const Ctl& c, int t) {
  Tile ti;
  ti.p = 0;
  if (t >= c.tiles[0]) {
    t -= c.tiles[0];
    ti.p = 1;
  }
  const int nf = P.f_tiles[ti.p];
  int tm, tmi, r0, r1;
  if (P.offsets[ti.p] != nullptr) {
    const int G = P.groups[ti.p];
    const int u = t / nf;
    int lo = 0, hi = G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (c.tp[mid] <= u) lo = mid; else hi = mid;
    }
    ti.g = lo;
    tm = c.tp[lo + 1] - c.tp[lo];
    const int local = t - c.tp[lo] * nf;
    ti.fidx = local / tm;
    tmi = local - ti.fidx * tm;
    r0 = c.off[lo];
    r1 = c.off[lo + 1];
  } else {
    tm = (P.rows[ti.p] + TOK - 1) / TOK;
    ti.g = 0;
    ti.fidx = t / tm;
    tmi = t - ti.fidx * tm;
    r0 = 0;
    r1 = P.rows[ti.p];
  }
  ti.row0 = r0 + tmi * TOK;
  ti.ntok = min(TOK, r1 - ti.row0);
  ti.nmma = (ti.ntok + 15) / 16 * 16;
  return ti;
}

// GATHER: some problem of the launch reads its token rows through gsrc
// (then the whole producer warp copies; otherwise its lane 0 alone).
template <Kind KIND, bool GATHER>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    ffn_pair_kernel(const __grid_constant__ PairParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* smem_a = smem;
  unsigned char* smem_b = smem + STAGES * A_STAGE;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
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
    for (int p = 0; p < P.nprob; ++p) {
      tma_prefetch_desc(&P.tma_w[p]);
      for (int b = 0; b < (P.gsrc[p] != nullptr ? 1 : kTokBoxes); ++b) tma_prefetch_desc(&P.tma_x[p][b]);
    }
  }
  if (warp == 5) tmem_alloc_pair(&c.tmem_base, TMEM_COLS);
  if (warp == 0) {  // per-problem tile counts; grouped problems: offsets + token-tile prefix
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
              run += (P.offsets[p][g + 1] - P.offsets[p][g] + TOK - 1) / TOK;
            }
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          if (lane == 0) {
            c.off[G] = P.offsets[p][G];
            c.tp[G] = total;
          }
          tiles = total * P.f_tiles[p];
        } else {
          tiles = ((P.rows[p] + TOK - 1) / TOK) * P.f_tiles[p];
        }
      }
      if (lane == 0) c.tiles[p] = tiles;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
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
    // Lane 0 takes the tile ids, waits on the ring and copies the weights
    // (and a contiguous token box).  For a gathered problem every lane copies
    // token rows 4 lane .. 4 lane + 3 of the CTA's half with one tile::gather4
    // per chunk, the hidden rows of the tokens the permutation put there.
    if (GATHER || lane == 0) {  // lanes 1-31 only help gathers
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      int q = 0;
      uint32_t qph = 0;
      int t_next = -2;  // next queue position, once fetched (lane 0)
      for (;;) {
        // Next tile: the first CTA takes it from the launch's queue and
        // publishes it to both CTAs; tiles go out in order to whichever pair
        // asks first, so pairs that drew cheap (ragged) tiles take more.
        int t = -1;
        int got = 1;
        if (lane == 0) {
          if (leader) {
            if (!mbar_wait_bounded<true>(&c.tq_empty[q], qph ^ 1u, abort_flag, P.wait_ns)) {
              fail(35);
              got = 0;
            } else {
              if (t_next == -2) t_next = atomicAdd(P.queue, 1);
              t = t_next < total_tiles ? t_next : -1;
              t_next = -2;
              c.tq[q] = t;
              st_cluster_u32(map_to_rank(smem_u32(&c.tq[q]), 1), static_cast<uint32_t>(t));
              mbar_arrive_cluster(map_to_rank(smem_u32(&c.tq_full[q]), 1));
              mbar_arrive(&c.tq_full[q]);
            }
          } else {
            if (!mbar_wait_bounded<true>(&c.tq_full[q], qph, abort_flag, P.wait_ns)) {
              fail(36);
              got = 0;
            } else {
              t = c.tq[q];
              mbar_arrive_cluster(leader_bar(&c.tq_empty[q]));
            }
          }
        }
        if (GATHER) {
          got = __shfl_sync(0xffffffffu, got, 0);
          t = __shfl_sync(0xffffffffu, t, 0);
        }
        if (!got) break;
        if (++q == QD) {
          q = 0;
          qph ^= 1u;
        }
        if (t < 0) break;
        const Tile ti = decode(P, c, t);
        const int p = ti.p;
        const int half = ti.nmma / 2;  // token rows of this CTA (a multiple of 8)
        const int xrow = ti.row0 + static_cast<int>(rank) * half;
        const bool gather = GATHER && P.gsrc[p] != nullptr;
        const bool my_rows = gather && 4 * lane < half;
        int g[4] = {0, 0, 0, 0};
        if (my_rows) {
          // token of permuted row r = slot src[r] / top_k; rows past the
          // problem's end (padding up to nmma) read token 0 and are never stored
  #pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = xrow + 4 * lane + j;
            g[j] = r < P.rows[p] ? __ldg(P.gsrc[p] + r) / P.gk[p] : 0;
          }
        }
        // the next id is fetched a few stages before this tile's last copy,
        // so the atomic's round trip overlaps the copies
        const int nkb = P.k_blocks[p];
        const int nstage = (nkb + KCH - 1) / KCH;  // the last stage of an odd count holds one chunk
        const int kpre = nstage > 2 ? nstage - 2 : 0;
        const int xb = tok_box_index(half);
        // this CTA's token bytes per chunk: its rows exactly (gather) or its box
        const uint32_t b_bytes = static_cast<uint32_t>(gather ? half : (TOK / 2) >> xb) * BK * 2;
        for (int st = 0; st < nstage; ++st) {
          int w_ok = 1;
          if (lane == 0) {
            if (!mbar_wait_bounded(&c.empty[stage], phase ^ 1u, abort_flag, P.wait_ns)) {
              fail(31);
              w_ok = 0;
            }
          }
          if (GATHER) w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
          if (!w_ok) {
            ok = false;
            break;
          }
          const int nk = min(KCH, nkb - st * KCH);
          if (lane == 0 && leader)
            mbar_arrive_expect_tx(&c.full[stage], 2u * static_cast<uint32_t>(nk) * (A_BYTES + b_bytes));
          const uint32_t bar = leader_bar(&c.full[stage]);
          for (int ch = 0; ch < nk; ++ch) {
            const int kc = (st * KCH + ch) * BK;
            unsigned char* sb = smem_b + stage * B_STAGE + ch * B_BYTES;  // 1024-byte aligned
            if (lane == 0) {
              unsigned char* sa = smem_a + stage * A_STAGE + ch * A_BYTES;  // 1024-byte aligned
              if (KIND == Kind::GateUp) {
                const int fb = ti.fidx * 16 + static_cast<int>(rank) * 8;  // first 8-feature block
                tma_load_5d_pair(sa, &P.tma_w[p], kc, 0, 0, fb, ti.g, bar);
              } else {
                const int n = ti.fidx * 256 + static_cast<int>(rank) * 128;
                tma_load_3d_pair(sa, &P.tma_w[p], kc, n, ti.g, bar);
              }
              if (!gather) tma_load_2d_pair(sb, &P.tma_x[p][xb], kc, xrow, bar);
            }
            if (my_rows) tma_gather4_pair(sb + lane * 512, &P.tma_x[p][0], kc, g[0], g[1], g[2], g[3], bar);
          }
          if (lane == 0 && leader && st == kpre) t_next = atomicAdd(P.queue, 1);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (lane == 0 && leader) {
        // retire from the queue; the last pair of the launch resets it (every
        // pair has taken its final tile id before it retires)
        __threadfence();
        if (atomicAdd(P.queue + 1, 1) == npairs - 1) {
          __threadfence();
          atomicExch(P.queue, 0);
          atomicExch(P.queue + 1, 0);
        }
        // drain: the last copy of each stage (both CTAs' bytes land here)
        const int nst = issued < STAGES ? issued : STAGES;
        for (int j = 0; j < nst; ++j) {
          const int i = issued - 1 - j;
          volatile int32_t never = 0;
          if (!mbar_wait_bounded(&c.full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1), &never, kTimeoutNs))
            report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 39);
        }
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
        if (!mbar_wait_bounded(&c.tq_full[q], qph, abort_flag, P.wait_ns)) {
          fail(37);
          break;
        }
        const int t = c.tq[q];
        mbar_arrive(&c.tq_empty[q]);
        if (++q == QD) {
          q = 0;
          qph ^= 1u;
        }
        if (t < 0) break;
        const Tile ti = decode(P, c, t);
        const int p = ti.p;
        const uint32_t idesc = umma_idesc_bf16(2 * ROWS, ti.nmma);
        if (!mbar_wait_bounded(&c.tmem_empty[acc], acc_phase ^ 1u, abort_flag, P.wait_ns)) {
          fail(32);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        const int nkb = P.k_blocks[p];
        const int nstage = (nkb + KCH - 1) / KCH;
        for (int st = 0; st < nstage; ++st) {
          if (!mbar_wait_bounded(&c.full[stage], phase, abort_flag, P.wait_ns)) {
            fail(33);
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(KCH, nkb - st * KCH);
          const uint32_t a_addr = smem_u32(smem_a + stage * A_STAGE);
          const uint32_t b_addr = smem_u32(smem_b + stage * B_STAGE);
#pragma unroll
          for (int ch = 0; ch < KCH; ++ch) {
            if (ch < nk) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16_pair(d_tmem, sw128_kmajor_desc(a_addr + ch * A_BYTES + kk * 32),
                               sw128_kmajor_desc(b_addr + ch * B_BYTES + kk * 32), idesc,
                               (st | ch | kk) != 0 ? 1u : 0u);
            }
          }
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
      if (!mbar_wait_bounded(&c.mma_done, 0, &never, kTimeoutNs)) report_error(P.err, MOE_ERR_DEVICE_TIMEOUT, 38);
    }
  } else {
    // ------------------------------------------- epilogue (warps 0 .. 3) --
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t empty_leader = map_to_rank(smem_u32(&c.tmem_empty[0]), 0);
    const uint32_t tq_empty_leader = map_to_rank(smem_u32(&c.tq_empty[0]), 0);
    int q = 0;
    uint32_t qph = 0;
    for (;;) {
      const bool gotq = mbar_wait_bounded<true>(&c.tq_full[q], qph, abort_flag, P.wait_ns);
      if (!named_barrier_and(1, 128, gotq)) {
        if (lane == 0 && !gotq) fail(40);
        break;
      }
      const int t = c.tq[q];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tq_empty_leader + static_cast<uint32_t>(q * sizeof(uint64_t)));
      if (++q == QD) {
        q = 0;
        qph ^= 1u;
      }
      if (t < 0) break;
      const Tile ti = decode(P, c, t);
      const int p = ti.p;
      const int N = P.n_out[p];
      const bool got = mbar_wait_bounded(&c.tmem_full[acc], acc_phase, abort_flag, P.wait_ns);
      // all four warps leave together: the gate/up exchange below uses named barriers
      if (!named_barrier_and(1, 128, got)) {
        if (lane == 0 && !got) fail(34);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * 256);
      const int nch = ti.nmma / 32 + ((ti.nmma & 31) ? 1 : 0);
      __nv_bfloat16* out = P.out[p];
      // Per 32-token chunk: TMEM -> registers (lane = weight row, register =
      // token) -> bf16 into obuf[token][feature] -> 16-byte row stores.
      __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(c.obuf);
      if (KIND == Kind::GateUp) {
        const int f0 = ti.fidx * 128 + static_cast<int>(rank) * 64;  // first feature of the CTA
        const float L = P.limit;
        unsigned char* hb = reinterpret_cast<unsigned char*>(c.obuf);
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
            const int fl = (2 * warp + h) * 8 + (lane >> 2);  // feature within the CTA's 64
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int tok = 8 * q + 2 * (lane & 3) + e;
                const float gv = fminf(__uint_as_float(v[h][4 * q + e]), L);
                const float uv = fminf(fmaxf(__uint_as_float(v[h][4 * q + 2 + e]), -L), L);
                *reinterpret_cast<__nv_bfloat16*>(hb + tok * HPITCH + fl * 2) =
                    __float2bfloat16_rn(__fdividef(gv, 1.f + __expf(-gv)) * uv);
              }
          }
          named_barrier_sync(1, 128);  // staging complete
          // 32 rows x 128 B: 8 vectors per row, two per thread
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int idx = threadIdx.x + 128 * r;
            const int row = idx >> 3, c16 = idx & 7;
            const int col = ch * 32 + row;
            const int f = f0 + c16 * 8;
            if (col < ti.ntok && f < N)
              *reinterpret_cast<uint4*>(out + static_cast<size_t>(ti.row0 + col) * N + f) =
                  *reinterpret_cast<const uint4*>(hb + row * HPITCH + c16 * 16);
          }
        }
      } else {
        const int nl = warp * 32 + lane;                              // weight row within this CTA's 128
        const int n0 = ti.fidx * 256 + static_cast<int>(rank) * 128;  // first output column of the CTA
        const float* rs = P.row_scale[p];
#pragma unroll 1
        for (int ch = 0; ch < nch; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + ch * 32, v);
          tmem_ld_wait();
          const int mycol = ch * 32 + lane;
          const float my_sc = (rs != nullptr && mycol < ti.ntok) ? rs[ti.row0 + mycol] : 1.f;
          named_barrier_sync(1, 128);  // previous chunk's obuf reads done
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sc = __shfl_sync(0xffffffffu, my_sc, j);
            ob[j * 128 + nl] = __float2bfloat16_rn(__uint_as_float(v[j]) * sc);
          }
          named_barrier_sync(1, 128);  // obuf complete
          // 32 rows x 256 B: 16 vectors per row, four per thread
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int idx = threadIdx.x + 128 * r;
            const int row = idx >> 4, c16 = idx & 15;
            const int col = ch * 32 + row;
            const int n = n0 + c16 * 8;
            if (col < ti.ntok && n < N)
              *reinterpret_cast<uint4*>(out + static_cast<size_t>(ti.row0 + col) * N + n) = c.obuf[idx];
          }
        }
      }
      // accumulator read: release it to the MMA issuer of the pair
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

bool encode_w(CUtensorMap* m, const void* base, int slices, int N, int K, int box_rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(slices)};
  const uint64_t strides[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * N * 2};
  const uint32_t box[3] = {BK, static_cast<uint32_t>(box_rows), 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// gate/up weight [G][2][N][K] seen as {K, r = 8, u = 2, b = N/8, G}: a box of
// {64, 8, 2, 8, 1} lands as 128 rows ordered (b, u, r).
bool encode_w_gu(CUtensorMap* m, const void* base, int groups, int N, int K) {
  const uint64_t dims[5] = {static_cast<uint64_t>(K), 8, 2, static_cast<uint64_t>(N / 8),
                            static_cast<uint64_t>(groups)};
  const uint64_t row = static_cast<uint64_t>(K) * 2;
  const uint64_t strides[4] = {row, row * N, row * 8, row * N * 2};
  const uint32_t box[5] = {BK, 8, 2, 8, 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool encode_x(CUtensorMap (&m)[kTokBoxes], const void* base, int rows, int K) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
  for (int b = 0; b < kTokBoxes; ++b) {
    const uint32_t box[2] = {BK, static_cast<uint32_t>((TOK / 2) >> b)};
    if (!encode_tma(&m[b], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

// Hidden rows of the tokens, [tokens, K], read four rows per copy.
bool encode_x_rows(CUtensorMap* m, const void* base, int tokens, int K) {
  const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(tokens)};
  const uint64_t strides[1] = {static_cast<uint64_t>(K) * 2};
  const uint32_t box[2] = {BK, 1};
  return encode_tma(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// CTA pairs that can be resident at once on the current device (a pair must
// sit in one GPC, so this can be below half the SM count); 0 if unknown.
template <Kind KIND, bool GATHER>
int resident_pairs() {
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
    if (cudaOccupancyMaxActiveClusters(&n, ffn_pair_kernel<KIND, GATHER>, &lc) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cached[dev] = n;
    known[dev] = true;
  }
  return cached[dev];
}

template <Kind KIND, bool GATHER>
cudaError_t start_pair(const PairParams& P, int num_sms, cudaStream_t stream) {
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(ffn_pair_kernel<KIND, GATHER>),
                                   static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  int grid = std::max(2, num_sms / 2 * 2);
  const int pairs = resident_pairs<KIND, GATHER>();
  if (pairs > 0) grid = std::min(grid, 2 * pairs);
  return launch_kernel(ffn_pair_kernel<KIND, GATHER>, dim3(grid), dim3(THREADS), kSmem, stream, P);
}

template <Kind KIND>
cudaError_t launch_pair(const FfnProblem* routed, const FfnProblem* shared, float limit, int32_t* err,
                        int32_t* queue, int num_sms, cudaStream_t stream) {
  PairParams P;
  memset(&P, 0, sizeof(P));
  const FfnProblem* probs[2];
  int np = 0;
  if (shared != nullptr && shared->rows > 0) probs[np++] = shared;  // larger tiles first
  if (routed != nullptr && routed->rows > 0) probs[np++] = routed;
  if (np == 0) return cudaSuccess;
  if (np == 2 && probs[0]->offsets != nullptr && probs[1]->offsets != nullptr)
    return cudaErrorInvalidValue;  // one grouped problem per launch (one offsets table in shared memory)
  for (int i = 0; i < np; ++i) {
    const FfnProblem& f = *probs[i];
    if (f.gather_src != nullptr) {
      if (KIND != Kind::GateUp || f.offsets == nullptr || f.gather_k < 1 || f.a_rows < 1) return cudaErrorInvalidValue;
      if (!encode_x_rows(&P.tma_x[i][0], f.a, f.a_rows, f.K)) return cudaErrorInvalidValue;
      P.gsrc[i] = f.gather_src;
      P.gk[i] = f.gather_k;
    } else if (!encode_x(P.tma_x[i], f.a, f.rows, f.K)) {
      return cudaErrorInvalidValue;
    }
    const bool okw = KIND == Kind::GateUp ? encode_w_gu(&P.tma_w[i], f.w, f.groups, f.N, f.K)
                                          : encode_w(&P.tma_w[i], f.w, f.groups, f.N, f.K, 128);
    if (!okw) return cudaErrorInvalidValue;
    P.offsets[i] = f.offsets;
    P.out[i] = static_cast<__nv_bfloat16*>(f.out);
    P.row_scale[i] = f.row_scale;
    P.groups[i] = f.groups;
    P.rows[i] = f.rows;
    P.n_out[i] = f.N;
    P.k_blocks[i] = (f.K + BK - 1) / BK;
    P.f_tiles[i] = KIND == Kind::GateUp ? (f.N + 127) / 128 : (f.N + 255) / 256;
  }
  if (queue == nullptr) return cudaErrorInvalidValue;
  P.nprob = np;
  P.limit = limit;
  P.err = err;
  P.queue = queue;
  P.wait_ns = kTimeoutNs;
  const bool gather = P.gsrc[0] != nullptr || P.gsrc[1] != nullptr;
  // (only gate/up problems gather; the down projection reads h in row order)
  return gather ? start_pair<KIND, KIND == Kind::GateUp>(P, num_sms, stream)
                : start_pair<KIND, false>(P, num_sms, stream);
}

}  // namespace

// Test hook: one tiny gate/up problem (16 tokens, 64 features, K = 64; zero
// operands in `scratch`) on one CTA pair whose first (only) accumulator is
// never signalled to the epilogue, with every wait on another role limited to
// 20 ms.  Both CTAs' epilogue waits run out and record
// MOE_ERR_DEVICE_TIMEOUT (detail 34); the producer, the MMA issuer and the
// pair's final cluster barrier finish on their normal paths (the copies and
// MMAs drained, the tile queue reset by the retiring pair, TMEM freed).
cudaError_t launch_pair_timeout_selftest(void* scratch, int32_t* err, int32_t* queue, cudaStream_t stream) {
  unsigned char* base = static_cast<unsigned char*>(scratch);
  void* x = base + 1024;   // bf16 [16, 64]
  void* w = base + 4096;   // bf16 [1, 2 x 64, 64]: gate rows, then up rows
  void* h = base + 20480;  // bf16 [16, 64]
  PairParams P;
  memset(&P, 0, sizeof(P));
  if (!encode_x(P.tma_x[0], x, 16, 64) || !encode_w_gu(&P.tma_w[0], w, 1, 64, 64)) return cudaErrorInvalidValue;
  P.offsets[0] = nullptr;
  P.out[0] = static_cast<__nv_bfloat16*>(h);
  P.groups[0] = 1;
  P.rows[0] = 16;
  P.n_out[0] = 64;
  P.k_blocks[0] = 1;
  P.f_tiles[0] = 1;
  P.nprob = 1;
  P.limit = 7.f;
  P.err = err;
  P.queue = queue;
  P.wait_ns = 20000000ull;
  P.test_withhold = 1;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(ffn_pair_kernel<Kind::GateUp, false>),
                                   static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  ffn_pair_kernel<Kind::GateUp, false><<<2, THREADS, kSmem, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_gemm_gateup(const FfnProblem* routed, const FfnProblem* shared, float limit, int32_t* err,
                               int32_t* queue, int num_sms, cudaStream_t stream) {
  return launch_pair<Kind::GateUp>(routed, shared, limit, err, queue, num_sms, stream);
}

cudaError_t launch_gemm_down(const FfnProblem* routed, const FfnProblem* shared, int32_t* err, int32_t* queue,
                             int num_sms, cudaStream_t stream) {
  return launch_pair<Kind::Down>(routed, shared, 0.f, err, queue, num_sms, stream);
}

}  // namespace moe
