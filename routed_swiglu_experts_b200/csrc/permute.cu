// Token sort / permute by expert ("Module glm5next_mlp", MOE_MODULE: the
// token sort / permute / unpermute kernels) as a deterministic stable
// counting sort of the slots i = t*k + j, in two launches:
//   1. per 2048-slot chunk: per-expert counts, and each slot's rank among the
//      earlier slots of its chunk with the same expert (warp match + popc);
//      the last chunk block to finish (a ticket counter it resets to zero)
//      turns the counts into per-(chunk, expert) bases = expert offset +
//      earlier chunks, and writes the expert offsets;
//   2. scatter: row = base + rank; row_of / src / w_perm, and the 16-byte
//      vector gather of the token's hidden row into x_perm -- or the maps
//      alone, when the grouped FFN gathers the rows in its own loads.
// No atomic decides an order (the ticket only picks which block scans), so
// the result is identical run to run.
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kPermWarps = 8;
constexpr int kPermIters = kPermChunk / (kPermWarps * 32);  // 8 slots per lane
static_assert(kPermIters * kPermWarps * 32 == kPermChunk, "chunk split");

// Count tables of at most this many (chunk, expert) entries are scanned in
// shared memory by the last block; larger ones column by column in global.
constexpr int kScanSmemEntries = 16384;

// Exclusive prefix over the chunks of every expert column of cnt[nb][E]
// (chunk-major), in place; tot[e] = the column total.  Run by one block.
__device__ void scan_columns_global(int32_t* __restrict__ cnt, int nb, int E, int32_t* tot) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int b0 = 0; b0 < nb; b0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = b0 + j < nb ? __ldcg(cnt + static_cast<size_t>(b0 + j) * E + e) : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (b0 + j < nb) {
          cnt[static_cast<size_t>(b0 + j) * E + e] = run;
          run += v[j];
        }
    }
    tot[e] = run;
  }
}

// dynamic smem: max(cnt[kPermWarps][E], table[nb][E] when nb * E <= kScanSmemEntries)
__global__ void __launch_bounds__(kPermWarps * 32)
    perm_count_rank_kernel(const int32_t* __restrict__ ids, int R, int E, int32_t* __restrict__ block_base,
                           int32_t* __restrict__ local_rank, int32_t* __restrict__ offsets,
                           int32_t* __restrict__ done) {
  extern __shared__ int32_t cnt[];
  __shared__ int32_t tot[MOE_MAX_EXPERTS];
  __shared__ int32_t wsum[kPermWarps];
  __shared__ int s_last;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int j = threadIdx.x; j < kPermWarps * E; j += blockDim.x) cnt[j] = 0;
  __syncthreads();

  const int base = blockIdx.x * kPermChunk + warp * (kPermIters * 32);
  int32_t* wcnt = cnt + warp * E;
  int rank[kPermIters];
  int idv[kPermIters];
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int it = 0; it < kPermIters; ++it) {
    const int i = base + it * 32 + lane;
    const int id = i < R ? ids[i] : -1;
    idv[it] = id;
    const uint32_t m = __match_any_sync(0xffffffffu, id);
    const int before = __popc(m & lt_mask);
    rank[it] = (id >= 0 ? wcnt[id] : 0) + before;
    __syncwarp();
    if (id >= 0 && before == 0) wcnt[id] += __popc(m);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over the warps of this chunk; chunk totals to global
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
    block_base[static_cast<size_t>(blockIdx.x) * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < kPermIters; ++it) {
    const int i = base + it * 32 + lane;
    if (i < R) local_rank[i] = wcnt[idv[it]] + rank[it];
  }

  // the last block to get here turns every chunk's counts into bases
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(done, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int nb = gridDim.x;
  const int n = nb * E;
  if (n <= kScanSmemEntries) {
    int32_t* tab = cnt;  // the chunk's counts are no longer needed
    for (int i = threadIdx.x; i < n; i += blockDim.x) tab[i] = __ldcg(block_base + i);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int run = 0;
      for (int b = 0; b < nb; ++b) {
        const int c = tab[b * E + e];
        tab[b * E + e] = run;
        run += c;
      }
      tot[e] = run;
    }
  } else {
    scan_columns_global(block_base, nb, E, tot);
  }
  __syncthreads();
  // exclusive scan of the expert totals (E <= 1024: 4 consecutive per thread)
  constexpr int kPer = MOE_MAX_EXPERTS / (kPermWarps * 32);
  int v[kPer];
  int local = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = threadIdx.x * kPer + j;
    v[j] = e < E ? tot[e] : 0;
    local += v[j];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = incl - local;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  __syncthreads();  // every thread has read tot[] for its own entries
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = threadIdx.x * kPer + j;
    if (e < E) {
      offsets[e] = before;
      tot[e] = before;
    }
    before += v[j];
  }
  if (threadIdx.x == kPermWarps * 32 - 1) offsets[E] = before;  // = R
  __syncthreads();
  if (n <= kScanSmemEntries) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) block_base[i] = cnt[i] + tot[i % E];
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) block_base[i] += tot[i % E];
  }
  if (threadIdx.x == 0) *done = 0;  // ready for the next launch
}

// One warp per slot: routed row, inverse maps, weight, and the hidden row
// (copied only for experts in [e0, e1): the experts this call computes).
__global__ void __launch_bounds__(256)
    perm_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w,
                        const __nv_bfloat16* __restrict__ x, int R, int k, int E, int H,
                        const int32_t* __restrict__ block_base, const int32_t* __restrict__ local_rank,
                        int32_t* __restrict__ row_of, int32_t* __restrict__ src, float* __restrict__ w_perm,
                        __nv_bfloat16* __restrict__ x_perm, int e0, int e1) {
  const int i = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (i >= R) return;
  const int id = ids[i];
  const int row = block_base[static_cast<size_t>(i / kPermChunk) * E + id] + local_rank[i];
  if (lane == 0) {
    row_of[i] = row;
    src[row] = i;
    w_perm[row] = topk_w[i];
  }
  if (id < e0 || id >= e1) return;
  const uint4* s = reinterpret_cast<const uint4*>(x + static_cast<size_t>(i / k) * H);
  uint4* d = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(row) * H);
  const int n16 = H / 8;
  int c = lane;
  for (; c + 96 < n16; c += 128) {
    const uint4 a0 = __ldg(s + c), a1 = __ldg(s + c + 32), a2 = __ldg(s + c + 64), a3 = __ldg(s + c + 96);
    d[c] = a0;
    d[c + 32] = a1;
    d[c + 64] = a2;
    d[c + 96] = a3;
  }
  for (; c < n16; c += 32) d[c] = __ldg(s + c);
}

// Maps only (the grouped FFN gathers the hidden rows itself): one thread per
// slot writes its routed row, the inverse map and the weight.
__global__ void __launch_bounds__(256)
    perm_maps_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int R, int E,
                     const int32_t* __restrict__ block_base, const int32_t* __restrict__ local_rank,
                     int32_t* __restrict__ row_of, int32_t* __restrict__ src, float* __restrict__ w_perm) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R) return;
  const int row = block_base[static_cast<size_t>(i / kPermChunk) * E + ids[i]] + local_rank[i];
  row_of[i] = row;
  src[row] = i;
  w_perm[row] = topk_w[i];
}

}  // namespace

cudaError_t launch_permute(const moe_config& cfg, const int32_t* ids, const float* topk_w, const void* x, int T,
                           int32_t* offsets, int32_t* row_of, int32_t* src, float* w_perm, void* x_perm,
                           int32_t* block_base, int32_t* local_rank, int32_t* done, cudaStream_t stream, int e0,
                           int e1) {
  const int E = cfg.num_experts, k = cfg.top_k, H = cfg.hidden;
  const int R = T * k;
  const int nb = perm_blocks(R);
  const size_t n = static_cast<size_t>(nb) * E;
  const size_t smem = std::max(static_cast<size_t>(kPermWarps) * E, n <= kScanSmemEntries ? n : 0) * sizeof(int32_t);
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(perm_count_rank_kernel),
                                   static_cast<int>(std::max(kPermWarps * MOE_MAX_EXPERTS, kScanSmemEntries) *
                                                    sizeof(int32_t)));
  if (e != cudaSuccess) return e;
  e = launch_kernel(perm_count_rank_kernel, dim3(nb), dim3(kPermWarps * 32), smem, stream, ids, R, E,
                            block_base, local_rank, offsets, done);
  if (e != cudaSuccess) return e;
  if (x_perm == nullptr)
    return launch_kernel(perm_maps_kernel, dim3((R + 255) / 256), dim3(256), 0, stream, ids, topk_w, R, E,
                                 static_cast<const int32_t*>(block_base), static_cast<const int32_t*>(local_rank),
                                 row_of, src, w_perm);
  return launch_kernel(perm_scatter_kernel, dim3((R + 7) / 8), dim3(256), 0, stream, ids, topk_w,
                               static_cast<const __nv_bfloat16*>(x), R, k, E, H,
                               static_cast<const int32_t*>(block_base), static_cast<const int32_t*>(local_rank),
                               row_of, src, w_perm, static_cast<__nv_bfloat16*>(x_perm), e0, e1 < 0 ? E : e1);
}

}  // namespace moe
