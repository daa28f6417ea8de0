// Token sort / permute by expert ("Module glm5next_mlp", MOE_MODULE: the
// token sort / permute / unpermute kernels) as a deterministic stable
// counting sort of the slots i = t*k + j:
//   1. per 2048-slot chunk: per-expert counts, and each slot's rank among the
//      earlier slots of its chunk with the same expert (warp match + popc);
//   2. one block: per-(chunk, expert) bases = expert offset + earlier chunks;
//   3. scatter: row = base + rank; row_of / src / w_perm, and the 16-byte
//      vector gather of the token's hidden row into x_perm.
// No atomics decide an order, so the result is identical run to run.
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kPermWarps = 8;
constexpr int kPermIters = kPermChunk / (kPermWarps * 32);  // 8 slots per lane
static_assert(kPermIters * kPermWarps * 32 == kPermChunk, "chunk split");

// dynamic smem: cnt[kPermWarps][E]
__global__ void __launch_bounds__(kPermWarps * 32)
    perm_count_rank_kernel(const int32_t* __restrict__ ids, int R, int E, int32_t* __restrict__ block_base,
                           int32_t* __restrict__ local_rank) {
  extern __shared__ int32_t cnt[];
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
}

// One block of 1024 threads.  block_base[b][e] (chunk counts) becomes the
// first routed row of chunk b's slots of expert e; offsets[0..E] written.
__global__ void __launch_bounds__(1024)
    perm_scan_kernel(int32_t* __restrict__ block_base, int nblocks, int E, int32_t* __restrict__ offsets) {
  __shared__ int32_t tot[MOE_MAX_EXPERTS];
  __shared__ int32_t wsum[32];
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblocks; ++b) {
      const int c = block_base[static_cast<size_t>(b) * E + e];
      block_base[static_cast<size_t>(b) * E + e] = run;
      run += c;
    }
    tot[e] = run;
  }
  __syncthreads();
  // exclusive scan of tot[0..E) (E <= 1024: one element per thread)
  const int v = tid < E ? tot[tid] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = wsum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += o;
    }
    wsum[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - v + (warp > 0 ? wsum[warp - 1] : 0);
  if (tid < E) {
    offsets[tid] = excl;
    tot[tid] = excl;
  }
  if (tid == E - 1) offsets[E] = excl + v;
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int o = tot[e];
    for (int b = 0; b < nblocks; ++b) block_base[static_cast<size_t>(b) * E + e] += o;
  }
}

// One warp per slot: routed row, inverse maps, weight, and the hidden row.
__global__ void __launch_bounds__(256)
    perm_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ topk_w,
                        const __nv_bfloat16* __restrict__ x, int R, int k, int E, int H,
                        const int32_t* __restrict__ block_base, const int32_t* __restrict__ local_rank,
                        int32_t* __restrict__ row_of, int32_t* __restrict__ src, float* __restrict__ w_perm,
                        __nv_bfloat16* __restrict__ x_perm) {
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

}  // namespace

cudaError_t launch_permute(const moe_config& cfg, const int32_t* ids, const float* topk_w, const void* x, int T,
                           int32_t* offsets, int32_t* row_of, int32_t* src, float* w_perm, void* x_perm,
                           int32_t* block_base, int32_t* local_rank, cudaStream_t stream) {
  const int E = cfg.num_experts, k = cfg.top_k, H = cfg.hidden;
  const int R = T * k;
  const int nb = perm_blocks(R);
  const size_t smem = static_cast<size_t>(kPermWarps) * E * sizeof(int32_t);
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(perm_count_rank_kernel),
                                   kPermWarps * MOE_MAX_EXPERTS * static_cast<int>(sizeof(int32_t)));
  if (e != cudaSuccess) return e;
  perm_count_rank_kernel<<<nb, kPermWarps * 32, smem, stream>>>(ids, R, E, block_base, local_rank);
  perm_scan_kernel<<<1, 1024, 0, stream>>>(block_base, nb, E, offsets);
  perm_scatter_kernel<<<(R + 7) / 8, 256, 0, stream>>>(ids, topk_w, static_cast<const __nv_bfloat16*>(x), R, k, E,
                                                       H, block_base, local_rank, row_of, src, w_perm,
                                                       static_cast<__nv_bfloat16*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
