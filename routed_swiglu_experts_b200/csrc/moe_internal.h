// Internal declarations shared by the library's translation units.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "moe_common.cuh"

namespace moe {

// Opt a kernel into `bytes` of dynamic shared memory on the current device
// (cached per device and kernel).
cudaError_t ensure_smem_attr(const void* func, int bytes);

// Launch `kernel` on `stream` (an ordinary, fully ordered launch) and
// return the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          Args&&... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = stream;
  return cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}

// Encode a tiled TMA descriptor (strides in bytes for dims 1..rank-1).
bool encode_tma(CUtensorMap* m, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle);

// Router: rows of fp32 partial logits (k-splits x tokens) the logits GEMM
// may write, per expert.
constexpr int kRouterPartialRows = 32768;
// Near-tie width on the fp32 biased score (2^-13) below which adjacent
// experts are re-ordered from fp64 logits.  It is far above the error of the
// tensor-core fp32 logits (exact bf16 x bf16 products, fp32 sums over K).
constexpr float kRouterTieTau = 1.220703125e-04f;

// MMA N of the router GEMM: E rounded up to 16, at most 256.
inline int router_mma_n(int E) { return std::min(256, (E + 15) / 16 * 16); }

struct RouterPlan {
  int ks;  // k-splits of the logits GEMM (partials summed by the top-k kernel)
};
RouterPlan router_plan(int T, int E, int H, int num_sms);
size_t router_partial_floats(int Tmax, int E);
size_t router_topk_smem(int E);
// Split-K tensor-core GEMM with fp32 partials part[s][rows][N] over `parts`
// passes of K (B slice p per pass); n_mma: MMA N, a multiple of 16 <= 256.
cudaError_t launch_splitk_gemm(const void* a, int rows, int K, const void* b, int parts, int N, int n_mma,
                               int k_splits, float* part, int32_t* err, int num_sms, cudaStream_t stream);
// K steps of one tile's full reduction (all B slices of a step share a stage
// when n_mma is small) and the split count a request of k_splits becomes.
int splitk_steps(int K, int parts, int n_mma, int rows);
int splitk_actual_splits(int K, int parts, int n_mma, int rows, int k_splits);
cudaError_t launch_splitk_timeout_selftest(void* scratch, int32_t* err, cudaStream_t stream);
// Test hooks of the CTA-pair kernels' timeout paths (see moe_selftest_pair_timeout).
cudaError_t launch_pair_timeout_selftest(void* scratch, int32_t* err, int32_t* queue, cudaStream_t stream);
cudaError_t launch_int4_pair_timeout_selftest(void* scratch, int32_t* err, int32_t* queue, cudaStream_t stream);
int router_actual_splits(int T, int E, int H, int k_splits);
cudaError_t launch_router_gemm(const void* x, int T, int H, const void* w_split, int E, int k_splits, float* part,
                               int32_t* err, int num_sms, cudaStream_t stream);
cudaError_t launch_router(const moe_config& cfg, const moe_weights& w, const void* x, int T, int32_t* ids,
                          float* wts, float* part, void* w_split, int32_t* err, int num_sms, cudaStream_t stream);

// Permute: slots per counting block.
constexpr int kPermChunk = 2048;
inline int perm_blocks(int R) { return std::max(1, (R + kPermChunk - 1) / kPermChunk); }
// block_base: [perm_blocks(T*k) * E] scratch; local_rank: [T*k] scratch;
// done: a ticket counter that is zero before the launch and left at zero.
// Hidden rows are copied into x_perm only for experts in [e0, e1) (e1 < 0:
// every expert); the maps and weights cover every slot.  x_perm == nullptr:
// maps and weights only (x unused).
cudaError_t launch_permute(const moe_config& cfg, const int32_t* ids, const float* topk_w, const void* x, int T,
                           int32_t* offsets, int32_t* row_of, int32_t* src, float* w_perm, void* x_perm,
                           int32_t* block_base, int32_t* local_rank, int32_t* done, cudaStream_t stream, int e0 = 0,
                           int e1 = -1);

// range: NULL, or device pointer to expert offsets: only routed rows in
// [range[0], range[range_len]) are added (expert parallelism's partial combine).
cudaError_t launch_combine(const moe_config& cfg, const void* y_perm, const int32_t* row_of, const float* topk_w,
                           const void* shared_out, int T, void* out, const int32_t* range, int range_len,
                           cudaStream_t stream);

// Grouped GEMMs (tcgen05).  One "problem" is a set of row groups that share
// an A operand tensor and a weight tensor; the routed experts are one problem
// (groups = experts, rows given by expert offsets), the shared expert another
// (one group covering all tokens).
struct FfnProblem {
  const void* a;                 // bf16 [rows, K]
  int rows;                      // total rows of a
  const int32_t* offsets;        // [groups+1] device, or nullptr: one group of `rows`
  int groups;
  const void* w;                 // bf16 weights: gate/up [groups, 2N, K]; down [groups, N, K]
  int N, K;                      // output columns, reduction length
  void* out;                     // bf16 [rows, N]
  const float* row_scale;        // per-row scale (down only) or nullptr
  // gate/up of a grouped problem may read its rows straight from the tokens:
  // row r of the problem is row gather_src[r] / gather_k of `a` ([a_rows, K])
  const int32_t* gather_src = nullptr;
  int gather_k = 0;
  int a_rows = 0;
};
// queue: the launch's two tile-queue words in the workspace header (zero).
cudaError_t launch_gemm_gateup(const FfnProblem* routed, const FfnProblem* shared, float limit, int32_t* err,
                               int32_t* queue, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_down(const FfnProblem* routed, const FfnProblem* shared, int32_t* err, int32_t* queue,
                             int num_sms, cudaStream_t stream);

// 4-bit routed expert GEMVs (dequantise in registers): W4A16 int4 or NVFP4
// weights, by cfg.expert_format.
// act16: scratch for the activations in MMA slot order (fp16, [rows, K]).
// With x_shared != NULL (T <= kW4a16SharedMaxTokens tokens) the shared
// expert's bf16 projections run in the same two launches: gate/up into
// gu_shared (fp32 [T, 2 I_s]), its SwiGLU into h_shared (bf16 [T, I_s]) with
// the down projection's activation prep, and down into shared_out.
constexpr int kW4a16SharedMaxTokens = 32;
bool w4a16_shared_fusable(int T, int Is);
// x_rows: the permuted rows [rows, H] (gather_src == NULL), or the tokens
// [T, H] with row r of the routed problem = token gather_src[r] / top_k.
cudaError_t launch_w4a16_gateup(const moe_config& cfg, const moe_weights& w, const void* x_rows,
                                const int32_t* gather_src, const int32_t* offsets, int rows, void* act16, float* gu,
                                const void* x_shared, int T, float* gu_shared, cudaStream_t stream);
cudaError_t launch_w4a16_down(const moe_config& cfg, const moe_weights& w, const float* gu, const int32_t* offsets,
                              int rows, void* act16, const float* w_perm, void* y_perm, const float* gu_shared,
                              int T, void* h_shared, void* shared_out, cudaStream_t stream);

// 4-bit grouped GEMMs for many tokens per expert (at least
// kInt4PrefillRowsPerExpert routed rows per expert on average): int4 (W4A16)
// or NVFP4 codes dequantised to fp16 in shared memory and fed to the CTA-pair
// tensor-core pipeline; cfg.expert_format picks the decoder.
// tokens16: scratch [rows, H] fp16; h16: scratch [rows, I] fp16; queues:
// four tile-queue words in the workspace header (gate/up, then down).
constexpr int kInt4PrefillRowsPerExpert = 32;
bool int4_prefill_preferred(int rows, int E);
// x_rows / gather_src as for launch_w4a16_gateup.
cudaError_t launch_int4_ffn_prefill(const moe_config& cfg, const moe_weights& w, const void* x_rows,
                                    const int32_t* gather_src, const int32_t* offsets, int rows, void* tokens16,
                                    void* h16, const float* w_perm, void* y_perm, int32_t* err, int32_t* queues,
                                    int num_sms, cudaStream_t stream);

// Shared expert for T <= 32 tokens: split-K tensor-core GEMMs streaming the
// weights across all SMs, then an ordered sum of the K slices.
constexpr int kDenseSmallMaxTokens = 32;
constexpr int kDenseSmallMaxSplits = 16;
bool dense_small_ok(int T, int H, int Is);
size_t dense_small_part_floats(int H, int Is);
cudaError_t launch_dense_small_ffn(const void* x, int T, int H, int Is, const void* w_gu, const void* w_d, float L,
                                   float* part, void* h_s, void* out, int32_t* err, int num_sms, cudaStream_t stream);

// Workspace layout (byte offsets from the workspace base; 256-aligned).
struct WsLayout {
  size_t header, logits, w_split, ids, wts, offsets, row_of, src, w_perm, block_base, local_rank;
  size_t x_perm, h, h_shared, y_perm, shared_out, act16, small_part, total;
};
WsLayout ws_layout(const moe_config& cfg, int Tmax);

}  // namespace moe
