// The C ABI (include/moe.h): argument validation, workspace layout, and the
// launch sequence of the layer forward.  No allocation, no host sync (except
// moe_read_device_error), no exceptions across the boundary.
#include <cmath>
#include <cstring>
#include <mutex>

#include "moe_internal.h"

namespace moe {

namespace {

inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

constexpr int64_t kMaxTokens = int64_t(1) << 21;  // grid-dimension bound of the router

int num_sms_current_device() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

moe_status check_tokens(const moe_config& cfg, int32_t T) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) > kMaxTokens) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ws(const moe_config& cfg, int32_t T, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(cfg, T).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

int32_t* err_word(void* ws) { return reinterpret_cast<int32_t*>(ws); }
int32_t* tile_queue(void* ws, TileQueueSlot slot) { return reinterpret_cast<WsHeader*>(ws)->tile_queue + slot; }
int32_t* perm_ticket(void* ws) { return &reinterpret_cast<WsHeader*>(ws)->perm_done; }

bool is_int4(const moe_config& cfg) { return cfg.expert_format == MOE_W_INT4_G128; }
bool is_nvfp4(const moe_config& cfg) { return cfg.expert_format == MOE_W_NVFP4; }
// both 4-bit formats: fp16 activations, the 4-bit kernels gather the routed rows
bool is_4bit(const moe_config& cfg) { return is_int4(cfg) || is_nvfp4(cfg); }

moe_status check_expert_weights(const moe_config& cfg, const moe_weights* w) {
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (w->w_gate_up == nullptr || w->w_down == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w_gate_up) || !aligned16(w->w_down)) return MOE_ERR_INVALID_ARG;
  if (is_4bit(cfg)) {
    if (w->s_gate_up == nullptr || w->s_down == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->s_gate_up) || !aligned16(w->s_down)) return MOE_ERR_INVALID_ARG;
  }
  if (is_nvfp4(cfg)) {
    if (w->g_gate_up == nullptr || w->g_down == nullptr) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(w->g_gate_up) & 3u) != 0 || (reinterpret_cast<uintptr_t>(w->g_down) & 3u) != 0)
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status check_shared_weights(const moe_config& cfg, const moe_weights* w) {
  if (cfg.shared_inter == 0) return MOE_OK;
  if (w == nullptr || w->shared_w_gate_up == nullptr || w->shared_w_down == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->shared_w_gate_up) || !aligned16(w->shared_w_down)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status check_router_weights(const moe_weights* w) {
  if (w == nullptr || w->router_w == nullptr || !aligned16(w->router_w)) return MOE_ERR_INVALID_ARG;
  if (w->correction_bias != nullptr && (reinterpret_cast<uintptr_t>(w->correction_bias) & 3u) != 0)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

#define MOE_TRY(expr)                       \
  do {                                      \
    const moe_status _s = (expr);           \
    if (_s != MOE_OK) return _s;            \
  } while (0)

#define MOE_CUDA_TRY(expr)                              \
  do {                                                  \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA;     \
  } while (0)

// The grouped FFN on the permuted rows (routed) plus, optionally, the
// shared expert on the raw tokens.  The routed rows are x_rows itself
// (gather_src == NULL: x_perm) or gathered from the tokens x_rows [T, H] by
// the permutation's slot map (row r = token gather_src[r] / top_k) inside the
// kernels' own loads.  cfg.num_experts is the number of experts this call
// computes (0 allowed: shared expert only), `offsets` their [E + 1] row
// offsets (absolute permuted rows), and w's routed weights hold exactly those
// experts; e_total is the router's expert count (the 4-bit paths pick their
// kernel by the average routed rows per expert, R / e_total).
moe_status run_ffn(const moe_config& cfg, const moe_weights& w, const void* x_rows, const int32_t* gather_src,
                   const int32_t* offsets, const float* w_perm, int32_t T, void* y_perm, const void* x_shared,
                   void* shared_out, void* ws, const WsLayout& L, cudaStream_t stream, int e_total) {
  const int H = cfg.hidden, I = cfg.expert_inter, Is = cfg.shared_inter, E = cfg.num_experts;
  const int R = T * cfg.top_k;
  const bool routed = E > 0;
  int32_t* err = err_word(ws);
  int32_t* qgu = tile_queue(ws, kQueueGateUp);
  int32_t* qd = tile_queue(ws, kQueueDown);
  void* h = at<void>(ws, L.h);
  void* hs = at<void>(ws, L.h_shared);
  const int sms = num_sms_current_device();
  const bool with_shared = x_shared != nullptr && Is > 0 && T > 0;

  // few tokens: the shared expert streams its weights with the split-K
  // kernels -- or, beside the int4 GEMVs, inside their launches; otherwise it
  // is one more problem of the tcgen05 launches
  const bool prefill_path = is_4bit(cfg) && int4_prefill_preferred(R, e_total);
  const bool gemv_path = is_4bit(cfg) && !prefill_path;
  const bool shared_in_gemv = with_shared && gemv_path && w4a16_shared_fusable(T, Is);
  const bool shared_small = with_shared && !shared_in_gemv && dense_small_ok(T, H, Is);
  const bool shared_tc = with_shared && !shared_in_gemv && !shared_small;
  FfnProblem s_gu{}, s_d{};
  if (shared_tc) {
    s_gu = FfnProblem{x_shared, T, nullptr, 1, w.shared_w_gate_up, Is, H, hs, nullptr};
    s_d = FfnProblem{hs, T, nullptr, 1, w.shared_w_down, H, Is, shared_out, nullptr};
  }
  if (shared_small)
    MOE_CUDA_TRY(launch_dense_small_ffn(x_shared, T, H, Is, w.shared_w_gate_up, w.shared_w_down, cfg.swiglu_limit,
                                        at<float>(ws, L.small_part), hs, shared_out, err, sms, stream));
  if (!is_4bit(cfg)) {
    FfnProblem r_gu{x_rows, R, offsets, E, w.w_gate_up, I, H, h, nullptr, gather_src, cfg.top_k, T};
    FfnProblem r_d{h, R, offsets, E, w.w_down, H, I, y_perm, w_perm};
    MOE_CUDA_TRY(launch_gemm_gateup(routed ? &r_gu : nullptr, shared_tc ? &s_gu : nullptr, cfg.swiglu_limit, err, qgu,
                                    sms, stream));
    MOE_CUDA_TRY(launch_gemm_down(routed ? &r_d : nullptr, shared_tc ? &s_d : nullptr, err, qd, sms, stream));
  } else {
    void* act16 = at<void>(ws, L.act16);
    if (prefill_path) {
      // many tokens per expert: dequantise in shared memory, tensor cores
      if (routed)
        MOE_CUDA_TRY(launch_int4_ffn_prefill(cfg, w, x_rows, gather_src, offsets, R, act16, at<void>(ws, L.h), w_perm,
                                             y_perm, err, tile_queue(ws, kQueueInt4GateUp), sms, stream));
      if (shared_tc) MOE_CUDA_TRY(launch_gemm_gateup(nullptr, &s_gu, cfg.swiglu_limit, err, qgu, sms, stream));
    } else {
      // gate/up in fp32 into the h region; the SwiGLU is applied while the
      // down projection's activations are prepared
      float* gu = at<float>(ws, L.h);
      float* gu_s = shared_in_gemv ? at<float>(ws, L.small_part) : nullptr;
      MOE_CUDA_TRY(launch_w4a16_gateup(cfg, w, x_rows, gather_src, offsets, R, act16, gu,
                                       shared_in_gemv ? x_shared : nullptr, T, gu_s, stream));
      if (shared_tc) MOE_CUDA_TRY(launch_gemm_gateup(nullptr, &s_gu, cfg.swiglu_limit, err, qgu, sms, stream));
      MOE_CUDA_TRY(launch_w4a16_down(cfg, w, gu, offsets, R, act16, w_perm, y_perm, gu_s, T, hs, shared_out, stream));
    }
    if (shared_tc) MOE_CUDA_TRY(launch_gemm_down(nullptr, &s_d, err, qd, sms, stream));
  }
  return MOE_OK;
}

// Where the forward's FFN reads the routed rows.  bf16 experts: the permute
// copies them into the workspace's x_perm and the tensor-core kernel loads
// contiguous token boxes (its per-row gather4 form, moe_grouped_swiglu_ffn_gather,
// takes about twice as long: one TMA copy per four 128-byte rows is
// latency-bound).  int4 and NVFP4 experts: the permute writes the maps only
// and the activation conversion that every 4-bit kernel runs first gathers
// the rows.
struct Rows {
  void* x_perm;                 // permute output, or nullptr (maps only)
  const void* x_rows;           // what run_ffn reads
  const int32_t* gather_src;    // nullptr, or the slot map of a gathered read
};
Rows routed_rows(const moe_config& cfg, void* ws, const WsLayout& L, const void* x, const int32_t* src) {
  if (is_4bit(cfg)) return Rows{nullptr, x, src};
  void* xp = at<void>(ws, L.x_perm);
  return Rows{xp, xp, nullptr};
}

}  // namespace

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  static std::mutex mu;
  struct Entry { int dev; const void* func; int bytes; };
  static Entry done[256];
  static int ndone = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < ndone; ++i)
    if (done[i].dev == dev && done[i].func == func && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (ndone < 256) done[ndone++] = Entry{dev, func, bytes};
  return cudaSuccess;
}

WsLayout ws_layout(const moe_config& cfg, int Tmax) {
  WsLayout L{};
  const size_t T = static_cast<size_t>(std::max(Tmax, 0));
  const size_t E = cfg.num_experts, k = cfg.top_k, H = cfg.hidden, I = cfg.expert_inter, Is = cfg.shared_inter;
  const size_t R = T * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.header = take(sizeof(WsHeader));
  L.logits = take(router_partial_floats(static_cast<int>(T), static_cast<int>(E)) * sizeof(float));
  L.w_split = take(3 * E * H * 2);
  L.ids = take(R * sizeof(int32_t));
  L.wts = take(R * sizeof(float));
  L.offsets = take((E + 1) * sizeof(int32_t));
  L.row_of = take(R * sizeof(int32_t));
  L.src = take(R * sizeof(int32_t));
  L.w_perm = take(R * sizeof(float));
  L.block_base = take(static_cast<size_t>(perm_blocks(static_cast<int>(R))) * E * sizeof(int32_t));
  L.local_rank = take(R * sizeof(int32_t));
  const bool four = cfg.expert_format == MOE_W_INT4_G128 || cfg.expert_format == MOE_W_NVFP4;
  // bf16 experts: the forward gathers the routed rows into x_perm (tiled TMA
  // copies then feed the tensor cores); 4-bit experts gather while converting
  L.x_perm = take(four ? 0 : R * H * 2);
  // bf16 h, the 4-bit grouped GEMMs' fp16 h [R, I], or the 4-bit GEMVs' fp32
  // gate/up [R, 2I] (taken only below kInt4PrefillRowsPerExpert rows per expert)
  const size_t r_gemv = std::min(R, static_cast<size_t>(kInt4PrefillRowsPerExpert) * E);
  L.h = take(four ? std::max(R * I * 2, r_gemv * 2 * I * 4) : R * I * 2);
  L.h_shared = take(T * Is * 2);
  L.y_perm = take(R * H * 2);
  L.shared_out = take(T * H * 2);
  const size_t kmax = std::max(H, I);
  L.act16 = take(four ? R * kmax * 2 : 0);
  L.small_part = take(Is > 0 ? dense_small_part_floats(static_cast<int>(H), static_cast<int>(Is)) * sizeof(float) : 0);
  L.total = off;
  return L;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status moe_config_validate(const moe_config* cfg) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  if (c.hidden < 8 || c.hidden % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.expert_inter < 8 || c.expert_inter % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.shared_inter < 0 || c.shared_inter % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.num_experts < 1) return MOE_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > c.num_experts) return MOE_ERR_INVALID_ARG;
  if (c.num_experts > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (c.top_k > MOE_MAX_TOP_K) return MOE_ERR_UNSUPPORTED;
  if (std::isnan(c.swiglu_limit) || !(c.swiglu_limit > 0.f)) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(c.routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  if (c.renormalize != 0 && c.renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (c.expert_format != MOE_W_BF16 && c.expert_format != MOE_W_INT4_G128 && c.expert_format != MOE_W_NVFP4)
    return MOE_ERR_INVALID_ARG;
  const bool four = c.expert_format != MOE_W_BF16;
  if (four && (c.hidden % 128 != 0 || c.expert_inter % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  // the 4-bit paths feed h to fp16 tensor-core operands: |h| <= L^2 must stay finite in fp16
  if (four && !(c.swiglu_limit <= MOE_INT4_MAX_SWIGLU_LIMIT)) return MOE_ERR_UNSUPPORTED;
  // TMA strides and boxes: rows of up to 2^31 bytes
  if (static_cast<int64_t>(c.hidden) * 2 >= (int64_t(1) << 31) ||
      static_cast<int64_t>(c.expert_inter) * 2 >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status moe_workspace_size(const moe_config* cfg, int32_t max_tokens, size_t* bytes) {
  MOE_TRY(moe_config_validate(cfg));
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_tokens(*cfg, max_tokens));
  *bytes = ws_layout(*cfg, max_tokens).total;
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, sizeof(WsHeader), stream));
}

moe_status moe_router_topk(const moe_config* cfg, const moe_weights* w, const void* x, int32_t T, int32_t* topk_ids,
                           float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_router_weights(w));
  if (x == nullptr || topk_ids == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(topk_ids) || !aligned16(topk_w)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  return from_cuda(launch_router(*cfg, *w, x, T, topk_ids, topk_w, at<float>(ws, L.logits), at<void>(ws, L.w_split),
                                 err_word(ws), num_sms_current_device(), stream));
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_ids, const float* topk_w, const void* x, int32_t T,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* src, float* w_perm, void* x_perm, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  const void* ptrs[] = {topk_ids, topk_w, expert_offsets, row_of, src, w_perm};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  // x_perm == NULL: maps and weights only (x is then not read)
  if (x_perm != nullptr && (x == nullptr || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  return from_cuda(launch_permute(*cfg, topk_ids, topk_w, x, T, expert_offsets, row_of, src, w_perm, x_perm,
                                  at<int32_t>(ws, L.block_base), at<int32_t>(ws, L.local_rank), perm_ticket(ws),
                                  stream));
}

moe_status moe_grouped_swiglu_ffn(const moe_config* cfg, const moe_weights* w, const void* x_perm,
                                  const int32_t* expert_offsets, const float* w_perm, int32_t T, void* y_perm,
                                  const void* x_shared, void* shared_out, void* ws, size_t ws_bytes,
                                  moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_expert_weights(*cfg, w));
  if (x_perm == nullptr || expert_offsets == nullptr || y_perm == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(expert_offsets) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  if (w_perm != nullptr && !aligned16(w_perm)) return MOE_ERR_INVALID_ARG;
  if (x_shared != nullptr) {
    if (cfg->shared_inter == 0 || shared_out == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_shared) || !aligned16(shared_out)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_shared_weights(*cfg, w));
  }
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  return run_ffn(*cfg, *w, x_perm, nullptr, expert_offsets, w_perm, T, y_perm, x_shared, shared_out, ws, L, stream,
                 cfg->num_experts);
}

moe_status moe_grouped_swiglu_ffn_gather(const moe_config* cfg, const moe_weights* w, const void* x, int32_t T,
                                         const int32_t* src, const int32_t* expert_offsets, const float* w_perm,
                                         void* y_perm, void* shared_out, void* ws, size_t ws_bytes,
                                         moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_expert_weights(*cfg, w));
  if (x == nullptr || src == nullptr || expert_offsets == nullptr || y_perm == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(src) || !aligned16(expert_offsets) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (w_perm != nullptr && !aligned16(w_perm)) return MOE_ERR_INVALID_ARG;
  if (shared_out != nullptr) {
    if (cfg->shared_inter == 0 || !aligned16(shared_out)) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_shared_weights(*cfg, w));
  }
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  return run_ffn(*cfg, *w, x, src, expert_offsets, w_perm, T, y_perm, shared_out != nullptr ? x : nullptr, shared_out,
                 ws, L, stream, cfg->num_experts);
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* row_of, const float* topk_w,
                       const void* shared_out, int32_t T, void* out, moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  if (y_perm == nullptr || row_of == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(row_of) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (topk_w != nullptr && !aligned16(topk_w)) return MOE_ERR_INVALID_ARG;
  if (shared_out != nullptr && !aligned16(shared_out)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  return from_cuda(launch_combine(*cfg, y_perm, row_of, topk_w, shared_out, T, out, nullptr, 0, stream));
}

moe_status moe_forward(const moe_config* cfg, const moe_weights* w, const void* x, int32_t T, void* out,
                       int32_t* topk_ids_opt, float* topk_w_opt, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_router_weights(w));
  MOE_TRY(check_expert_weights(*cfg, w));
  MOE_TRY(check_shared_weights(*cfg, w));
  if (x == nullptr || out == nullptr || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if ((topk_ids_opt != nullptr && !aligned16(topk_ids_opt)) || (topk_w_opt != nullptr && !aligned16(topk_w_opt)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  int32_t* ids = topk_ids_opt != nullptr ? topk_ids_opt : at<int32_t>(ws, L.ids);
  float* wts = topk_w_opt != nullptr ? topk_w_opt : at<float>(ws, L.wts);
  MOE_CUDA_TRY(launch_router(*cfg, *w, x, T, ids, wts, at<float>(ws, L.logits), at<void>(ws, L.w_split),
                             err_word(ws), num_sms_current_device(), stream));
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  float* w_perm = at<float>(ws, L.w_perm);
  int32_t* src = at<int32_t>(ws, L.src);
  const Rows rows = routed_rows(*cfg, ws, L, x, src);
  MOE_CUDA_TRY(launch_permute(*cfg, ids, wts, x, T, offsets, row_of, src, w_perm, rows.x_perm,
                              at<int32_t>(ws, L.block_base), at<int32_t>(ws, L.local_rank), perm_ticket(ws),
                              stream));
  void* y_perm = at<void>(ws, L.y_perm);
  const bool shared = cfg->shared_inter > 0;
  void* shared_out = shared ? at<void>(ws, L.shared_out) : nullptr;
  MOE_TRY(run_ffn(*cfg, *w, rows.x_rows, rows.gather_src, offsets, w_perm, T, y_perm, shared ? x : nullptr,
                  shared_out, ws, L, stream, cfg->num_experts));
  return from_cuda(launch_combine(*cfg, y_perm, row_of, nullptr, shared_out, T, out, nullptr, 0, stream));
}

moe_status moe_forward_ep(const moe_config* cfg, const moe_weights* w, int32_t expert_begin, int32_t expert_end,
                          const void* x, int32_t T, void* out_partial, int32_t* topk_ids_opt, float* topk_w_opt,
                          void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(moe_config_validate(cfg));
  MOE_TRY(check_tokens(*cfg, T));
  MOE_TRY(check_router_weights(w));
  if (expert_begin < 0 || expert_end < expert_begin || expert_end > cfg->num_experts) return MOE_ERR_INVALID_ARG;
  const int El = expert_end - expert_begin;
  if (El > 0) MOE_TRY(check_expert_weights(*cfg, w));
  MOE_TRY(check_shared_weights(*cfg, w));
  if (x == nullptr || out_partial == nullptr || !aligned16(x) || !aligned16(out_partial)) return MOE_ERR_INVALID_ARG;
  if ((topk_ids_opt != nullptr && !aligned16(topk_ids_opt)) || (topk_w_opt != nullptr && !aligned16(topk_w_opt)))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(*cfg, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(*cfg, T);
  int32_t* ids = topk_ids_opt != nullptr ? topk_ids_opt : at<int32_t>(ws, L.ids);
  float* wts = topk_w_opt != nullptr ? topk_w_opt : at<float>(ws, L.wts);
  // the router ranks every expert ([glm5next]: it is given the full count)
  MOE_CUDA_TRY(launch_router(*cfg, *w, x, T, ids, wts, at<float>(ws, L.logits), at<void>(ws, L.w_split),
                             err_word(ws), num_sms_current_device(), stream));
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  float* w_perm = at<float>(ws, L.w_perm);
  int32_t* src = at<int32_t>(ws, L.src);
  const Rows rows = routed_rows(*cfg, ws, L, x, src);
  MOE_CUDA_TRY(launch_permute(*cfg, ids, wts, x, T, offsets, row_of, src, w_perm, rows.x_perm,
                              at<int32_t>(ws, L.block_base), at<int32_t>(ws, L.local_rank), perm_ticket(ws), stream,
                              expert_begin, expert_end));
  void* y_perm = at<void>(ws, L.y_perm);
  const bool shared = cfg->shared_inter > 0;
  void* shared_out = shared ? at<void>(ws, L.shared_out) : nullptr;
  moe_config local = *cfg;
  local.num_experts = El;
  MOE_TRY(run_ffn(local, *w, rows.x_rows, rows.gather_src, offsets + expert_begin, w_perm, T, y_perm,
                  shared ? x : nullptr, shared_out, ws, L, stream, cfg->num_experts));
  return from_cuda(launch_combine(*cfg, y_perm, row_of, nullptr, shared_out, T, out_partial, offsets + expert_begin,
                                  El, stream));
}

moe_status moe_selftest_device_timeout(void* scratch, size_t scratch_bytes, moe_stream_t stream) {
  if (scratch == nullptr || scratch_bytes < MOE_SELFTEST_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(cudaMemsetAsync(scratch, 0, MOE_SELFTEST_SCRATCH_BYTES, stream));
  return from_cuda(launch_splitk_timeout_selftest(scratch, err_word(scratch), stream));
}

moe_status moe_selftest_pair_timeout(void* scratch, size_t scratch_bytes, int32_t kernel, moe_stream_t stream) {
  if (scratch == nullptr || scratch_bytes < MOE_SELFTEST_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (kernel != MOE_SELFTEST_PAIR_BF16 && kernel != MOE_SELFTEST_PAIR_INT4) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(cudaMemsetAsync(scratch, 0, MOE_SELFTEST_SCRATCH_BYTES, stream));
  if (kernel == MOE_SELFTEST_PAIR_BF16)
    return from_cuda(launch_pair_timeout_selftest(scratch, err_word(scratch), tile_queue(scratch, kQueueGateUp), stream));
  return from_cuda(
      launch_int4_pair_timeout_selftest(scratch, err_word(scratch), tile_queue(scratch, kQueueInt4GateUp), stream));
}

moe_status moe_read_device_error(void* ws, moe_stream_t stream, int32_t* code) {
  if (ws == nullptr || code == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  WsHeader h;
  if (cudaMemcpy(&h, ws, sizeof(int32_t) * 2, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *code = h.error;
  if (h.error != 0 && cudaMemset(ws, 0, sizeof(int32_t) * 2) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
