// moe_permute_no_alloc: the token permute for callers that cannot hand the
// library a workspace.
//
// Who needs it: hosts that own every byte of device memory and only pass
// their own input/output buffers at enqueue time -- inference-server and
// framework plugins, and latency-critical serving loops -- are often not
// allowed to call cudaMalloc on that path, because allocating can stall or
// synchronise the device and breaks their fixed memory budget.  This entry
// point takes only inputs and outputs; its scratch (per-chunk expert counts
// and per-slot ranks) lives in one fixed device array in this library.
//
// The array is a file-scope __device__ symbol, so every GPU that loads the
// library holds it (MOE_NO_ALLOC_SCRATCH_BYTES) until the process exits.
// Host code may not use the symbol's name as a device address: the first
// call in each CUDA context (normally: on each device) looks up the real
// address with cudaGetSymbolAddress (with that device current) and caches it
// under the context's id.  Every call reuses the same
// array, so two calls whose kernels overlap on the GPU (different streams,
// or different host threads) race on it; order them on one stream.
#include <mutex>

#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kNoAllocMaxChunks = MOE_NO_ALLOC_MAX_ROWS / kPermChunk;
constexpr size_t kNoAllocTicketInts = 64;  // one ticket word, padded to 256 bytes
constexpr size_t kNoAllocBlockBaseInts = static_cast<size_t>(kNoAllocMaxChunks) * MOE_MAX_EXPERTS;
constexpr size_t kNoAllocScratchInts = kNoAllocTicketInts + kNoAllocBlockBaseInts + MOE_NO_ALLOC_MAX_ROWS;
static_assert(MOE_NO_ALLOC_MAX_ROWS % kPermChunk == 0, "whole chunks");
static_assert(kNoAllocScratchInts * sizeof(int32_t) == MOE_NO_ALLOC_SCRATCH_BYTES, "documented size");

// [64] the count blocks' ticket counter (word 0), then [kNoAllocMaxChunks * E]
// chunk counts / bases, then [T*k] in-chunk ranks.  The counter is zero when
// the module loads and every call leaves it at zero; the other two parts are
// fully written by the count kernel before anything reads them.  So nothing
// has to be cleared between calls.
static __device__ __align__(256) int32_t g_perm_scratch[kNoAllocScratchInts];

// Driver entry points for the context the runtime made current (fetched
// through the runtime, as for the TMA encoder: no libcuda at link time).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Device address of g_perm_scratch in the current context.  Each CUDA
// context holds its own copy of the module, so the address is looked up
// (cudaGetSymbolAddress, with the device current) once per context and
// cached under the context's process-unique id: a context made after a
// cudaDeviceReset, or a non-primary context the caller made current, gets an
// id of its own and its own lookup, never a stale address.
cudaError_t scratch_address(int32_t** out) {
  static std::mutex mu;
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool fns_loaded = false;
  constexpr int kSlots = 64;
  static unsigned long long ids[kSlots];
  static int32_t* addrs[kSlots];
  static int used = 0;
  static int next_victim = 0;
  cudaError_t e = cudaSuccess;
  std::lock_guard<std::mutex> lk(mu);
  if (!fns_loaded) {
    get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    fns_loaded = true;
  }
  if (get_ctx == nullptr || get_id == nullptr) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  unsigned long long id = 0;
  void* p = nullptr;
  if (ctx == nullptr) {
    // no context current on this thread yet: the runtime makes the device's
    // primary context current while it looks the symbol up
    e = cudaGetSymbolAddress(&p, g_perm_scratch);
    if (e != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  if (get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  for (int i = 0; i < used; ++i)
    if (ids[i] == id) {
      *out = addrs[i];
      return cudaSuccess;
    }
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_perm_scratch);
    if (e != cudaSuccess) return e;
  }
  int slot = used < kSlots ? used++ : (next_victim++ % kSlots);
  ids[slot] = id;
  addrs[slot] = static_cast<int32_t*>(p);
  *out = addrs[slot];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace moe

extern "C" MOE_API moe_status moe_permute_no_alloc(const moe_config* cfg, const int32_t* topk_ids,
                                                   const float* topk_w, const void* x, int32_t T,
                                                   int32_t* expert_offsets, int32_t* row_of, int32_t* src,
                                                   float* w_perm, void* x_perm, moe_stream_t stream) {
  using namespace moe;
  const moe_status st = moe_config_validate(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * cfg->top_k > MOE_NO_ALLOC_MAX_ROWS) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {topk_ids, topk_w, x, expert_offsets, row_of, src, w_perm, x_perm};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  int32_t* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t* ticket = scratch;
  int32_t* block_base = scratch + kNoAllocTicketInts;
  int32_t* local_rank = block_base + kNoAllocBlockBaseInts;
  const cudaError_t e = launch_permute(*cfg, topk_ids, topk_w, x, T, expert_offsets, row_of, src, w_perm, x_perm,
                                       block_base, local_rank, ticket, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
