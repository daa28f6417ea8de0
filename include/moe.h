/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts SwiGLU
 * layer forward: fp32 router with sigmoid scores and correction-bias top-k,
 * token permute by expert, grouped gate/up GEMM with the clamped SwiGLU
 * fused, grouped down GEMM with the combine weights fused, and one combine
 * kernel that adds the shared expert.
 *
 * Sources for what each call computes (web pages on the method):
 *   [glm5next] "Module glm5next_mlp" (metrale model-arch docs): §Numerics the
 *              kernels rely on; §One all-reduce for both EP and TP; constant
 *              KERNEL_MAX_TOP_K; modules forward, forward_prefill_gemm, build;
 *              MOE_MODULE (token sort / permute / unpermute);
 *              W4A16_GEMV_MODULE (routed projections outside the grouped
 *              prefill GEMM).
 *   [mstar]    "mstar.model.components.distributed.mlp", ParallelGatedMLP:
 *              fused gate/up projection (gate = shard 0, up = shard 1).
 *   [beam]     "bridge.models.beam.modeling_beam", beam_router_gating_linear
 *              and BeamTopKRouter: router logits inp @ weight.T with both
 *              operands in fp32.
 *
 * Notation: T tokens, H hidden, E routed experts, k top_k, I expert
 * intermediate, I_s shared-expert intermediate, L swiglu_limit,
 * alpha routed_scaling_factor, R = T*k routed rows.
 *
 * Conventions that hold for every call:
 *   - Every data pointer is a DEVICE pointer (cudaMalloc / torch CUDA
 *     memory) on the current device, unless a parameter says otherwise.
 *     The caller owns every buffer.  The library never allocates, frees,
 *     synchronises (except moe_read_device_error) or throws.
 *   - All work is enqueued on `stream` (NULL = the legacy default stream).
 *   - Arguments are validated on the host before anything is launched; a
 *     non-OK status means nothing was enqueued.
 *   - Row-major layouts; bf16 is IEEE bfloat16 stored as uint16.
 *   - Data pointers must be 16-byte aligned (the NVFP4 tensor scales: 4
 *     bytes); H, I and I_s multiples of 8 (16-byte rows); the W4A16 and
 *     NVFP4 formats need H and I multiples of 128.
 *   - T == 0 returns MOE_OK and launches nothing.
 *   - `ws` is a caller-owned device workspace of at least
 *     moe_workspace_size(cfg, T) bytes, 256-byte aligned, whose first 256
 *     bytes (the header) were zeroed once by moe_workspace_init.  The same
 *     workspace serves every call below for token counts <= that T.  Calls
 *     that share one workspace must be ordered on the GPU (same stream).
 */
#ifndef ROUTED_SWIGLU_EXPERTS_B200_MOE_H
#define ROUTED_SWIGLU_EXPERTS_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size or value */
  MOE_ERR_UNSUPPORTED = 2,    /* valid but outside this build's limits */
  MOE_ERR_WORKSPACE = 3,      /* workspace missing or too small */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5  /* a bounded wait inside a kernel gave up */
} moe_status;

typedef enum moe_weight_format {
  MOE_W_BF16 = 0,        /* routed expert weights in bf16 */
  MOE_W_INT4_G128 = 1,   /* W4A16: uint4 codes, bf16 scale per 128 along K */
  MOE_W_NVFP4 = 2        /* NVFP4: E2M1 codes, E4M3 scale per 16 along K,
                            fp32 scale per expert weight tensor */
} moe_weight_format;

/* Largest k the router kernel selects per token ([glm5next] constant
 * KERNEL_MAX_TOP_K: the per-token selection lives in 16-entry arrays). */
#define MOE_MAX_TOP_K 16
/* Largest routed expert count this build supports. */
#define MOE_MAX_EXPERTS 1024

/* Geometry and numerics of one MoE layer. */
typedef struct moe_config {
  int32_t hidden;                /* H  (multiple of 8) */
  int32_t num_experts;           /* E  (1..MOE_MAX_EXPERTS); the FULL routed
                                    count: the router ranks all experts */
  int32_t top_k;                 /* k  (1..min(E, MOE_MAX_TOP_K)) */
  int32_t expert_inter;          /* I  (multiple of 8) */
  int32_t shared_inter;          /* I_s (multiple of 8; 0 = no shared expert) */
  float swiglu_limit;            /* L > 0, required (no default); +inf = no
                                    clamp.  gate <- min(gate, L),
                                    up <- clamp(up, -L, L).  W4A16 and NVFP4
                                    experts: L <= MOE_INT4_MAX_SWIGLU_LIMIT */
  float routed_scaling_factor;   /* alpha: multiplies the routed weights; the
                                    shared expert is added unscaled */
  int32_t renormalize;           /* 1: divide the k unbiased scores by their
                                    sum before alpha; 0: no renormalisation */
  int32_t expert_format;         /* moe_weight_format */
} moe_config;

/* Device weight handles of one layer.  Gate rows come first in every fused
 * gate/up weight ([mstar] ParallelGatedMLP: gate = shard 0, up = shard 1). */
typedef struct moe_weights {
  const float* router_w;         /* fp32 [E, H] */
  const float* correction_bias;  /* fp32 [E], or NULL for zero bias */
  /*                                bf16            | W4A16                  | NVFP4 */
  const void* w_gate_up;         /* bf16 [E, 2I, H] | uint8 [E, 2I, H/2]     | uint8 [E, 2I, H/2] */
  const void* s_gate_up;         /* NULL            | bf16  [E, 2I, H/128]   | E4M3 uint8 [E, 2I, H/16] */
  const void* w_down;            /* bf16 [E, H, I]  | uint8 [E, H, I/2]      | uint8 [E, H, I/2] */
  const void* s_down;            /* NULL            | bf16  [E, H, I/128]    | E4M3 uint8 [E, H, I/16] */
  const void* shared_w_gate_up;  /* bf16 [2I_s, H] (NULL iff I_s == 0), every format */
  const void* shared_w_down;     /* bf16 [H, I_s]  (NULL iff I_s == 0), every format */
  const float* g_gate_up;        /* NVFP4: fp32 [E] tensor scale of each gate/up weight; else ignored */
  const float* g_down;           /* NVFP4: fp32 [E] tensor scale of each down weight; else ignored */
} moe_weights;
/* W4A16 (int4) packing: byte q[n, c] holds the codes of k = 2c (low nibble)
 * and k = 2c + 1 (high nibble); w[n, k] = (code - 8) * scale[n, k / 128].
 *
 * Range of the W4A16 paths.  Both int4 paths multiply on fp16 tensor-core
 * operands (fp32 accumulation): the tokens x and the SwiGLU activations h
 * (already rounded to bf16) are converted to fp16, and the grouped prefill
 * GEMM also forms the weights (code - 8) * scale in fp16.  Hence:
 *   - swiglu_limit must be finite and at most MOE_INT4_MAX_SWIGLU_LIMIT, so
 *     that |h| <= L * L stays finite in fp16 (moe_config_validate returns
 *     MOE_ERR_UNSUPPORTED otherwise; bf16 experts have no such limit);
 *   - |x| must stay below 65504 (larger activations become inf; this is not
 *     checked, the values live on the device);
 *   - |x| and |h| below about 1e-3, and scales below 2^-14 (prefill GEMM),
 *     fall into fp16's subnormal range and keep fewer significant bits
 *     (the GEMV stores half of the activations divided by 16);
 *   - 8 * |scale| must stay below 65504 (prefill GEMM).
 * The benchmark layers (x ~ N(0, 1), scales in [0.005, 0.02], L = 7) sit far
 * inside these bounds. */
#define MOE_INT4_MAX_SWIGLU_LIMIT 255.0f

/* NVFP4 packing ([glm5next] module summary: routed NVFP4 MoE; element
 * formats of the OCP specifications: FP4 E2M1 of Microscaling Formats v1.0,
 * FP8 E4M3 of 8-bit Floating Point): byte q[n, c] holds the E2M1 codes of
 * k = 2c (low nibble) and k = 2c + 1 (high nibble);
 *   w[n, k] = e2m1(code) * e4m3(s[n, k / 16]) * g[e].
 * Both NVFP4 kernels form e2m1 * e4m3 in fp16, which is exact for every
 * finite E4M3 scale (the E4M3 NaN patterns give NaN weights), and multiply
 * the fp32 sums by g[e]; the activation limits of the W4A16 range note above
 * (fp16 x and h, swiglu_limit) hold as stated there. */

/* Human-readable name of a status.  Never NULL. */
MOE_API const char* moe_status_string(moe_status status);

/* Validate a configuration (sizes, limits, swiglu_limit not NaN and > 0).
 * Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_config_validate(const moe_config* cfg);

/* Host only.  Bytes of device workspace that every call below needs for up
 * to `max_tokens` tokens.  *bytes is written on MOE_OK. */
MOE_API moe_status moe_workspace_size(const moe_config* cfg, int32_t max_tokens, size_t* bytes);

/* Zero the workspace header on `stream`: the device error word and the
 * tile counters of the grouped GEMMs (every launch leaves those at zero
 * again).  Call once after allocating a workspace. */
MOE_API moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router: logit[t, e] = sum_h x[t, h] * router_w[e, h] in fp32 ([beam]
 * beam_router_gating_linear; no linear bias); s = sigmoid(logit); the k
 * experts with the largest s + correction_bias, ties to the lower id
 * ([glm5next] §Numerics: the bias steers selection only).  The logits run
 * on the tensor cores with the fp32 weight split exactly into three bf16
 * parts; selections whose fp32 biased scores are within 2^-13 of a neighbour
 * are re-ranked from fp64 logits so the ids equal the exact-arithmetic
 * selection.
 *   x         bf16 [T, H]
 *   topk_ids  int32 [T, k] out: selection order (biased desc, id asc)
 *   topk_w    fp32  [T, k] out: alpha * s_e (renormalised first if enabled),
 *             from the UNBIASED score. */
MOE_API moe_status moe_router_topk(const moe_config* cfg, const moe_weights* w,
                           const void* x, int32_t T,
                           int32_t* topk_ids, float* topk_w,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Token sort / permute by expert ([glm5next] MOE_MODULE): a deterministic
 * stable counting sort of the slots i = t*k + j by expert id.
 *   topk_ids        int32 [T, k] in (each in [0, E), distinct per token)
 *   topk_w          fp32  [T, k] in
 *   x               bf16  [T, H] in (not read when x_perm is NULL)
 *   expert_offsets  int32 [E+1] out: expert e owns rows [off[e], off[e+1])
 *   row_of          int32 [T*k] out: routed row of slot i
 *   src             int32 [T*k] out: slot i of routed row r (inverse of row_of)
 *   w_perm          fp32  [T*k] out: w_perm[row_of[i]] = topk_w[i]
 *   x_perm          bf16  [T*k, H] out: x_perm[row_of[i]] = x[i / k];
 *                   or NULL: the maps and weights only, for
 *                   moe_grouped_swiglu_ffn_gather, which reads the rows
 *                   from x itself
 * Inside an expert, rows are in ascending token order.  Ids outside [0, E)
 * are undefined behaviour. */
MOE_API moe_status moe_permute(const moe_config* cfg, const int32_t* topk_ids,
                       const float* topk_w, const void* x, int32_t T,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* src,
                       float* w_perm, void* x_perm,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped expert FFN, one launch per projection for all experts
 * ([glm5next] forward_prefill_gemm): for every routed row r of expert e,
 *   y_perm[r] = bf16( w_perm[r] * W_down[e] h ),
 *   h = bf16( silu(min(W_gate[e] x_perm[r], L)) * clamp(W_up[e] x_perm[r], -L, L) )
 * ([glm5next] §Numerics: asymmetric clamp).  w_perm == NULL: unweighted.
 * bf16 weights run on the tcgen05 tensor cores.  MOE_W_INT4_G128 weights
 * run the W4A16 GEMV kernels that dequantise in registers ([glm5next]
 * W4A16_GEMV_MODULE) when there are fewer than 32 routed rows per expert on
 * average, else a grouped tensor-core GEMM that dequantises the int4 codes
 * into fp16 tiles in shared memory ([glm5next] MOE_GROUPED_MODULE).
 * MOE_W_NVFP4 weights take the same two kernels by the same rule, decoding
 * E2M1 codes and E4M3 block scales (in registers, or into the fp16 tiles).
 * Every format rounds h to bf16 as the bf16 path does.
 * When x_shared != NULL the shared expert runs in the same launches:
 *   shared_out[t] = bf16( SwiGLU_clamped FFN_shared(x_shared[t]) ), unscaled.
 *   x_perm          bf16 [T*k, H]    expert_offsets int32 [E+1]
 *   w_perm          fp32 [T*k] or NULL
 *   y_perm          bf16 [T*k, H] out
 *   x_shared        bf16 [T, H] or NULL;  shared_out bf16 [T, H] out */
MOE_API moe_status moe_grouped_swiglu_ffn(const moe_config* cfg, const moe_weights* w,
                                  const void* x_perm, const int32_t* expert_offsets,
                                  const float* w_perm, int32_t T, void* y_perm,
                                  const void* x_shared, void* shared_out,
                                  void* ws, size_t ws_bytes, moe_stream_t stream);

/* The grouped expert FFN with the permute's gather fused into its first
 * loads ([glm5next] MOE_MODULE token permute and forward_prefill_gemm): the
 * same result as moe_grouped_swiglu_ffn on x_perm[r] = x[src[r] / k], but
 * routed row r is read straight from token src[r] / k of x, so x_perm is
 * never written.  The 4-bit kernels gather while converting the activations
 * to fp16 (the conversion pass they run anyway).  The bf16 tensor-core
 * kernel copies four token rows per TMA gather: correct, but on a B200 its
 * gate/up launch takes about twice as long as with the contiguous token
 * boxes of moe_grouped_swiglu_ffn, more than the x_perm copy it saves, so
 * moe_forward keeps the copy for bf16 experts.
 * The shared expert runs on x in the same launches when shared_out != NULL.
 *   x               bf16 [T, H]      src int32 [T*k] (moe_permute's)
 *   expert_offsets  int32 [E+1]      w_perm fp32 [T*k] or NULL
 *   y_perm          bf16 [T*k, H] out
 *   shared_out      bf16 [T, H] out, or NULL (no shared expert)
 * src must be a permutation of [0, T*k) (moe_permute's output); other
 * values are undefined behaviour. */
MOE_API moe_status moe_grouped_swiglu_ffn_gather(const moe_config* cfg, const moe_weights* w,
                                                 const void* x, int32_t T, const int32_t* src,
                                                 const int32_t* expert_offsets, const float* w_perm,
                                                 void* y_perm, void* shared_out,
                                                 void* ws, size_t ws_bytes, moe_stream_t stream);

/* Combine ([glm5next] §One all-reduce: shared output and routed slots are
 * added in one combine kernel):
 *   out[t] = bf16( shared_out[t] + sum_{j<k} c_j * y_perm[row_of[t*k + j]] )
 * summed in fp32 in slot order, c_j = topk_w[t, j], or 1 when topk_w is
 * NULL (y_perm already weighted).  shared_out may be NULL (no shared term).
 *   y_perm bf16 [T*k, H]; row_of int32 [T*k]; out bf16 [T, H] (must not
 *   alias the inputs). */
MOE_API moe_status moe_combine(const moe_config* cfg, const void* y_perm,
                       const int32_t* row_of, const float* topk_w,
                       const void* shared_out, int32_t T, void* out,
                       moe_stream_t stream);

/* The whole layer in one call: router -> permute -> grouped FFN (routed +
 * shared) -> combine, enqueued on `stream` with no host synchronisation.
 * bf16 experts: the permute writes x_perm into the workspace and the FFN
 * loads contiguous token boxes.  int4 and NVFP4 experts: the permute writes
 * the maps only and the FFN gathers the rows as moe_grouped_swiglu_ffn_gather
 * does.
 *   x    bf16 [T, H];  out bf16 [T, H]
 *   topk_ids_opt int32 [T, k] / topk_w_opt fp32 [T, k]: if non-NULL, the
 *   router's selection is also written there. */
MOE_API moe_status moe_forward(const moe_config* cfg, const moe_weights* w,
                       const void* x, int32_t T, void* out,
                       int32_t* topk_ids_opt, float* topk_w_opt,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* Expert-parallel forward of one rank ([glm5next] §One all-reduce for both EP
 * and TP: each rank combines the shared output and its local routed slots,
 * then one all-reduce of the [T, H] partial sums gives the layer output;
 * the router is replicated and ranks all experts, and the ranks' expert
 * ranges partition [0, E)).
 *   out_partial[t] = bf16( shared_r(x[t])
 *                          + sum over slots j with expert_begin <= e_j < expert_end
 *                            of w_j * FFN_{e_j}(x[t]) )
 * summed in fp32 in slot order, where shared_r is this rank's slice of the
 * shared expert (its SwiGLU is per intermediate feature, so a slice of the
 * intermediate dimension is a narrower shared expert, and the slices' down
 * projections add up to the whole).  Adding the ranks' out_partial gives
 * moe_forward's output (up to rounding) when their expert ranges partition
 * [0, E) and their shared slices partition [0, I_s).
 *   cfg   as for moe_forward, except cfg->shared_inter = this rank's slice
 *         width of the shared intermediate (0: no shared work on this rank);
 *         cfg->num_experts is the full E (the router ranks every expert).
 *   w     router_w / correction_bias: the full [E, H] / [E];
 *         w_gate_up, w_down (and s_gate_up, s_down, g_gate_up, g_down):
 *         the LOCAL experts only,
 *         [expert_end - expert_begin, ...], local expert 0 = global expert
 *         expert_begin (may be NULL when the range is empty);
 *         shared_w_gate_up [2 I_s_local, H] (the slice's gate rows, then its
 *         up rows) and shared_w_down [H, I_s_local] (the slice's columns).
 *   0 <= expert_begin <= expert_end <= E, else MOE_ERR_INVALID_ARG.
 *   x bf16 [T, H] (every rank gets all T tokens); out_partial bf16 [T, H].
 *   topk_ids_opt / topk_w_opt: as for moe_forward (every token's selection).
 * The workspace is sized by moe_workspace_size(cfg, T) with this rank's cfg.
 * The all-reduce itself is the caller's (NCCL over NVLink, one call). */
MOE_API moe_status moe_forward_ep(const moe_config* cfg, const moe_weights* w, int32_t expert_begin,
                                  int32_t expert_end, const void* x, int32_t T, void* out_partial,
                                  int32_t* topk_ids_opt, float* topk_w_opt, void* ws, size_t ws_bytes,
                                  moe_stream_t stream);

/* Permute without a workspace, for callers that may not allocate device
 * memory on their enqueue path (framework / inference-server plugins and
 * serving loops that own all device memory and only pass their own input
 * and output buffers; allocating there can stall the device and breaks
 * their fixed memory budget).  The method's pages have no counterpart of
 * this call: it exists only for that deployment constraint.
 *
 * Same arguments, outputs and results as moe_permute, minus ws/ws_bytes.
 * Its scratch is one fixed array inside this library
 * (MOE_NO_ALLOC_SCRATCH_BYTES on every GPU that loads the library, held
 * until the process exits), so:
 *   - T * k above MOE_NO_ALLOC_MAX_ROWS returns MOE_ERR_UNSUPPORTED (use
 *     moe_permute with a workspace for larger batches);
 *   - the first call in each CUDA context (normally the device's primary
 *     context: once per device) looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it under
 *     the context's id, so a context created after cudaDeviceReset, or a
 *     non-primary context made current by the caller, gets its own lookup;
 *     make that first call before capturing any stream;
 *   - every call shares the array: calls whose kernels may overlap on the
 *     GPU (other streams, other host threads) race and must be ordered on
 *     one stream.  Nothing in it needs clearing between calls: the one
 *     word that must start at zero (the count kernel's ticket counter) is
 *     zero when the library loads and every call leaves it at zero.
 * Never calls cudaMalloc / cudaFree or any allocating routine. */
#define MOE_NO_ALLOC_MAX_ROWS 131072
#define MOE_NO_ALLOC_SCRATCH_BYTES 786688
MOE_API moe_status moe_permute_no_alloc(const moe_config* cfg, const int32_t* topk_ids,
                                        const float* topk_w, const void* x, int32_t T,
                                        int32_t* expert_offsets, int32_t* row_of, int32_t* src,
                                        float* w_perm, void* x_perm, moe_stream_t stream);

/* Synchronise `stream`, then read and clear the workspace's device error
 * word.  *code receives MOE_OK, or MOE_ERR_DEVICE_TIMEOUT if a kernel's
 * bounded wait gave up since the last read.  Intended for tests and
 * debugging. */
MOE_API moe_status moe_read_device_error(void* ws, moe_stream_t stream, int32_t* code);

/* Test hook for the device-timeout path; the pages have no counterpart (it
 * checks this library's own failure handling).  Zeroes `scratch` (device,
 * 256-byte aligned, at least MOE_SELFTEST_SCRATCH_BYTES) and launches the
 * split-K tensor-core GEMM on one 128 x 16 x 64 tile of zero operands held
 * in it, with the signal that the tile's MMAs finished withheld and every
 * wait limited to 20 ms.  The epilogue's wait runs out, the kernel records
 * MOE_ERR_DEVICE_TIMEOUT in scratch's error word, drains its own copy and
 * MMAs, frees its tensor memory and exits; the context stays usable.  Read
 * the result with moe_read_device_error(scratch, ...).  Returns MOE_OK once
 * the launch is enqueued. */
#define MOE_SELFTEST_SCRATCH_BYTES 65536
MOE_API moe_status moe_selftest_device_timeout(void* scratch, size_t scratch_bytes, moe_stream_t stream);

/* Test hook for the timeout paths of the grouped GEMMs that run on CTA
 * pairs; the pages have no counterpart.  Zeroes `scratch` (as above; its
 * first 256 bytes are laid out like a workspace header) and launches one
 * pair (two CTAs on two SMs) of
 *   MOE_SELFTEST_PAIR_BF16: the bf16 grouped gate/up kernel, or
 *   MOE_SELFTEST_PAIR_INT4: the int4 (W4A16 prefill) grouped gate/up kernel,
 * on one tiny tile of zero operands held in scratch, with the signal that
 * the tile's accumulator is complete never sent to the epilogue and every
 * wait on another role limited to 20 ms.  Both CTAs' epilogue waits run
 * out; the kernel records MOE_ERR_DEVICE_TIMEOUT in scratch's error word,
 * every other role finishes, the copies and MMAs drain, the pair resets
 * its tile-queue words in the header to zero and frees its tensor memory,
 * and the context stays usable.  Read the result with
 * moe_read_device_error(scratch, ...).  Returns MOE_OK once the launch is
 * enqueued; MOE_ERR_INVALID_ARG for another `kernel`. */
#define MOE_SELFTEST_PAIR_BF16 0
#define MOE_SELFTEST_PAIR_INT4 1
MOE_API moe_status moe_selftest_pair_timeout(void* scratch, size_t scratch_bytes, int32_t kernel,
                                             moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ROUTED_SWIGLU_EXPERTS_B200_MOE_H */
