// Router: the fp32 logits GEMM runs on the tensor cores (splitk_gemm.cu, three
// passes over K) on an exact bf16 split of the fp32 weight; here are the split
// and the sigmoid + biased top-k (one warp per token, with an fp64 re-rank
// of near-ties).
//
// "Module glm5next_mlp" §Numerics: sigmoid score; the correction bias steers
// selection only; the emitted weight is the unbiased score times
// routed_scaling_factor.  "bridge.models.beam.modeling_beam"
// beam_router_gating_linear: logits = inp @ weight.T with fp32 operands.
#include "moe_internal.h"

namespace moe {

namespace {

// Exact three-way split of the fp32 router weight into bf16 parts:
// hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid); both
// subtractions are exact in fp32, and hi + mid + lo carries 24 significant
// bits, so x * (hi + mid + lo) equals the fp32 product to the fp32 rounding
// of w itself.  Output [3, E, H] (part-major) for the tensor-core GEMM.
__global__ void __launch_bounds__(256)
    router_split_kernel(const float4* __restrict__ wr, int n4, uint2* __restrict__ parts) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 w = __ldg(wr + i);
  const float v[4] = {w.x, w.y, w.z, w.w};
  uint32_t hi[2], mid[2], lo[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float h2[2], m2[2], l2[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float x = v[2 * j + q];
      const float h = __bfloat162float(__float2bfloat16_rn(x));
      const float r1 = x - h;
      const float m = __bfloat162float(__float2bfloat16_rn(r1));
      const float r2 = r1 - m;
      h2[q] = h;
      m2[q] = m;
      l2[q] = r2;
    }
    hi[j] = pack_bf16x2(h2[0], h2[1]);
    mid[j] = pack_bf16x2(m2[0], m2[1]);
    lo[j] = pack_bf16x2(l2[0], l2[1]);
  }
  parts[i] = make_uint2(hi[0], hi[1]);
  parts[n4 + i] = make_uint2(mid[0], mid[1]);
  parts[2 * n4 + i] = make_uint2(lo[0], lo[1]);
}

// (value, id) argmax across the warp: larger value wins, equal values go to
// the smaller id.  Returns the winner in every lane.
template <typename V>
__device__ __forceinline__ void warp_argmax(V& v, int& id) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const V ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oid = __shfl_xor_sync(0xffffffffu, id, off);
    if (ov > v || (ov == v && oid < id)) {
      v = ov;
      id = oid;
    }
  }
}

constexpr int kTopkWarps = 8;

// Per-warp dynamic shared memory: v64[E] (fp64), s[E], b[E], lv[E] (fp32),
// lst[E], res[MOE_MAX_TOP_K] (int32); rounded to 16 bytes so every warp's
// fp64 array stays aligned.
__host__ __device__ inline size_t topk_smem_per_warp(int E) {
  return (static_cast<size_t>(E) * (8 + 4 + 4 + 4 + 4) + MOE_MAX_TOP_K * 4 + 15) / 16 * 16;
}

// fp64 biased score of expert e for one token: exact bf16 x fp32 products,
// fp64 sum split over the warp's lanes.  Two experts per pass.
__device__ __forceinline__ void exact_biased_pair(const __nv_bfloat16* __restrict__ xr,
                                                  const float* __restrict__ wr, const float* __restrict__ bias,
                                                  int H, int lane, int e0, int e1, double& b0, double& b1) {
  const float* w0r = wr + static_cast<size_t>(e0) * H;
  const float* w1r = wr + static_cast<size_t>(e1) * H;
  double a0 = 0.0, a1 = 0.0;
#pragma unroll 4
  for (int h = lane * 8; h < H; h += 256) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + h));
    const float4 p0 = __ldg(reinterpret_cast<const float4*>(w0r + h));
    const float4 p1 = __ldg(reinterpret_cast<const float4*>(w0r + h + 4));
    const float4 q0 = __ldg(reinterpret_cast<const float4*>(w1r + h));
    const float4 q1 = __ldg(reinterpret_cast<const float4*>(w1r + h + 4));
    const double xv8[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                           bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
    const float pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const float qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      a0 = fma(xv8[j], static_cast<double>(pw[j]), a0);
      a1 = fma(xv8[j], static_cast<double>(qw[j]), a1);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a0 += __shfl_xor_sync(0xffffffffu, a0, off);
    a1 += __shfl_xor_sync(0xffffffffu, a1, off);
  }
  b0 = 1.0 / (1.0 + exp(-a0)) + (bias != nullptr ? static_cast<double>(bias[e0]) : 0.0);
  b1 = 1.0 / (1.0 + exp(-a1)) + (bias != nullptr ? static_cast<double>(bias[e1]) : 0.0);
}

// Single-expert form of exact_biased_pair (same per-lane summation order).
__device__ __forceinline__ double exact_biased_one(const __nv_bfloat16* __restrict__ xr,
                                                   const float* __restrict__ wr, const float* __restrict__ bias,
                                                   int H, int lane, int e0) {
  const float* w0r = wr + static_cast<size_t>(e0) * H;
  double a0 = 0.0;
#pragma unroll 4
  for (int h = lane * 8; h < H; h += 256) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + h));
    const float4 p0 = __ldg(reinterpret_cast<const float4*>(w0r + h));
    const float4 p1 = __ldg(reinterpret_cast<const float4*>(w0r + h + 4));
    const double xv8[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                           bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
    const float pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) a0 = fma(xv8[j], static_cast<double>(pw[j]), a0);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a0 += __shfl_xor_sync(0xffffffffu, a0, off);
  return 1.0 / (1.0 + exp(-a0)) + (bias != nullptr ? static_cast<double>(bias[e0]) : 0.0);
}

// A warp's scratch for selecting one token's experts (see
// topk_smem_per_warp): fp32 unbiased and biased scores of every expert, the
// experts extracted in order with their biased scores, fp64 scores of
// near-tie clusters, and the k chosen ids.
struct WarpArea {
  double* v64;
  float* s;
  float* b;
  float* lv;
  int* lst;
  int* res;
};

__device__ __forceinline__ WarpArea warp_area(unsigned char* base, int E) {
  WarpArea w;
  w.v64 = reinterpret_cast<double*>(base);
  w.s = reinterpret_cast<float*>(base + static_cast<size_t>(E) * 8);
  w.b = w.s + E;
  w.lv = w.b + E;
  w.lst = reinterpret_cast<int*>(w.lv + E);
  w.res = w.lst + E;
  return w;
}

// Phase 2 (one warp, w.s and w.b filled): extract experts in descending
// order -- the top k+1, and, while the k-th/(k+1)-th boundary is a near-tie,
// every further expert that continues the run of adjacent gaps below tau.
// Returns how many were extracted; res[0..k) = the first k.
//
// Each round is one warp-wide max (redux.sync) of 32-bit keys: the upper 22
// bits of the order-preserving integer image of b (sign, exponent and 13
// mantissa bits) above 10 bits of (1023 - id), so equal prefixes go to the
// lower id.  Two experts whose b share a 22-bit prefix may come out in either
// order.  Out of order, they sit next to each other in the extracted list
// with a negative gap, below tau, so they land in the same near-tie cluster
// and are re-ordered exactly in phase 3; in order, they are where exact fp32
// order puts them.  So the selection is the same as extracting by exact
// fp32 order.
__device__ __forceinline__ uint32_t order_key(float b, int e) {
  const uint32_t u = __float_as_uint(b);
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (o & 0xFFFFFC00u) | (1023u - static_cast<uint32_t>(e));
}

__device__ int warp_extract(const WarpArea& w, int E, int k, float tau, int lane) {
  const int nm = (E + 31) / 32;  // entries per lane: e = lane + 32 m
  uint32_t taken = 0;
  auto lane_best = [&]() {
    uint32_t best = 0;
    for (int m = 0; m < nm; ++m) {
      const int e = lane + 32 * m;
      if (e < E && !((taken >> m) & 1u)) best = max(best, order_key(w.b[e], e));
    }
    return best;
  };
  uint32_t mine = lane_best();
  const int k1 = min(k + 1, E);
  int n = 0;
  while (n < E) {
    const uint32_t top = __reduce_max_sync(0xffffffffu, mine);
    const int id = 1023 - static_cast<int>(top & 1023u);
    const float v = w.b[id];
    if (n >= k1) {  // past k+1: only while the boundary run continues
      const bool boundary_tie = w.lv[k - 1] - w.lv[k] < tau;
      if (!boundary_tie || !(w.lv[n - 1] - v < tau)) break;
    }
    if ((id & 31) == lane) {
      taken |= 1u << (id / 32);
      mine = lane_best();
    }
    if (lane == 0) {
      w.lst[n] = id;
      w.lv[n] = v;
    }
    __syncwarp();
    ++n;
  }
  if (lane < k) w.res[lane] = w.lst[lane];
  __syncwarp();
  return n;
}

// Phase 3 (one warp): re-order by fp64 biased scores every near-tie cluster
// -- a maximal run [a, b] of adjacent gaps below tau with a < k -- ties to
// the lower id.  With have_v64 the fp64 scores of the clustered entries are
// already in w.v64; otherwise this warp computes them.  Order between
// clusters is certain: tau is far above the fp32 error of the logits.
__device__ void warp_rerank(const WarpArea& w, int n, const __nv_bfloat16* __restrict__ xr,
                            const float* __restrict__ wr, const float* __restrict__ bias, int H, int k, float tau,
                            bool have_v64, int lane) {
  int a = 0;
  while (a < k) {
    int b = a;
    while (b + 1 < n && w.lv[b] - w.lv[b + 1] < tau) ++b;
    if (b > a) {
      if (!have_v64) {
        for (int i = a; i <= b; i += 2) {
          const int j = min(i + 1, b);
          double d0, d1;
          exact_biased_pair(xr, wr, bias, H, lane, w.lst[i], w.lst[j], d0, d1);
          if (lane == 0) {
            w.v64[i] = d0;
            w.v64[j] = d1;
          }
        }
      }
      __syncwarp();
      uint32_t ctaken = 0;
      const int slots = min(b, k - 1) - a + 1;
      for (int sidx = 0; sidx < slots; ++sidx) {
        double v = -INFINITY;
        int id = 0x7fffffff;
        for (int i = a + lane, m = 0; i <= b; i += 32, ++m) {
          if (!((ctaken >> m) & 1u)) {
            const double bv = w.v64[i];
            const int e = w.lst[i];
            if (bv > v || (bv == v && e < id)) {
              v = bv;
              id = e;
            }
          }
        }
        warp_argmax(v, id);
        for (int i = a + lane, m = 0; i <= b; i += 32, ++m)
          if (w.lst[i] == id) ctaken |= 1u << m;
        if (lane == 0) w.res[a + sidx] = id;
      }
      __syncwarp();
    }
    a = b + 1;
  }
}

// Phase 4 (one warp): ids and alpha * s of the chosen experts from the
// unbiased fp32 scores, renormalised over the k (in selection order) if asked.
__device__ void warp_emit(const WarpArea& w, int k, float alpha, int renorm, int lane, int32_t* __restrict__ ids_row,
                          float* __restrict__ w_row) {
  float wsum = 0.f;
  for (int r = 0; r < k; ++r) wsum += w.s[w.res[r]];
  if (lane < k) {
    const int id = w.res[lane];
    const float sv = w.s[id];
    ids_row[lane] = id;
    w_row[lane] = renorm ? (sv / wsum) * alpha : sv * alpha;
  }
}

// Few tokens: one token per block of kTopkWarps warps.  All threads sum the
// token's K-slice partial logits (slices in ascending order) into s and b;
// warp 0 extracts; every warp computes fp64 scores of the clustered entries;
// warp 0 re-orders and emits.
__global__ void __launch_bounds__(kTopkWarps * 32)
    router_topk_coop_kernel(const float* __restrict__ part, int KS, const __nv_bfloat16* __restrict__ x,
                            const float* __restrict__ wr, const float* __restrict__ bias, int T, int E, int H, int k,
                            float alpha, int renorm, float tau, int32_t* __restrict__ ids_out,
                            float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_n;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x;
  const WarpArea w = warp_area(smem_raw, E);
  const size_t slice = static_cast<size_t>(T) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float l = 0.f;
    const float* pp = part + static_cast<size_t>(t) * E + e;
    int ks = 0;
    for (; ks + 8 <= KS; ks += 8) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __ldg(pp + (ks + j) * slice);
#pragma unroll
      for (int j = 0; j < 8; ++j) l += v[j];
    }
    for (; ks < KS; ++ks) l += __ldg(pp + ks * slice);
    const float sv = 1.f / (1.f + expf(-l));
    w.s[e] = sv;
    w.b[e] = sv + (bias != nullptr ? bias[e] : 0.f);
  }
  __syncthreads();
  if (warp == 0) {
    const int n = warp_extract(w, E, k, tau, lane);
    if (lane == 0) s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
  for (int i = warp; i < n; i += kTopkWarps) {
    // entry i needs an fp64 score if its cluster has two entries or more
    int a = 0, b = 0;
    while (true) {
      b = a;
      while (b + 1 < n && w.lv[b] - w.lv[b + 1] < tau) ++b;
      if (i <= b || b + 1 >= k) break;
      a = b + 1;
    }
    if (a < k && i >= a && i <= b && b > a) {
      const double d = exact_biased_one(xr, wr, bias, H, lane, w.lst[i]);
      if (lane == 0) w.v64[i] = d;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  warp_rerank(w, n, xr, wr, bias, H, k, tau, true, lane);
  warp_emit(w, k, alpha, renorm, lane, ids_out + static_cast<size_t>(t) * k, w_out + static_cast<size_t>(t) * k);
}

// Many tokens: a block takes `tb` consecutive tokens.
//  1. All 256 threads sum the block's K-slice partial logits -- contiguous
//     rows, 16-byte loads, slices in ascending order -- and write every
//     token's s = sigmoid(l) and b = s + bias rows to shared memory.
//  2. Each warp takes one token of the block and runs the same extraction,
//     fp64 re-order of near-tie clusters and emission as the few-token
//     kernel, reading that token's rows in place.  With many warps per SM,
//     each on its own token, the latency of the extraction rounds and of the
//     occasional fp64 dot products overlaps across tokens.
constexpr int kRowsThreads = 256;
constexpr int kRowsWarps = kRowsThreads / 32;

// A warp's own scratch in the row kernel: v64[E] (fp64), lv[E], lst[E],
// res[MOE_MAX_TOP_K]; 16-byte multiple.
__host__ __device__ inline size_t rows_scratch_per_warp(int E) {
  return (static_cast<size_t>(E) * (8 + 4 + 4) + MOE_MAX_TOP_K * 4 + 15) / 16 * 16;
}

// dynamic smem: kRowsWarps scratch areas | s rows [tb][E] | b rows [tb][E]
__global__ void __launch_bounds__(kRowsThreads)
    router_topk_rows_kernel(const float* __restrict__ part, int KS, const __nv_bfloat16* __restrict__ x,
                            const float* __restrict__ wr, const float* __restrict__ bias, int T, int E, int H, int k,
                            float alpha, int renorm, float tau, int tb, int32_t* __restrict__ ids_out,
                            float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const size_t pw = rows_scratch_per_warp(E);
  float* s_rows = reinterpret_cast<float*>(smem_raw + kRowsWarps * pw);
  float* b_rows = s_rows + static_cast<size_t>(tb) * E;
  const int t0 = blockIdx.x * tb;
  const int nt = min(tb, T - t0);

  // 1. partial sums of the block's nt x E logits (one contiguous range per slice)
  const size_t slice = static_cast<size_t>(T) * E;
  const float* base = part + static_cast<size_t>(t0) * E;
  const int n = nt * E;
  auto put = [&](int i, float l) {
    const int e = i % E;
    const float sv = 1.f / (1.f + expf(-l));
    s_rows[i] = sv;
    b_rows[i] = sv + (bias != nullptr ? __ldg(bias + e) : 0.f);
  };
  if ((E & 3) == 0) {
    const int n4 = n / 4;
    for (int i0 = threadIdx.x; i0 < n4; i0 += 4 * kRowsThreads) {
      float4 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
      for (int ks = 0; ks < KS; ++ks) {
        const float4* src = reinterpret_cast<const float4*>(base + ks * slice);
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = (i0 + u * kRowsThreads < n4) ? __ldg(src + i0 + u * kRowsThreads) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc[u].x += v[u].x;
          acc[u].y += v[u].y;
          acc[u].z += v[u].z;
          acc[u].w += v[u].w;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i4 = i0 + u * kRowsThreads;
        if (i4 < n4) {
          put(4 * i4, acc[u].x);
          put(4 * i4 + 1, acc[u].y);
          put(4 * i4 + 2, acc[u].z);
          put(4 * i4 + 3, acc[u].w);
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < n; i += kRowsThreads) {
      float l = 0.f;
      for (int ks = 0; ks < KS; ++ks) l += __ldg(base + ks * slice + i);
      put(i, l);
    }
  }
  __syncthreads();

  // 2. one warp per token
  unsigned char* mine = smem_raw + warp * pw;
  WarpArea w;
  w.v64 = reinterpret_cast<double*>(mine);
  w.lv = reinterpret_cast<float*>(mine + static_cast<size_t>(E) * 8);
  w.lst = reinterpret_cast<int*>(w.lv + E);
  w.res = w.lst + E;
  for (int r = warp; r < nt; r += kRowsWarps) {
    const int t = t0 + r;
    w.s = s_rows + static_cast<size_t>(r) * E;
    w.b = b_rows + static_cast<size_t>(r) * E;
    const int nn = warp_extract(w, E, k, tau, lane);
    warp_rerank(w, nn, x + static_cast<size_t>(t) * H, wr, bias, H, k, tau, false, lane);
    warp_emit(w, k, alpha, renorm, lane, ids_out + static_cast<size_t>(t) * k, w_out + static_cast<size_t>(t) * k);
    __syncwarp();
  }
}

// Tokens per block of the row kernel: one per warp, so that every token's
// latency-bound selection runs on a warp of its own.
int rows_tokens_per_block(int) { return kRowsWarps; }

size_t rows_smem(int E, int tb) {
  return kRowsWarps * rows_scratch_per_warp(E) + 2 * static_cast<size_t>(tb) * E * sizeof(float);
}

}  // namespace

RouterPlan router_plan(int T, int E, int H, int num_sms) {
  RouterPlan p;
  const int n_mma = router_mma_n(E);
  const int tiles0 = ((T + 127) / 128) * ((E + n_mma - 1) / n_mma);
  const int steps = splitk_steps(H, 3, n_mma, T);
  int ks = std::max(1, num_sms / tiles0);        // at most one wave of CTAs
  ks = std::min(ks, std::max(1, steps / 4));     // at least 4 K steps per split
  ks = std::min(ks, std::max(1, kRouterPartialRows / std::max(T, 1)));
  ks = std::min(ks, 32);  // the top-k kernel adds every slice: keep its reads short
  p.ks = router_actual_splits(T, E, H, std::max(ks, 1));
  return p;
}

size_t router_partial_floats(int Tmax, int E) {
  return static_cast<size_t>(E) * static_cast<size_t>(std::max(Tmax + 64, kRouterPartialRows));
}

size_t router_topk_smem(int E) { return topk_smem_per_warp(E); }

cudaError_t launch_router(const moe_config& cfg, const moe_weights& w, const void* x, int T, int32_t* ids,
                          float* wts, float* part, void* w_split, int32_t* err, int num_sms, cudaStream_t stream) {
  const int E = cfg.num_experts, H = cfg.hidden, k = cfg.top_k;
  const RouterPlan p = router_plan(T, E, H, num_sms);
  const int n4 = E * H / 4;
  cudaError_t err_c = launch_kernel(router_split_kernel, dim3((n4 + 255) / 256), dim3(256), 0, stream,
                                            reinterpret_cast<const float4*>(w.router_w), n4,
                                            static_cast<uint2*>(w_split));
  if (err_c != cudaSuccess) return err_c;
  err_c = launch_router_gemm(x, T, H, w_split, E, p.ks, part, err, num_sms, stream);
  if (err_c != cudaSuccess) return err_c;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (T < num_sms * kTopkWarps) {
    // few tokens: one token per block, so 256 threads read its partial sums
    err_c = ensure_smem_attr(reinterpret_cast<const void*>(router_topk_coop_kernel),
                             static_cast<int>(router_topk_smem(MOE_MAX_EXPERTS)));
    if (err_c != cudaSuccess) return err_c;
    return launch_kernel(router_topk_coop_kernel, dim3(T), dim3(kTopkWarps * 32), router_topk_smem(E),
                                 stream, static_cast<const float*>(part), p.ks, xb, w.router_w, w.correction_bias, T,
                                 E, H, k, cfg.routed_scaling_factor, cfg.renormalize, kRouterTieTau, ids, wts);
  }
  const int tb = rows_tokens_per_block(E);
  err_c = ensure_smem_attr(reinterpret_cast<const void*>(router_topk_rows_kernel),
                           static_cast<int>(rows_smem(MOE_MAX_EXPERTS, rows_tokens_per_block(MOE_MAX_EXPERTS))));
  if (err_c != cudaSuccess) return err_c;
  return launch_kernel(router_topk_rows_kernel, dim3(static_cast<unsigned>((T + tb - 1) / tb)),
                               dim3(kRowsThreads), rows_smem(E, tb), stream, static_cast<const float*>(part), p.ks,
                               xb, w.router_w, w.correction_bias, T, E, H, k, cfg.routed_scaling_factor,
                               cfg.renormalize, kRouterTieTau, tb, ids, wts);
}

}  // namespace moe
