// Router: the fp32 logits GEMM runs on the tensor cores (splitk_gemm.cu, three
// passes over K) on an exact bf16 split of the fp32 weight; here are the split
// and the warp-per-token sigmoid + biased top-k with an fp64 re-rank of
// near-ties.
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

// One warp per token (with one token per block, every warp of the block
// shares that token's fp64 scores).
//  1. s = sigmoid(sum of the partial logits), b = s + bias (fp32).
//  2. Extract experts in (b desc, id asc) order: the top k+1, and, while the
//     k-th/(k+1)-th boundary is a near-tie, every further expert that
//     continues the run of adjacent gaps below tau.
//  3. Any run ("cluster") of adjacent gaps below tau that reaches into the
//     top k is re-ordered by fp64 biased scores (ties to the lower id); order
//     between clusters is certain because tau is far above the fp32 error.
//  4. Emit ids and alpha * s (renormalised over the k if asked).
__global__ void __launch_bounds__(kTopkWarps * 32)
    router_topk_kernel(const float* __restrict__ part, int KS, const __nv_bfloat16* __restrict__ x,
                       const float* __restrict__ wr, const float* __restrict__ bias, int T, int E, int H,
                       int k, float alpha, int renorm, float tau, int tpb, int32_t* __restrict__ ids_out,
                       float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t0 = blockIdx.x * tpb;
  const size_t pw = topk_smem_per_warp(E);

  // 1. all threads of the block: sum the split-H partial logits of the
  //    block's tpb tokens, s = sigmoid, b = s + bias, into the token's warp area
  for (int idx = threadIdx.x; idx < tpb * E; idx += blockDim.x) {
    const int w = idx / E, e = idx - w * E;
    const int tt = t0 + w;
    if (tt < T) {
      // slices are added in ascending order, loaded 8 at a time
      float l = 0.f;
      const float* pp = part + static_cast<size_t>(tt) * E + e;
      const size_t slice = static_cast<size_t>(T) * E;
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
      float* sw = reinterpret_cast<float*>(smem_raw + pw * w + static_cast<size_t>(E) * 8);
      sw[e] = sv;
      sw[E + e] = sv + (bias != nullptr ? bias[e] : 0.f);
    }
  }
  __syncthreads();
  const bool coop = tpb == 1;  // block-uniform
  const int t = t0 + (coop ? 0 : warp);
  if (coop ? t >= T : (warp >= tpb || t >= T)) return;
  const bool owner = !coop || warp == 0;

  unsigned char* base = smem_raw + pw * (coop ? 0 : warp);
  double* v64 = reinterpret_cast<double*>(base);
  float* s_sm = reinterpret_cast<float*>(base + static_cast<size_t>(E) * 8);
  float* b_sm = s_sm + E;
  float* lv = b_sm + E;
  int* lst = reinterpret_cast<int*>(lv + E);
  int* res = lst + E;
  const int nm = (E + 31) / 32;  // entries per lane: e = lane + 32 m

  // 2. ordered extraction (the owner warp)
  __shared__ int s_n;
  int n = 0;
  if (owner) {
  uint32_t taken = 0;
  const int k1 = min(k + 1, E);
  while (n < E) {
    float v = -INFINITY;
    int id = 0x7fffffff;
    for (int m = 0; m < nm; ++m) {
      const int e = lane + 32 * m;
      if (e < E && !((taken >> m) & 1u)) {
        const float bv = b_sm[e];
        if (bv > v || (bv == v && e < id)) {
          v = bv;
          id = e;
        }
      }
    }
    warp_argmax(v, id);
    if (n >= k1) {  // past k+1: only while the boundary run continues
      const bool boundary_tie = lv[k - 1] - lv[k] < tau;
      if (!boundary_tie || !(lv[n - 1] - v < tau)) break;
    }
    if ((id & 31) == lane) taken |= 1u << (id / 32);
    if (lane == 0) {
      lst[n] = id;
      lv[n] = v;
    }
    __syncwarp();
    ++n;
  }
  if (lane < k) res[lane] = lst[lane];
  if (coop && lane == 0) s_n = n;
  __syncwarp();
  }

  // 3. fp64 re-order of the near-tie clusters that reach into the top k.
  //    Cluster [a, b]: a maximal run of adjacent gaps below tau starting at
  //    a < k.  With one token per block all warps first compute the fp64
  //    scores of every clustered entry, then the owner orders them.
  const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
  if (coop) {
    __syncthreads();
    n = s_n;
    for (int i = warp; i < n; i += kTopkWarps) {
      // entry i needs an fp64 score if its cluster has two entries or more
      int a = 0, b = 0;
      while (true) {
        b = a;
        while (b + 1 < n && lv[b] - lv[b + 1] < tau) ++b;
        if (i <= b || b + 1 >= k) break;
        a = b + 1;
      }
      if (a < k && i >= a && i <= b && b > a) {
        const double d = exact_biased_one(xr, wr, bias, H, lane, lst[i]);
        if (lane == 0) v64[i] = d;
      }
    }
    __syncthreads();
    if (!owner) return;
  }
  int a = 0;
  while (a < k) {
    int b = a;
    while (b + 1 < n && lv[b] - lv[b + 1] < tau) ++b;
    if (b > a) {
      if (!coop) {
        for (int i = a; i <= b; i += 2) {
          const int j = min(i + 1, b);
          double d0, d1;
          exact_biased_pair(xr, wr, bias, H, lane, lst[i], lst[j], d0, d1);
          if (lane == 0) {
            v64[i] = d0;
            v64[j] = d1;
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
            const double bv = v64[i];
            const int e = lst[i];
            if (bv > v || (bv == v && e < id)) {
              v = bv;
              id = e;
            }
          }
        }
        warp_argmax(v, id);
        for (int i = a + lane, m = 0; i <= b; i += 32, ++m)
          if (lst[i] == id) ctaken |= 1u << m;
        if (lane == 0) res[a + sidx] = id;
      }
      __syncwarp();
    }
    a = b + 1;
  }

  // 4. emitted weights from the unbiased fp32 scores
  float wsum = 0.f;
  for (int r = 0; r < k; ++r) wsum += s_sm[res[r]];
  if (lane < k) {
    const int id = res[lane];
    const float sv = s_sm[id];
    ids_out[static_cast<size_t>(t) * k + lane] = id;
    w_out[static_cast<size_t>(t) * k + lane] = renorm ? (sv / wsum) * alpha : sv * alpha;
  }
}

}  // namespace

RouterPlan router_plan(int T, int E, int H) {
  RouterPlan p;
  const int n_mma = router_mma_n(E);
  const int tiles0 = ((T + 127) / 128) * ((E + n_mma - 1) / n_mma);
  const int total_kb = 3 * ((H + 63) / 64);
  int ks = (148 + tiles0 - 1) / tiles0;          // about one wave of CTAs
  ks = std::min(ks, std::max(1, total_kb / 4));  // at least 4 k-blocks per split
  ks = std::min(ks, std::max(1, kRouterPartialRows / std::max(T, 1)));
  ks = std::min(ks, 32);  // the top-k kernel adds every slice: keep its reads short
  p.ks = router_actual_splits(H, std::max(ks, 1));
  return p;
}

size_t router_partial_floats(int Tmax, int E) {
  return static_cast<size_t>(E) * static_cast<size_t>(std::max(Tmax + 64, kRouterPartialRows));
}

size_t router_topk_smem(int E) { return static_cast<size_t>(kTopkWarps) * topk_smem_per_warp(E); }

cudaError_t launch_router(const moe_config& cfg, const moe_weights& w, const void* x, int T, int32_t* ids,
                          float* wts, float* part, void* w_split, int32_t* err, int num_sms, cudaStream_t stream) {
  const int E = cfg.num_experts, H = cfg.hidden, k = cfg.top_k;
  const RouterPlan p = router_plan(T, E, H);
  const int n4 = E * H / 4;
  router_split_kernel<<<(n4 + 255) / 256, 256, 0, stream>>>(reinterpret_cast<const float4*>(w.router_w), n4,
                                                             static_cast<uint2*>(w_split));
  cudaError_t err_c = cudaGetLastError();
  if (err_c != cudaSuccess) return err_c;
  err_c = launch_router_gemm(x, T, H, w_split, E, p.ks, part, err, num_sms, stream);
  if (err_c != cudaSuccess) return err_c;
  const size_t smem = router_topk_smem(E);
  err_c = ensure_smem_attr(reinterpret_cast<const void*>(router_topk_kernel),
                           static_cast<int>(router_topk_smem(MOE_MAX_EXPERTS)));
  if (err_c != cudaSuccess) return err_c;
  // few tokens: one token per block so the partial sums are read by 256
  // threads at once; many tokens: one token per warp
  const int tpb = T >= 148 * kTopkWarps ? kTopkWarps : 1;
  router_topk_kernel<<<(T + tpb - 1) / tpb, kTopkWarps * 32, smem, stream>>>(
      part, p.ks, static_cast<const __nv_bfloat16*>(x), w.router_w, w.correction_bias, T, E, H, k,
      cfg.routed_scaling_factor, cfg.renormalize, kRouterTieTau, tpb, ids, wts);
  return cudaGetLastError();
}

}  // namespace moe
