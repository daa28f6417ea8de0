// Router: fp32 logits GEMM (SIMT, split over H for small token counts) and a
// warp-per-token sigmoid + biased top-k with an fp64 re-rank of near-ties.
//
// "Module glm5next_mlp" §Numerics: sigmoid score; the correction bias steers
// selection only; the emitted weight is the unbiased score times
// routed_scaling_factor.  "bridge.models.beam.modeling_beam"
// beam_router_gating_linear: logits = inp @ weight.T with fp32 operands.
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterKC = 32;

// logits_part[ks, t, e] = sum_{h in split ks} x[t, h] * wr[e, h]   (fp32)
// Block tile: BT tokens x 64 experts; 16 x 16 threads, each BT/16 x 4 outputs.
template <int BT>
__global__ void __launch_bounds__(kRouterThreads)
    router_logits_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                         float* __restrict__ part, int T, int E, int H, int k_per_split) {
  constexpr int BE = 64;
  constexpr int TPT = BT / 16;
  __shared__ __align__(16) float xs[kRouterKC][BT];
  __shared__ __align__(16) float wsm[kRouterKC][BE];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int e0 = blockIdx.x * BE;
  const int t0 = blockIdx.y * BT;
  const int ks = blockIdx.z;
  const int hb = ks * k_per_split;
  const int he = min(H, hb + k_per_split);

  float acc[TPT][4];
#pragma unroll
  for (int i = 0; i < TPT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int h0 = hb; h0 < he; h0 += kRouterKC) {
    // x tile: BT tokens x 32 k, one 16-byte (8 x bf16) load per thread
    if (tid < BT * (kRouterKC / 8)) {
      const int tt = tid / (kRouterKC / 8);
      const int kk = (tid % (kRouterKC / 8)) * 8;
      const int t = t0 + tt, h = h0 + kk;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T && h < he) v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + h));
      xs[kk + 0][tt] = bf16lo(v.x);
      xs[kk + 1][tt] = bf16hi(v.x);
      xs[kk + 2][tt] = bf16lo(v.y);
      xs[kk + 3][tt] = bf16hi(v.y);
      xs[kk + 4][tt] = bf16lo(v.z);
      xs[kk + 5][tt] = bf16hi(v.z);
      xs[kk + 6][tt] = bf16lo(v.w);
      xs[kk + 7][tt] = bf16hi(v.w);
    }
    // router weight tile: 64 experts x 32 k fp32, two float4 per thread
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int idx = tid + r * kRouterThreads;
      const int ee = idx / (kRouterKC / 4);
      const int kk = (idx % (kRouterKC / 4)) * 4;
      const int e = e0 + ee, h = h0 + kk;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E && h < he) v = __ldg(reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H + h));
      wsm[kk + 0][ee] = v.x;
      wsm[kk + 1][ee] = v.y;
      wsm[kk + 2][ee] = v.z;
      wsm[kk + 3][ee] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterKC; ++kk) {
      float a[TPT];
#pragma unroll
      for (int i = 0; i < TPT; ++i) a[i] = xs[kk][ty * TPT + i];
      const float4 b = *reinterpret_cast<const float4*>(&wsm[kk][tx * 4]);
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        acc[i][0] = fmaf(a[i], b.x, acc[i][0]);
        acc[i][1] = fmaf(a[i], b.y, acc[i][1]);
        acc[i][2] = fmaf(a[i], b.z, acc[i][2]);
        acc[i][3] = fmaf(a[i], b.w, acc[i][3]);
      }
    }
    __syncthreads();
  }
  float* out = part + static_cast<size_t>(ks) * T * E;
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = t0 + ty * TPT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) out[static_cast<size_t>(t) * E + e] = acc[i][j];
    }
  }
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

// Per-warp dynamic shared memory: cand_b[E] (fp64), s[E], b[E] (fp32),
// cand[E] (int32); rounded to 16 bytes so every warp's fp64 array is aligned.
__host__ __device__ inline size_t topk_smem_per_warp(int E) {
  return (static_cast<size_t>(E) * (8 + 4 + 4 + 4) + 15) / 16 * 16;
}

// One warp per token.  Dynamic smem per warp: s[E], b[E] (fp32),
// cand[E] (int), cand_b[E] (fp64).
__global__ void __launch_bounds__(kTopkWarps * 32)
    router_topk_kernel(const float* __restrict__ part, int KS, const __nv_bfloat16* __restrict__ x,
                       const float* __restrict__ wr, const float* __restrict__ bias, int T, int E, int H,
                       int k, float alpha, int renorm, float tau, int32_t* __restrict__ ids_out,
                       float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;

  const size_t per_warp = topk_smem_per_warp(E);
  unsigned char* base = smem_raw + per_warp * warp;
  double* cand_b = reinterpret_cast<double*>(base);
  float* s_sm = reinterpret_cast<float*>(base + static_cast<size_t>(E) * 8);
  float* b_sm = s_sm + E;
  int* cand = reinterpret_cast<int*>(b_sm + E);

  const int nm = (E + 31) / 32;  // entries per lane: e = lane + 32 m
  for (int m = 0; m < nm; ++m) {
    const int e = lane + 32 * m;
    if (e < E) {
      float l = 0.f;
      for (int ks = 0; ks < KS; ++ks) l += part[(static_cast<size_t>(ks) * T + t) * E + e];
      const float s = 1.f / (1.f + expf(-l));
      s_sm[e] = s;
      b_sm[e] = s + (bias != nullptr ? bias[e] : 0.f);
    }
  }
  __syncwarp();

  // top-(k+1) in fp32 (the extra one measures the selection boundary gap)
  const int k1 = min(k + 1, E);
  int sel_e[MOE_MAX_TOP_K + 1];
  float sel_b[MOE_MAX_TOP_K + 1];
  uint32_t taken = 0;
#pragma unroll
  for (int r = 0; r < MOE_MAX_TOP_K + 1; ++r) {
    if (r < k1) {
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
      if ((id & 31) == lane) taken |= 1u << (id / 32);
      sel_e[r] = id;
      sel_b[r] = v;
    }
  }
  float min_gap = INFINITY;
#pragma unroll
  for (int r = 0; r < MOE_MAX_TOP_K; ++r)
    if (r + 1 < k1) min_gap = fminf(min_gap, sel_b[r] - sel_b[r + 1]);

  if (min_gap < tau) {
    // Near-tie: every expert whose fp32 biased score is within tau of the
    // k-th is re-scored from an fp64 logit (exact bf16 x fp32 products, fp64
    // sum) and the k largest are taken again, ties to the lower id.
    const float thr = sel_b[k - 1] - tau;
    int n_c = 0;
    for (int m = 0; m < nm; ++m) {
      const int e = lane + 32 * m;
      const bool p = e < E && b_sm[e] >= thr;
      const uint32_t bal = __ballot_sync(0xffffffffu, p);
      if (p) cand[n_c + __popc(bal & ((1u << lane) - 1u))] = e;
      n_c += __popc(bal);
    }
    __syncwarp();
    const __nv_bfloat16* xr = x + static_cast<size_t>(t) * H;
    for (int c = 0; c < n_c; ++c) {
      const int e = cand[c];
      const float* wrow = wr + static_cast<size_t>(e) * H;
      double acc = 0.0;
      for (int h = lane * 8; h < H; h += 256) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + h));
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wrow + h));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wrow + h + 4));
        acc = fma(static_cast<double>(bf16lo(xv.x)), static_cast<double>(w0.x), acc);
        acc = fma(static_cast<double>(bf16hi(xv.x)), static_cast<double>(w0.y), acc);
        acc = fma(static_cast<double>(bf16lo(xv.y)), static_cast<double>(w0.z), acc);
        acc = fma(static_cast<double>(bf16hi(xv.y)), static_cast<double>(w0.w), acc);
        acc = fma(static_cast<double>(bf16lo(xv.z)), static_cast<double>(w1.x), acc);
        acc = fma(static_cast<double>(bf16hi(xv.z)), static_cast<double>(w1.y), acc);
        acc = fma(static_cast<double>(bf16lo(xv.w)), static_cast<double>(w1.z), acc);
        acc = fma(static_cast<double>(bf16hi(xv.w)), static_cast<double>(w1.w), acc);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) {
        const double s = 1.0 / (1.0 + exp(-acc));
        cand_b[c] = s + (bias != nullptr ? static_cast<double>(bias[e]) : 0.0);
      }
    }
    __syncwarp();
    const int ncm = (n_c + 31) / 32;
    uint32_t ctaken = 0;
#pragma unroll
    for (int r = 0; r < MOE_MAX_TOP_K; ++r) {
      if (r < k) {
        double v = -INFINITY;
        int id = 0x7fffffff, slot = -1;
        for (int m = 0; m < ncm; ++m) {
          const int c = lane + 32 * m;
          if (c < n_c && !((ctaken >> m) & 1u)) {
            const double bv = cand_b[c];
            const int e = cand[c];
            if (bv > v || (bv == v && e < id)) {
              v = bv;
              id = e;
              slot = c;
            }
          }
        }
        int owner_slot = slot;
        warp_argmax(v, id);
        // the lane whose candidate won marks it taken
        if (owner_slot >= 0 && cand[owner_slot] == id) ctaken |= 1u << (owner_slot / 32);
        sel_e[r] = id;
      }
    }
  }

  // emitted weights from the unbiased fp32 scores
  float wsum = 0.f;
  float wj[MOE_MAX_TOP_K];
#pragma unroll
  for (int r = 0; r < MOE_MAX_TOP_K; ++r) {
    if (r < k) {
      wj[r] = s_sm[sel_e[r]];
      wsum += wj[r];
    }
  }
#pragma unroll
  for (int r = 0; r < MOE_MAX_TOP_K; ++r) {
    if (r < k && lane == r) {
      const float v = renorm ? (wj[r] / wsum) * alpha : wj[r] * alpha;
      ids_out[static_cast<size_t>(t) * k + r] = sel_e[r];
      w_out[static_cast<size_t>(t) * k + r] = v;
    }
  }
}

}  // namespace

RouterPlan router_plan(int T, int E, int H) {
  RouterPlan p;
  const int eb = (E + 63) / 64;
  p.bt = 64;
  if (eb * ((T + 63) / 64) < 2 * 148) p.bt = 32;
  if (p.bt == 32 && T < 64) p.bt = 16;
  const int tpad = (T + p.bt - 1) / p.bt * p.bt;
  const int blocks0 = ((E + 63) / 64) * (tpad / p.bt);
  int ks = 1;
  const int target = 2 * 148;
  if (blocks0 < target) ks = (target + blocks0 - 1) / blocks0;
  const int max_by_h = std::max(1, H / 256);
  ks = std::min(ks, max_by_h);
  ks = std::min(ks, std::max(1, kRouterPartialRows / std::max(tpad, 1)));
  ks = std::max(ks, 1);
  int kps = (H + ks - 1) / ks;
  kps = (kps + kRouterKC - 1) / kRouterKC * kRouterKC;
  ks = (H + kps - 1) / kps;
  p.ks = ks;
  p.k_per_split = kps;
  return p;
}

size_t router_partial_floats(int Tmax, int E) {
  return static_cast<size_t>(E) * static_cast<size_t>(std::max(Tmax + 64, kRouterPartialRows));
}

size_t router_topk_smem(int E) { return static_cast<size_t>(kTopkWarps) * topk_smem_per_warp(E); }

cudaError_t launch_router(const moe_config& cfg, const moe_weights& w, const void* x, int T, int32_t* ids,
                          float* wts, float* part, cudaStream_t stream) {
  const int E = cfg.num_experts, H = cfg.hidden, k = cfg.top_k;
  const RouterPlan p = router_plan(T, E, H);
  const dim3 grid((E + 63) / 64, (T + p.bt - 1) / p.bt, p.ks);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  switch (p.bt) {
    case 64:
      router_logits_kernel<64><<<grid, kRouterThreads, 0, stream>>>(xb, w.router_w, part, T, E, H, p.k_per_split);
      break;
    case 32:
      router_logits_kernel<32><<<grid, kRouterThreads, 0, stream>>>(xb, w.router_w, part, T, E, H, p.k_per_split);
      break;
    default:
      router_logits_kernel<16><<<grid, kRouterThreads, 0, stream>>>(xb, w.router_w, part, T, E, H, p.k_per_split);
      break;
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = router_topk_smem(E);
  err = ensure_smem_attr(reinterpret_cast<const void*>(router_topk_kernel),
                         static_cast<int>(router_topk_smem(MOE_MAX_EXPERTS)));
  if (err != cudaSuccess) return err;
  router_topk_kernel<<<(T + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, smem, stream>>>(
      part, p.ks, xb, w.router_w, w.correction_bias, T, E, H, k, cfg.routed_scaling_factor, cfg.renormalize,
      kRouterTieTau, ids, wts);
  return cudaGetLastError();
}

}  // namespace moe
