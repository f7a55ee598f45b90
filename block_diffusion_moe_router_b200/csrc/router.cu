// router.cu -- the MoE router: the router's own (1+gamma) RMSNorm of the raw
// residual, fp32 logits against router_w (+ bias), softmax, top-k with the
// lower expert index winning ties, renormalised weights.
//
// Source: Quant-Tuner pull request "Add DiffusionGemma (Gemma-4 MoE
// block-diffusion) support", "Answers to the motivating questions" (the
// router reads the raw residual through its own internal norm; Gemma's
// (1+gamma) RMSNorm convention); top-8 of 128 from its Summary and from the
// "kingjones777/DiffusionGemma-26B-A4B-it-ROCmFP4-GGUF" card header.
//
// Work split: a CTA owns kRouterTT tokens x kRouterTE experts; the CTAs that
// share a token tile form one thread-block cluster along the expert groups.
// Each of the 8 warps reduces one eighth of d for all (token, expert) pairs
// of the tile (lane = expert); partial sums are added in warp order (fixed,
// deterministic).  The cluster's rank-0 CTA then reads every group's logits
// through distributed shared memory and one warp per token runs the top-k
// with warp shuffles.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;  // = K-slices of d
static_assert(kWarps == kRouterTT, "one warp per token while loading x");

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(kThreads) router_kernel(RouterArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int d = a.d;
  const int E = a.E;
  float* xs = sm;                              // [TT][d]  x rows in fp32
  float* red = xs + kRouterTT * d;             // [8][TT][32] partial sums
  float* zloc = red + kWarps * kRouterTT * 32; // [TT][32] this CTA's logits
  float* zall = zloc + kRouterTT * 32;         // [TT][E]   all logits (rank 0)
  float* inv_rms = zall + kRouterTT * kMaxE;   // [TT]

  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRouterTT;
  const int eg = blockIdx.y;  // expert group == rank in the cluster

  // ---- x rows -> fp32 in smem, and 1/rms per token (warp = token)
  {
    const int t = t0 + warp;
    float* row = xs + warp * d;
    float ss = 0.f;
    if (t < a.T) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * d);
      for (int i = lane; i < d / 8; i += 32) {
        uint4 pk = __ldg(src + i);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&pk);
        float4 lo, hi;
        float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
        float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
        lo = make_float4(f0.x, f0.y, f1.x, f1.y);
        hi = make_float4(f2.x, f2.y, f3.x, f3.y);
        reinterpret_cast<float4*>(row)[2 * i] = lo;
        reinterpret_cast<float4*>(row)[2 * i + 1] = hi;
        ss = fmaf(lo.x, lo.x, ss); ss = fmaf(lo.y, lo.y, ss);
        ss = fmaf(lo.z, lo.z, ss); ss = fmaf(lo.w, lo.w, ss);
        ss = fmaf(hi.x, hi.x, ss); ss = fmaf(hi.y, hi.y, ss);
        ss = fmaf(hi.z, hi.z, ss); ss = fmaf(hi.w, hi.w, ss);
      }
    } else {
      for (int i = lane; i < d; i += 32) row[i] = 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) inv_rms[warp] = 1.0f / sqrtf(ss / (float)d + a.eps);
  }
  __syncthreads();

  // ---- partial logits: warp = K-slice, lane = expert, all TT tokens
  const int e = eg * kRouterTE + lane;
  const int ks = d / kWarps;  // multiple of 16 (d % 128 == 0)
  const int k0 = warp * ks;
  float acc[kRouterTT];
#pragma unroll
  for (int t = 0; t < kRouterTT; ++t) acc[t] = 0.f;
  if (e < E) {
    const float4* wrow = reinterpret_cast<const float4*>(a.router_w + (size_t)e * d + k0);
    const float4* g4 = reinterpret_cast<const float4*>(a.gamma + k0);
#pragma unroll 2
    for (int c = 0; c < ks / 4; ++c) {
      float4 wv = __ldg(wrow + c);
      const float4 gv = __ldg(g4 + c);
      // (1 + gamma) folded into the weight: z = (sum_i w_i (1+g_i) x_i) / rms
      wv.x *= 1.f + gv.x; wv.y *= 1.f + gv.y; wv.z *= 1.f + gv.z; wv.w *= 1.f + gv.w;
#pragma unroll
      for (int t = 0; t < kRouterTT; ++t) {
        const float4 xv = reinterpret_cast<const float4*>(xs + t * d + k0)[c];
        float s = acc[t];
        s = fmaf(wv.x, xv.x, s); s = fmaf(wv.y, xv.y, s);
        s = fmaf(wv.z, xv.z, s); s = fmaf(wv.w, xv.w, s);
        acc[t] = s;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kRouterTT; ++t) red[(warp * kRouterTT + t) * 32 + lane] = acc[t];
  __syncthreads();
  {
    const int t = threadIdx.x >> 5;  // 8 tokens x 32 experts = 256 threads
    const int l = threadIdx.x & 31;
    const int ee = eg * kRouterTE + l;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[(w * kRouterTT + t) * 32 + l];
    float z = -INFINITY;
    if (ee < E) {
      z = s * inv_rms[t];
      if (a.bias) z += __ldg(a.bias + ee);
      if (z != z) z = -INFINITY;  // a NaN logit never wins
    }
    zloc[t * 32 + l] = z;
  }

  // ---- gather all expert groups' logits in the rank-0 CTA
  cluster.sync();
  const int groups = (E + kRouterTE - 1) / kRouterTE;
  if (eg == 0) {
    for (int i = threadIdx.x; i < kRouterTT * E; i += kThreads) {
      const int t = i / E;
      const int ee = i - t * E;
      const float* rz = cluster.map_shared_rank(zloc, ee / kRouterTE);
      zall[t * E + ee] = rz[t * 32 + (ee % kRouterTE)];
    }
  }
  cluster.sync();  // the other CTAs' zloc stays alive until here
  if (eg != 0) return;
  __syncthreads();
  (void)groups;

  // ---- top-k per token: warp = token, lane holds experts lane + 32c
  const int t = t0 + warp;
  if (t >= a.T) return;
  float v[kMaxE / 32];
#pragma unroll
  for (int c = 0; c < kMaxE / 32; ++c) {
    const int ee = lane + 32 * c;
    v[c] = (ee < E) ? zall[warp * E + ee] : -INFINITY;
  }
  uint32_t taken = 0;
  float my_sel = -INFINITY;
  float next_v = -INFINITY;
  const int rounds = (a.k < E) ? a.k + 1 : a.k;
  for (int j = 0; j < rounds; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int c = 0; c < kMaxE / 32; ++c) {
      const int ee = lane + 32 * c;
      if (ee < E && !((taken >> c) & 1u) && better(v[c], ee, bv, bi)) {
        bv = v[c];
        bi = ee;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (j < a.k) {
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (lane == j) my_sel = bv;
      if (lane == 0) a.idx[(size_t)t * a.k + j] = bi;
    } else {
      next_v = bv;
    }
  }
  // w_j = exp(z_j - z_0) / sum_j' exp(z_j' - z_0): the full softmax restricted
  // to the selected set and renormalised.
  const float top = __shfl_sync(0xffffffffu, my_sel, 0);
  const float ex = (lane < a.k) ? expf(my_sel - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < a.k) a.w[(size_t)t * a.k + lane] = ex / sum;
  const float last = __shfl_sync(0xffffffffu, my_sel, a.k - 1);
  if (lane == 0 && a.gap) a.gap[t] = (a.k < E) ? (last - next_v) : INFINITY;
}

}  // namespace

}  // namespace moe

static size_t router_smem_bytes(int d) {
  return sizeof(float) * ((size_t)moe::kRouterTT * d + 8 * moe::kRouterTT * 32 +
                          moe::kRouterTT * 32 + moe::kRouterTT * moe::kMaxE + moe::kRouterTT);
}

cudaError_t moe_launch_router(const moe::RouterArgs& a, cudaStream_t s) {
  const size_t smem = router_smem_bytes(a.d);
  cudaError_t err = cudaFuncSetAttribute(moe::router_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int groups = (a.E + moe::kRouterTE - 1) / moe::kRouterTE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.T + moe::kRouterTT - 1) / moe::kRouterTT, groups, 1);
  cfg.blockDim = dim3(moe::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = groups;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe::router_kernel, a);
}
