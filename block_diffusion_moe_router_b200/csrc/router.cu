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
// Work split: a CTA owns kRouterTT tokens x kRouterTE experts over the whole
// hidden dimension; the CTAs that share a token tile form one thread-block
// cluster along the expert groups.
//   - warp 8 streams the CTA's router_w rows in [32 x 128] fp32 chunks with
//     TMA into a 4-stage ring (no multicast);
//   - warps 0..7 first stage 1+gamma and x * (1+gamma) in fp32 (and each
//     token's sum of squares), issuing every load of a row before using it, then every lane accumulates 8 tokens x 4 experts over its 4
//     columns of each chunk (12 LDS.128 per 128 FFMA);
//   - a fixed shuffle-halving reduction leaves lane l of warp w with the
//     logit of (token l/4, expert 4w + l%4): z = sum / rms + bias;
//   - the cluster's rank-0 CTA gathers every group's logits through
//     distributed shared memory and one warp per token runs the top-k with
//     warp shuffles.
// All reductions run in a fixed order, so the result is deterministic.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kCompWarps = 8;
constexpr int kThreads = (kCompWarps + 1) * 32;
constexpr int kChunk = 128;  // hidden columns per stage
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;  // dynamic shared memory per CTA on sm_100
constexpr int kExpPerWarp = kRouterTE / kCompWarps;  // 4
constexpr int kXVec = 16;  // uint4 of an x row per lane (d <= 4096)
static_assert(kCompWarps == kRouterTT, "one warp per token while staging x");
static_assert(kRouterTT * kExpPerWarp == 32, "one reduced logit per lane");

struct RouterSmem {
  float* us;       // [TT][d]   x * (1 + gamma), fp32
  float* g1;       // [d]       1 + gamma
  float* wst;      // [S][TE][kChunk] router_w chunks
  float* zloc;     // [TT][TE]  this CTA's logits
  float* zall;     // [TT][E]   all logits (rank 0)
  float* inv_rms;  // [TT]
  uint64_t* full;
  uint64_t* empty;
  int* abort;
};

// Floats of everything but the weight ring.
__host__ __device__ inline int router_fixed_floats(int d) {
  return kRouterTT * d + d + kRouterTT * kRouterTE + kRouterTT * kMaxE + kRouterTT;
}
// Weight-ring depth: as many 16 KB chunks as the rest of shared memory holds
// (the ring's bytes in flight are what hide the L2 latency), at most 8.
__host__ __device__ inline int router_stages(int d) {
  const int avail = kSmemLimit - 1024 - 16 - 2 * kMaxStages * 8 - 4 * router_fixed_floats(d);
  const int st = avail / (kRouterTE * kChunk * 4);
  return st < kMaxStages ? st : kMaxStages;
}

__device__ RouterSmem carve(float* sm, int d, int S) {
  RouterSmem s;
  s.wst = sm;                                      // 1024-aligned (TMA destination)
  s.us = s.wst + S * kRouterTE * kChunk;
  s.g1 = s.us + kRouterTT * d;
  s.zloc = s.g1 + d;
  s.zall = s.zloc + kRouterTT * kRouterTE;
  s.inv_rms = s.zall + kRouterTT * kMaxE;
  s.full = reinterpret_cast<uint64_t*>(s.inv_rms + kRouterTT);
  s.empty = s.full + kMaxStages;
  s.abort = reinterpret_cast<int*>(s.empty + kMaxStages);
  return s;
}

__global__ void __launch_bounds__(kThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_rw, RouterArgs a) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  // TMA destinations start on a 1024-byte boundary
  float* sm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int d = a.d;
  const int E = a.E;
  const int S = router_stages(d);
  RouterSmem s = carve(sm, d, S);
  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRouterTT;
  const int eg = blockIdx.y;  // expert group == rank in the cluster
  const int nch = d / kChunk;
  const uint64_t timeout_ns = 1000000000ull;
  volatile int* abort = s.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kCompWarps);
    }
    *abort = 0;
    fence_mbar_init();
  }
  // Pull the first wave of expert weights into L2 while routing runs: HBM is
  // otherwise idle until the expert kernel starts.  Safe before the wait: a
  // prefetch only moves lines into the coherent L2.
  if (a.l2_prefetch) prefetch_l2_grid(a.l2_prefetch, a.l2_prefetch_bytes);
  __syncthreads();
  pdl_wait();  // x (and the weights) may come from the previous kernel
  pdl_launch_dependents();

  if (warp == kCompWarps) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_rw);
      const uint64_t pol = l2_policy_evict_last();
      uint32_t issued = 0, par = 0;
      for (int c = 0; c < nch; ++c) {
        const int st = c % S;
        if (c >= S &&
            !mbar_wait(&s.empty[st], ((c / S) - 1) & 1, abort, a.ctl, timeout_ns, 301))
          break;
        mbar_arrive_expect_tx(&s.full[st], kRouterTE * kChunk * 4);
        tma_load_2d(s.wst + st * kRouterTE * kChunk, &tm_rw, c * kChunk, eg * kRouterTE,
                    &s.full[st], pol);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | ((uint32_t)((c / S) & 1) << st);
      }
      // every issued copy lands before the CTA can leave
      for (int st = 0; st < S; ++st) {
        if (!((issued >> st) & 1u)) continue;
        const uint32_t b = smem_u32(&s.full[st]);
        const uint64_t t_0 = globaltimer_ns();
        while (!mbar_try_wait(b, (par >> st) & 1u))
          if (globaltimer_ns() - t_0 > timeout_ns) {
            record_error(a.ctl, MOE_ERR_TIMEOUT, 302);
            break;
          }
      }
    }
  } else {
    // ---------------------------------------------------------- compute warps
    // this warp's x row: its loads go out first, so they overlap the (1 + gamma)
    // staging below
    const int t = t0 + warp;
    const int n8 = d / 8;  // <= 512
    uint4 pk[kXVec];
    if (t < a.T) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * d);
#pragma unroll
      for (int j = 0; j < kXVec; ++j)
        if (lane + 32 * j < n8) pk[j] = __ldg(src + lane + 32 * j);
    }
    {  // (1 + gamma) once for the CTA, every load in flight together
      const float4* g4 = reinterpret_cast<const float4*>(a.gamma);
      for (int i = threadIdx.x; i < d / 4; i += kCompWarps * 32) {
        const float4 g = __ldg(g4 + i);
        reinterpret_cast<float4*>(s.g1)[i] = make_float4(1.f + g.x, 1.f + g.y, 1.f + g.z,
                                                         1.f + g.w);
      }
    }
    named_barrier(1, kCompWarps * 32);
    {  // u = x * (1 + gamma) for the token of this warp; 1/rms from x itself
      float* row = s.us + warp * d;
      float ss = 0.f;
      if (t < a.T) {
#pragma unroll
        for (int j = 0; j < kXVec; ++j) {
          const int i = lane + 32 * j;
          if (i < n8) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&pk[j]);
            const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
            const float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
            const float4 ga = reinterpret_cast<const float4*>(s.g1)[2 * i];
            const float4 gb = reinterpret_cast<const float4*>(s.g1)[2 * i + 1];
            ss = fmaf(f0.x, f0.x, ss); ss = fmaf(f0.y, f0.y, ss);
            ss = fmaf(f1.x, f1.x, ss); ss = fmaf(f1.y, f1.y, ss);
            ss = fmaf(f2.x, f2.x, ss); ss = fmaf(f2.y, f2.y, ss);
            ss = fmaf(f3.x, f3.x, ss); ss = fmaf(f3.y, f3.y, ss);
            reinterpret_cast<float4*>(row)[2 * i] =
                make_float4(f0.x * ga.x, f0.y * ga.y, f1.x * ga.z, f1.y * ga.w);
            reinterpret_cast<float4*>(row)[2 * i + 1] =
                make_float4(f2.x * gb.x, f2.y * gb.y, f3.x * gb.z, f3.y * gb.w);
          }
        }
      } else {
        for (int i = lane; i < d; i += 32) row[i] = 0.f;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s.inv_rms[warp] = 1.0f / sqrtf(ss / (float)d + a.eps);
    }
    named_barrier(1, kCompWarps * 32);

    float acc[kRouterTT * kExpPerWarp];
#pragma unroll
    for (int i = 0; i < kRouterTT * kExpPerWarp; ++i) acc[i] = 0.f;
    for (int c = 0; c < nch; ++c) {
      const int st = c % S;
      if (!mbar_wait(&s.full[st], (c / S) & 1, abort, a.ctl, timeout_ns, 303)) break;
      const float* wchunk = s.wst + st * kRouterTE * kChunk;
      float4 wv[kExpPerWarp];
#pragma unroll
      for (int i = 0; i < kExpPerWarp; ++i)
        wv[i] = reinterpret_cast<const float4*>(wchunk + (warp * kExpPerWarp + i) * kChunk)[lane];
#pragma unroll
      for (int t = 0; t < kRouterTT; ++t) {
        const float4 u = reinterpret_cast<const float4*>(s.us + t * d + c * kChunk)[lane];
#pragma unroll
        for (int i = 0; i < kExpPerWarp; ++i) {
          float v = acc[t * kExpPerWarp + i];
          v = fmaf(u.x, wv[i].x, v);
          v = fmaf(u.y, wv[i].y, v);
          v = fmaf(u.z, wv[i].z, v);
          v = fmaf(u.w, wv[i].w, v);
          acc[t * kExpPerWarp + i] = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.empty[st]);
    }
    // Shuffle-halving reduction of the 32 partial sums over the 32 lanes:
    // afterwards lane l holds the full sum of entry l (= token l/4, expert l%4).
#pragma unroll
    for (int step = 16; step >= 1; step >>= 1) {
      const bool upper = (lane & step) != 0;
#pragma unroll
      for (int j = 0; j < step; ++j) {
        const float send = upper ? acc[j] : acc[j + step];
        const float keep = upper ? acc[j + step] : acc[j];
        acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, step);
      }
    }
    {
      const int t = lane / kExpPerWarp;
      const int el = warp * kExpPerWarp + (lane % kExpPerWarp);
      const int e = eg * kRouterTE + el;
      float z = -INFINITY;
      if (e < E) {
        z = acc[0] * s.inv_rms[t];
        if (a.bias) z += __ldg(a.bias + e);
        if (z != z) z = -INFINITY;  // a NaN logit never wins
      }
      s.zloc[t * kRouterTE + el] = z;
    }
  }

  // ---- gather all expert groups' logits in the rank-0 CTA
  cluster.sync();
  if (eg == 0) {
    for (int i = threadIdx.x; i < kRouterTT * E; i += kThreads) {
      const int t = i / E;
      const int ee = i - t * E;
      const float* rz = cluster.map_shared_rank(s.zloc, ee / kRouterTE);
      s.zall[t * E + ee] = rz[t * kRouterTE + (ee % kRouterTE)];
    }
  }
  cluster.sync();  // the other CTAs' zloc stays alive until here
  if (eg != 0 || warp >= kRouterTT) return;

  // ---- top-k per token: warp = token, lane holds experts lane + 32c
  const int t = t0 + warp;
  if (t >= a.T) return;
  float v[kMaxE / 32];
#pragma unroll
  for (int c = 0; c < kMaxE / 32; ++c) {
    const int ee = lane + 32 * c;
    const float z = (ee < E) ? s.zall[warp * E + ee] : -INFINITY;
    v[c] = (z != z) ? -INFINITY : z;
  }
  warp_topk(v, E, a.k, lane, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k,
            a.gap ? a.gap + t : nullptr);
}

}  // namespace

}  // namespace moe

size_t moe_router_smem_bytes(int d) {
  return sizeof(float) * ((size_t)moe::router_stages(d) * moe::kRouterTE * moe::kChunk +
                          (size_t)moe::router_fixed_floats(d)) +
         2 * moe::kMaxStages * sizeof(uint64_t) + 16 + 1024;
}

cudaError_t moe_launch_router(const moe::RouterArgs& a, const CUtensorMap& tm_rw, cudaStream_t s,
                              bool pdl) {
  const size_t smem = moe_router_smem_bytes(a.d);
  cudaError_t err = cudaFuncSetAttribute(moe::router_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int groups = (a.E + moe::kRouterTE - 1) / moe::kRouterTE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.T + moe::kRouterTT - 1) / moe::kRouterTT, groups, 1);
  cfg.blockDim = dim3(moe::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = groups;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, moe::router_kernel, tm_rw, a);
}
