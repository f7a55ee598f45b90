// router_tc.cu -- the MoE router on tcgen05 tensor cores (E <= 128).
//
// Same result as the FFMA router (router.cu): the router's own (1+gamma)
// RMSNorm of the raw residual, fp32 logits against router_w (+ bias),
// softmax, top-k with the lower index winning ties, renormalised weights
// (Quant-Tuner pull request "Add DiffusionGemma (Gemma-4 MoE block-diffusion)
// support", "Answers to the motivating questions"; top-8 of 128 from its
// Summary).
//
// Exactness of the tensor-core logits: the logit is
//   z_e = (sum_i x_i * W'_ei) / rms(x),  W'_ei = router_w[e][i] * (1 + gamma_i)
// with x already bf16.  W' (fp32, 24-bit significand) is split exactly into
// three bf16 terms hi + mid + lo (each captures the next 8 bits), so every
// product x_i * part is exact in fp32 and the UMMA accumulates in fp32: the
// logits carry fp32 accumulation error only, as an FFMA dot product would.
//
// Work split: a CTA owns 128 tokens (UMMA M) x all experts (UMMA N = E
// rounded up to 16) over a slice of the hidden dimension; the 8 (or fewer)
// CTAs that share a token tile form a cluster along the hidden dimension.
// Each accumulates its partial logits in TMEM (plus the partial sum of x^2,
// read from the staged x tiles) and pushes every token row to the rank that
// owns it (ceil(128 / cluster) tokens per rank) with distributed-shared-
// memory stores; each rank sums its slots in rank order (deterministic) and
// one warp per token runs the top-k.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kTThreads = 192;   // producer, UMMA, 4 epilogue warps
constexpr int kTM = 128;         // tokens per CTA
constexpr int kTStages = 3;
constexpr int kXTile = kTM * kBK * 2;          // 16 KB
constexpr int kMaxEP = 128;                    // experts (N) handled here
constexpr int kWTile = kMaxEP * kBK * 2;       // 16 KB per split part
constexpr int kTStage = kXTile + 3 * kWTile;   // 64 KB
constexpr int kMaxCluster = 8;
constexpr int kRecvRows = kTM + kMaxCluster;   // >= nsplit * ceil(kTM / nsplit)
constexpr int kTSmem = 1024 + kTStages * kTStage + 1024;
static_assert((kRecvRows * kMaxEP + kRecvRows + kTM * kMaxEP + kTM) * 4 <= kTStages * kTStage,
              "receive buffers and reduced logits reuse the ring");

// W'[e][i] = router_w[e][i] * (1 + gamma[i]) split into three bf16 parts,
// wsplit[p][e][i], rows e >= E zero.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ rw,
                                                           const float* __restrict__ gamma, int E,
                                                           int EP, int d,
                                                           __nv_bfloat16* __restrict__ wsplit) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n = (size_t)EP * d;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / d);
    const int k = (int)(i - (size_t)e * d);
    float v = 0.f;
    if (e < E) v = __ldg(rw + i) * (1.f + __ldg(gamma + k));
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    wsplit[i] = hi;
    wsplit[n + i] = mid;
    wsplit[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

__global__ void __launch_bounds__(kTThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_w, RouterArgs a, int EP, int nsplit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  // After the main loop the ring is reused: the receive buffer for the
  // partial logits of this rank's tokens from every rank, their x^2
  // partials, then this rank's reduced logits.
  float* recv = reinterpret_cast<float*>(smem);          // [nsplit*tpr <= kRecvRows][kMaxEP]
  float* recv_ssq = recv + kRecvRows * kMaxEP;            // [kRecvRows]
  float* zall = recv_ssq + kRecvRows;                     // [tpr][kMaxEP]
  float* inv_rms = zall + kTM * kMaxEP;                   // [tpr]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTStages * kTStage);
  uint64_t* empty = full + kTStages;
  uint64_t* sqd = empty + kTStages;   // x tile's sum of squares taken
  uint64_t* tfull = sqd + kTStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = blockIdx.y;  // K slice == rank in the cluster
  const int t0 = blockIdx.x * kTM;
  const int nst = a.d / kBK;
  const int kb0 = rank * nst / nsplit;
  const int kb1 = (rank + 1) * nst / nsplit;
  const uint64_t timeout_ns = 1000000000ull;
  Ctl* ctl = a.ctl;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&sqd[i], 4);
    }
    mbar_init(tfull, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMaxEP);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  // first-wave expert weights into L2 while routing runs (see router.cu)
  if (a.l2_prefetch) prefetch_l2_grid(a.l2_prefetch, a.l2_prefetch_bytes);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // x and the split weight come from earlier kernels
  pdl_launch_dependents();

  float my_ssq = 0.f;
  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------- producer
      const uint64_t pol = l2_policy_evict_last();
      const uint32_t tx = kXTile + 3 * EP * kBK * 2;
      uint32_t issued = 0, par = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0;
        const int st = i % kTStages;
        // refill only after the UMMAs and the x^2 readers are done with it
        if (i >= kTStages &&
            (!mbar_wait(&empty[st], ((i / kTStages) - 1) & 1, s_abort, ctl, timeout_ns, 401) ||
             !mbar_wait(&sqd[st], ((i / kTStages) - 1) & 1, s_abort, ctl, timeout_ns, 406)))
          break;
        uint8_t* sx = ring + st * kTStage;
        mbar_arrive_expect_tx(&full[st], tx);
        tma_load_2d(sx, &tm_x, kb * kBK, t0, &full[st], pol);
        for (int p = 0; p < 3; ++p)
          tma_load_2d(sx + kXTile + p * kWTile, &tm_w, kb * kBK, p * EP, &full[st], pol);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | ((uint32_t)((i / kTStages) & 1) << st);
      }
      for (int st = 0; st < kTStages; ++st) {  // drain
        if (!((issued >> st) & 1u)) continue;
        const uint32_t b = smem_u32(&full[st]);
        const uint64_t tq = globaltimer_ns();
        while (!mbar_try_wait(b, (par >> st) & 1u))
          if (globaltimer_ns() - tq > timeout_ns) {
            record_error(ctl, MOE_ERR_TIMEOUT, 402);
            break;
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------- UMMA issuer
      const uint32_t idesc = idesc_bf16_f32(kTM, EP);
      for (int kb = kb0; kb < kb1; ++kb) {
        const int i = kb - kb0;
        const int st = i % kTStages;
        if (!mbar_wait(&full[st], (i / kTStages) & 1, s_abort, ctl, timeout_ns, 403)) break;
        tc_fence_after();
        const uint32_t sx = smem_u32(ring + st * kTStage);
#pragma unroll
        for (int kk = 0; kk < kBK / kUmmaK; ++kk)
#pragma unroll
          for (int p = 0; p < 3; ++p)
            umma_bf16(tmem_base, sdesc_k_sw128(sx + kk * kUmmaK * 2),
                      sdesc_k_sw128(sx + kXTile + p * kWTile + kk * kUmmaK * 2), idesc,
                      (i | kk | p) ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      umma_commit(tfull);  // also drains every issued UMMA
    }
  } else {
    // ---------------------------------------------------------- x^2 partials
    // Each epilogue thread owns one token row of the staged x tiles (128-byte
    // swizzled rows): 16-byte chunk c of row r sits at chunk c ^ (r % 8).
    const int r = (warp & 3) * 32 + lane;
    for (int kb = kb0; kb < kb1; ++kb) {
      const int i = kb - kb0;
      const int st = i % kTStages;
      if (!mbar_wait(&full[st], (i / kTStages) & 1, s_abort, ctl, timeout_ns, 404)) break;
      const uint8_t* row = ring + st * kTStage + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 pk = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) * 16));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&pk);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(h2[q]);
          my_ssq = fmaf(f.x, f.x, my_ssq);
          my_ssq = fmaf(f.y, f.y, my_ssq);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sqd[st]);
    }
  }
  __syncthreads();

  // ---- partial logits.  Rank r of the cluster owns tokens [r*tpr, r*tpr +
  // tpr) of the tile.  Every CTA pushes each of its partial rows straight into
  // the owner's receive buffer with distributed-shared-memory stores (which
  // pipeline, unlike remote loads), then each rank sums its slots in rank
  // order.  The first cluster barrier makes sure every CTA is done with its
  // stage ring (the receive buffers live there) before anyone writes.
  const int tpr = (kTM + nsplit - 1) / nsplit;  // ceil split: the last rank may take fewer
  const int tb = rank * tpr;
  const int tcount = max(0, min(tpr, kTM - tb));
  bool tmem_ok = true;
  if (warp >= 2) {
    tmem_ok = mbar_wait(tfull, 0, s_abort, ctl, timeout_ns, 405);
    tc_fence_after();
  }
  cluster.sync();
  if (warp >= 2) {
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;     // token row of the tile
    const int owner = r / tpr;
    const int tl = r - owner * tpr;
    float* dst = cluster.map_shared_rank(recv, owner) + (size_t)(rank * tpr + tl) * kMaxEP;
    for (int c0 = 0; c0 < EP; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem_base + ((uint32_t)(q4 * 32) << 16) + c0, v);
      tmem_wait_ld();
      if (!tmem_ok) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = 0u;
      }
#pragma unroll
      for (int jj = 0; jj < 32; jj += 4)
        *reinterpret_cast<float4*>(dst + c0 + jj) =
            make_float4(__uint_as_float(v[jj]), __uint_as_float(v[jj + 1]),
                        __uint_as_float(v[jj + 2]), __uint_as_float(v[jj + 3]));
    }
    cluster.map_shared_rank(recv_ssq, owner)[rank * tpr + tl] = my_ssq;
  }
  tc_fence_before();
  cluster.sync();  // every push has landed
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMaxEP);
  }
  // rank-order sums, four experts per thread (EP is a multiple of 16)
  const int EP4 = EP / 4;
  for (int idx = threadIdx.x; idx < tcount * EP4; idx += kTThreads) {
    const int tl = idx / EP4;
    const int e = 4 * (idx - tl * EP4);
    float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < nsplit; ++q) {
      const float4 r = *reinterpret_cast<const float4*>(recv + (size_t)(q * tpr + tl) * kMaxEP + e);
      sacc.x += r.x;
      sacc.y += r.y;
      sacc.z += r.z;
      sacc.w += r.w;
    }
    *reinterpret_cast<float4*>(zall + tl * kMaxEP + e) = sacc;
  }
  if (threadIdx.x < tcount) {
    float s2 = 0.f;
    for (int q = 0; q < nsplit; ++q) s2 += recv_ssq[q * tpr + threadIdx.x];
    inv_rms[threadIdx.x] = 1.0f / sqrtf(s2 / (float)a.d + a.eps);
  }
  __syncthreads();

  // ---- top-k: one warp per token, lane holds experts lane + 32c
  const int E = a.E;
  for (int tl = warp; tl < tcount; tl += kTThreads / 32) {
    const int t = t0 + tb + tl;
    if (t >= a.T) break;
    float v[kMaxEP / 32];
#pragma unroll
    for (int c = 0; c < kMaxEP / 32; ++c) {
      const int ee = lane + 32 * c;
      float z = -INFINITY;
      if (ee < E) {
        z = zall[tl * kMaxEP + ee] * inv_rms[tl];
        if (a.bias) z += __ldg(a.bias + ee);
        if (z != z) z = -INFINITY;
      }
      v[c] = z;
    }
    warp_topk(v, E, a.k, lane, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k,
              a.gap ? a.gap + t : nullptr);
  }
}

}  // namespace

}  // namespace moe

namespace {

// Clusters of each size that can be resident at once on this device (a
// cluster must fit inside one GPC, so the count is not simply SMs / size).
constexpr int kMaxDevices = 64;
int g_max_clusters[kMaxDevices][moe::kMaxCluster + 1];
bool g_max_clusters_ok[kMaxDevices];
std::mutex g_max_clusters_mu;

int max_active_clusters(int ns) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_max_clusters_mu);
  if (!g_max_clusters_ok[dev]) {
    if (cudaFuncSetAttribute(moe::router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             moe::kTSmem) != cudaSuccess)
      return 0;
    for (int c = 1; c <= moe::kMaxCluster; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, c, 1);
      cfg.blockDim = dim3(moe::kTThreads, 1, 1);
      cfg.dynamicSmemBytes = moe::kTSmem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 1;
      attr.val.clusterDim.y = c;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, moe::router_tc_kernel, &cfg) != cudaSuccess) n = 0;
      g_max_clusters[dev][c] = n;
    }
    g_max_clusters_ok[dev] = true;
  }
  return g_max_clusters[dev][ns];
}

}  // namespace

// Hidden-dimension split (= cluster size): as many as there are K stages up
// to the cluster limit, lowered while the token tiles would not all be
// resident in one wave of clusters.
int moe_router_tc_splits(int d, int T) {
  const int nst = d / moe::kBK;
  const int cap = nst < moe::kMaxCluster ? nst : moe::kMaxCluster;
  const int tiles = (T + moe::kTM - 1) / moe::kTM;
  for (int c = cap; c >= 1; --c)
    if (tiles <= max_active_clusters(c)) return c;
  return cap;
}

cudaError_t moe_launch_router_split(const float* rw, const float* gamma, int E, int EP, int d,
                                    __nv_bfloat16* wsplit, int num_sms, cudaStream_t s,
                                    bool pdl) {
  const size_t n = (size_t)EP * d;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 4 * num_sms) blocks = 4 * num_sms;
  return moe::launch_pdl(moe::router_split_kernel, dim3(blocks), dim3(256), 0, s, pdl, rw, gamma,
                         E, EP, d, wsplit);
}

cudaError_t moe_launch_router_tc(const moe::RouterArgs& a, const CUtensorMap& tm_x,
                                 const CUtensorMap& tm_w, int EP, cudaStream_t s, bool pdl) {
  const int nsplit = moe_router_tc_splits(a.d, a.T);
  cudaError_t err = cudaFuncSetAttribute(moe::router_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         moe::kTSmem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.T + moe::kTM - 1) / moe::kTM, nsplit, 1);
  cfg.blockDim = dim3(moe::kTThreads, 1, 1);
  cfg.dynamicSmemBytes = moe::kTSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = nsplit;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, moe::router_tc_kernel, tm_x, tm_w, a, EP, nsplit);
}
