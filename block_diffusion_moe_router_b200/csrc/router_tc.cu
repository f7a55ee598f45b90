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
// three bf16 terms hi + mid + lo (successive 8-bit pieces of the significand),
// so every product x_i * part is exact in fp32, and all three parts accumulate into
// the same fp32 TMEM accumulator: the logits carry fp32 accumulation error
// only, as an FFMA dot product would.
//
// Work split: a CTA owns 128 tokens (UMMA M) x all experts (UMMA N = E
// rounded up to 16) over a slice of the hidden dimension; the KS (<= 16)
// CTAs that share a token tile form one cluster along the hidden dimension.
// Roles per CTA (320 threads):
//   warp 0      TMA producer: x tile [128 x 64] bf16 (128-byte swizzle) per
//               64-column step, three stages;
//   warp 1      UMMA issuer (owns the TMEM accumulator, 128 columns);
//   warps 2..9  load the fp32 router_w rows of the step (one step ahead, in
//               registers), split them times (1 + gamma) into the three
//               bf16 parts, written straight into the swizzled K-major
//               layout the UMMA reads (two buffers), and take the x^2
//               partials of the x tile;
//               afterwards they read the accumulator and push every token
//               row to the cluster rank that owns it (ceil(128 / KS) tokens
//               per rank) with distributed-shared-memory stores;
//   all warps   each rank sums its slots in rank order (deterministic) and
//               one warp per token runs the top-k.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kTThreads = 320;  // producer, UMMA, 8 converter / epilogue warps
constexpr int kConvWarps = 8;
constexpr int kTM = 128;        // tokens per CTA
constexpr int kMaxEP = 128;     // experts (N) handled here
constexpr int kXTile = kTM * kBK * 2;           // 16 KB bf16
constexpr int kWPart = kMaxEP * kBK * 2;        // 16 KB per bf16 part
constexpr int kXStages = 3;                     // x tiles (TMA)
constexpr int kWBufs = 2;                       // split router_w buffers (3 parts each)
constexpr int kWsOff = kXStages * kXTile;
constexpr int kRingBytes = kWsOff + kWBufs * 3 * kWPart;  // 144 KB
constexpr int kRowsPerThread = kMaxEP / 16;     // fp32 router_w rows a converter thread splits
constexpr int kMaxCluster = 16;
constexpr int kRecvRows = kTM + kMaxCluster;    // >= KS * ceil(kTM / KS)
// One exchanged token row: EP partial logits (padded to 128) and the two x^2
// partials (padded to four floats, so every block is a multiple of 16 bytes).
constexpr int kRowFloats = kMaxEP + 4;
constexpr int kRowBytes = kRowFloats * 4;       // 528
constexpr int kRecvOff = kRingBytes;
constexpr int kRecvBytes = kRecvRows * kRowBytes;
constexpr int kBarOff = kRecvOff + kRecvBytes;
constexpr int kTSmem = 1024 + kBarOff + 256;
// after the main loop: the outgoing rows (staging) and this rank's reduced
// logits reuse the stage ring and the part buffer
constexpr int kZallOff = (kRecvRows * kRowBytes + 1023) / 1024 * 1024;
static_assert(kZallOff + (kTM * kMaxEP + kTM) * 4 <= kRingBytes,
              "staging rows and reduced logits fit in the ring");
static_assert(kTSmem <= 232448, "router smem above the sm_100 limit");

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// v = w * g split into bf16 hi + mid + lo, packed two per 32-bit word, by
// truncation: hi keeps the top 16 bits of v's fp32 pattern (sign, exponent,
// 7 mantissa bits), r = v - hi is exact and holds the remaining 16 bits of
// significand, mid = trunc(r) its top 8, and lo = r - mid has at most 8
// significant bits, so it is already a bf16 value.  hi + mid + lo == v
// exactly, with only logic ops and subtractions on the dependency chain.
__device__ __forceinline__ float trunc_bf16(float v) {
  return __uint_as_float(__float_as_uint(v) & 0xFFFF0000u);
}
__device__ __forceinline__ uint32_t pack_hi16(float a, float b) {  // (a, b) as bf16x2
  return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x7632);
}
__device__ __forceinline__ void split3(float v0, float v1, uint32_t& hi, uint32_t& mid,
                                       uint32_t& lo) {
  const float r0 = v0 - trunc_bf16(v0), r1 = v1 - trunc_bf16(v1);
  const float q0 = r0 - trunc_bf16(r0), q1 = r1 - trunc_bf16(r1);
  hi = pack_hi16(v0, v1);
  mid = pack_hi16(r0, r1);
  lo = pack_hi16(q0, q1);
}

__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Bulk copy of `bytes` from this CTA's shared memory into a peer CTA's
// (both addresses as the peer sees them), completing on the peer's mbarrier.
__device__ __forceinline__ void bulk_to_peer(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                             uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst_cluster), "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}

__global__ void __launch_bounds__(kTThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_x, RouterArgs a, int EP, int KS) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wsp = smem + kWsOff;                                 // bf16 parts hi, mid, lo
  float* stage_rows = reinterpret_cast<float*>(smem);           // [128][kRowFloats] outgoing
  float* recv = reinterpret_cast<float*>(smem + kRecvOff);      // [KS*tpr][kRowFloats] incoming
  float* zall = reinterpret_cast<float*>(smem + kZallOff);      // [tpr][kMaxEP]
  float* inv_rms = zall + kTM * kMaxEP;                         // [tpr]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kXStages;
  uint64_t* conv = empty + kXStages;
  uint64_t* wfree = conv + kWBufs;
  uint64_t* tfull = wfree + kWBufs;
  uint64_t* rbar = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)cluster.block_rank();  // K slice
  const int t0 = blockIdx.x * kTM;
  const int nst = a.d / kBK;
  const int kb0 = rank * nst / KS;
  const int kb1 = (rank + 1) * nst / KS;
  const int nk = kb1 - kb0;
  // Rank r owns tokens [r*tpr, r*tpr + tpr) of the tile (the last ranks may
  // own fewer, or none).
  const int tpr = (kTM + KS - 1) / KS;
  const int tb = rank * tpr;
  const int tcount = max(0, min(tpr, kTM - tb));
  const uint64_t timeout_ns = 1000000000ull;
  Ctl* ctl = a.ctl;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kWBufs; ++i) {
      mbar_init(&conv[i], kConvWarps);
      mbar_init(&wfree[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(rbar, 1);
    *s_abort = 0;
    fence_mbar_init();
    // every rank sends this one its rows of our tokens (tx may run ahead of
    // this: an mbarrier's transaction count may go negative)
    mbar_arrive_expect_tx(rbar, (uint32_t)(KS * tcount * kRowBytes));
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMaxEP);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
  }
  // Pull the first expert weights into L2 while routing runs: HBM is
  // otherwise idle until the expert kernel starts.
  if (a.l2_prefetch) prefetch_l2_grid(a.l2_prefetch, a.l2_prefetch_bytes);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Peers may target this CTA's barrier only once it is initialised: arrive
  // now, wait just before the first remote copy.
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // x, router_w and gamma may come from the previous kernel
  pdl_launch_dependents();

  float my_ssq = 0.f;
  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------- producer
      const uint64_t pol = l2_policy_evict_last();
      uint32_t issued = 0, par = 0;
      for (int i = 0; i < nk; ++i) {
        const int st = i % kXStages;
        // refill only after the UMMAs of the step that last used the stage
        if (i >= kXStages &&
            !mbar_wait(&empty[st], ((i / kXStages) - 1) & 1, s_abort, ctl, timeout_ns, 401))
          break;
        mbar_arrive_expect_tx(&full[st], kXTile);
        tma_load_2d(smem + st * kXTile, &tm_x, (kb0 + i) * kBK, t0, &full[st], pol);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | ((uint32_t)((i / kXStages) & 1) << st);
      }
      for (int st = 0; st < kXStages; ++st) {  // every issued copy lands before exit
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
      for (int i = 0; i < nk; ++i) {
        const int st = i % kXStages;
        const int wb = i % kWBufs;
        if (!mbar_wait(&full[st], (i / kXStages) & 1, s_abort, ctl, timeout_ns, 403) ||
            !mbar_wait(&conv[wb], (i / kWBufs) & 1, s_abort, ctl, timeout_ns, 403))
          break;
        tc_fence_after();
        const uint32_t sx = smem_u32(smem + st * kXTile);
        const uint32_t sw = smem_u32(wsp + wb * 3 * kWPart);
#pragma unroll
        for (int kk = 0; kk < kBK / kUmmaK; ++kk)
#pragma unroll
          for (int p = 0; p < 3; ++p)
            umma_bf16(tmem_base, sdesc_k_sw128(sx + kk * kUmmaK * 2),
                      sdesc_k_sw128(sw + p * kWPart + kk * kUmmaK * 2), idesc,
                      (i | kk | p) ? 1u : 0u);
        umma_commit(&empty[st]);  // the x tile
        umma_commit(&wfree[wb]);  // the part buffer
      }
      umma_commit(tfull);  // arrives once every issued UMMA is done
    }
  } else {
    // ------------------------------------------------ converters (256 threads)
    // Split: thread c owns fp32 column group j = c % 16 (4 columns) of rows
    // n = c / 16 + 16 r (three steps of them in flight).  The bf16 parts land in 128-byte K-major rows whose 16-byte
    // chunk q sits at q ^ (n % 8) (the 128-byte swizzle).  x^2: the thread
    // owns row c % 128, half c / 128 of the x tile's 64 columns.
    const int c = threadIdx.x - 64;
    const int j = c & 15;
    const int n0 = c >> 4;
    const int xr = c & (kTM - 1);
    const int xh = c >> 7;
    const int E = a.E;
    // fp32 router_w rows in registers, three steps in flight: step i sits in
    // slot i % 3 and its slot is refilled with step i + 3 once split
    // (slot entry kRowsPerThread holds the step's four gamma values)
    float4 w0[kRowsPerThread + 1], w1[kRowsPerThread + 1], w2[kRowsPerThread + 1];
    auto load_rows = [&](float4 (&dst)[kRowsPerThread + 1], int i) {
      if (i >= nk) return;
      const int kb = kb0 + i;
#pragma unroll
      for (int r = 0; r < kRowsPerThread; ++r) {
        const int n = n0 + 16 * r;
        dst[r] = (n < E) ? __ldg(reinterpret_cast<const float4*>(a.router_w + (size_t)n * a.d +
                                                                  kb * kBK) + j)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      dst[kRowsPerThread] = __ldg(reinterpret_cast<const float4*>(a.gamma + kb * kBK) + j);
    };
    // split step i (rows in wr) into part buffer i % 2, then the x^2 of its x
    // tile; false when a wait gave up
    auto step = [&](const float4 (&wr)[kRowsPerThread + 1], int i) -> bool {
      const int st = i % kXStages;
      const int wb = i % kWBufs;
      const float4 g = wr[kRowsPerThread];
      const float g0 = 1.f + g.x, g1 = 1.f + g.y, g2 = 1.f + g.z, g3 = 1.f + g.w;
      // the part buffer is free once the UMMAs two steps back are done
      if (i >= kWBufs &&
          !mbar_wait(&wfree[wb], ((i / kWBufs) - 1) & 1, s_abort, ctl, timeout_ns, 406))
        return false;
      uint8_t* wp = wsp + wb * 3 * kWPart;
#pragma unroll
      for (int r = 0; r < kRowsPerThread; ++r) {
        const int n = n0 + 16 * r;
        if (n < EP) {
          uint32_t h0, m0, l0, h1, m1, l1;
          split3(wr[r].x * g0, wr[r].y * g1, h0, m0, l0);
          split3(wr[r].z * g2, wr[r].w * g3, h1, m1, l1);
          const int off = n * 128 + (((j >> 1) ^ (n & 7)) << 4) + ((j & 1) << 3);
          *reinterpret_cast<uint2*>(wp + off) = make_uint2(h0, h1);
          *reinterpret_cast<uint2*>(wp + kWPart + off) = make_uint2(m0, m1);
          *reinterpret_cast<uint2*>(wp + 2 * kWPart + off) = make_uint2(l0, l1);
        }
      }
      if (!mbar_wait(&full[st], (i / kXStages) & 1, s_abort, ctl, timeout_ns, 404)) return false;
      const uint8_t* row = smem + st * kXTile + xr * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 pk = *reinterpret_cast<const uint4*>(row + (((xh * 4 + q) ^ (xr & 7)) << 4));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&pk);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = __bfloat1622float2(h2[u]);
          my_ssq = fmaf(f.x, f.x, my_ssq);
          my_ssq = fmaf(f.y, f.y, my_ssq);
        }
      }
      fence_async_smem();  // generic-proxy stores -> visible to the UMMA
      __syncwarp();
      if (lane == 0) mbar_arrive(&conv[wb]);
      return true;
    };
    load_rows(w0, 0);
    load_rows(w1, 1);
    load_rows(w2, 2);
#pragma unroll 1
    for (int i = 0; i < nk; i += 3) {
      if (!step(w0, i)) break;
      load_rows(w0, i + 3);
      if (i + 1 >= nk || !step(w1, i + 1)) break;
      load_rows(w1, i + 4);
      if (i + 2 >= nk || !step(w2, i + 2)) break;
      load_rows(w2, i + 5);
    }
  }

  // ---- exchange.  Each converter thread copies its accumulator row (and its
  // x^2 partial) into the staging rows; row r of the tile goes to rank
  // r / tpr, where it lands as row (rank * tpr + r % tpr) of the receive
  // buffer.  The rows for one owner are contiguous, so one bulk copy per
  // owner moves them (completing on the owner's barrier); each rank then sums
  // its slots in rank order, which keeps the result deterministic.
  if (warp >= 2) {
    const bool tmem_ok = mbar_wait(tfull, 0, s_abort, ctl, timeout_ns, 405);
    tc_fence_after();
    const int c = threadIdx.x - 64;
    const int q4 = warp & 3;       // TMEM lane quarter this warp may read
    const int r = q4 * 32 + lane;  // token row of the tile
    float* dst = stage_rows + (size_t)r * kRowFloats;
    for (int c0 = ((warp - 2) >> 2) * 32; c0 < EP; c0 += 64) {
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
    stage_rows[(size_t)(c & (kTM - 1)) * kRowFloats + kMaxEP + (c >> 7)] = my_ssq;
    fence_async_smem();  // staging rows -> visible to the bulk copies
  }
  tc_fence_before();
  __syncthreads();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (threadIdx.x == 0) {
    const uint32_t src0 = smem_u32(stage_rows);
    const uint32_t dst0 = smem_u32(recv) + (uint32_t)(rank * tpr * kRowBytes);
    const uint32_t bar0 = smem_u32(rbar);
    for (int q = 0; q < KS; ++q) {
      const int rows = min(tpr, kTM - q * tpr);
      if (rows <= 0) break;
      bulk_to_peer(mapa_shared(dst0, q), src0 + (uint32_t)(q * tpr * kRowBytes),
                   (uint32_t)(rows * kRowBytes), mapa_shared(bar0, q));
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMaxEP);
  }
  if (threadIdx.x == 32) {  // every rank's rows of our tokens have landed
    const uint32_t b = smem_u32(rbar);
    const uint64_t tq = globaltimer_ns();
    while (!mbar_try_wait(b, 0))
      if (globaltimer_ns() - tq > timeout_ns) {
        record_error(ctl, MOE_ERR_TIMEOUT, 407);
        break;
      }
  }
  __syncthreads();

  // rank-order sums, four experts per thread (EP is a multiple of 16)
  const int EP4 = EP / 4;
  for (int idx = threadIdx.x; idx < tcount * EP4; idx += kTThreads) {
    const int tl = idx / EP4;
    const int e = 4 * (idx - tl * EP4);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < KS; ++q) {
      const float4 r =
          *reinterpret_cast<const float4*>(recv + (size_t)(q * tpr + tl) * kRowFloats + e);
      s.x += r.x;
      s.y += r.y;
      s.z += r.z;
      s.w += r.w;
    }
    *reinterpret_cast<float4*>(zall + tl * kMaxEP + e) = s;
  }
  if (threadIdx.x < tcount) {
    float s2 = 0.f;
    for (int q = 0; q < KS; ++q) {
      const float* rr = recv + (size_t)(q * tpr + threadIdx.x) * kRowFloats + kMaxEP;
      s2 += rr[0] + rr[1];
    }
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
    for (int cc = 0; cc < kMaxEP / 32; ++cc) {
      const int ee = lane + 32 * cc;
      float z = -INFINITY;
      if (ee < E) {
        z = zall[tl * kMaxEP + ee] * inv_rms[tl];
        if (a.bias) z += __ldg(a.bias + ee);
        if (z != z) z = -INFINITY;
      }
      v[cc] = z;
    }
    warp_topk(v, E, a.k, lane, a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k,
              a.gap ? a.gap + t : nullptr);
  }
  if (threadIdx.x == 0)  // the outgoing copies have read the staging rows
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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

cudaError_t set_attrs() {
  cudaError_t err = cudaFuncSetAttribute(
      moe::router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, moe::kTSmem);
  if (err != cudaSuccess) return err;
  return cudaFuncSetAttribute(moe::router_tc_kernel,
                              cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

int max_active_clusters(int ns) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_max_clusters_mu);
  if (!g_max_clusters_ok[dev]) {
    if (set_attrs() != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
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
      if (cudaOccupancyMaxActiveClusters(&n, moe::router_tc_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      g_max_clusters[dev][c] = n;
    }
    g_max_clusters_ok[dev] = true;
  }
  return g_max_clusters[dev][ns];
}

}  // namespace

// Hidden-dimension split (= cluster size): as many 64-column steps as there
// are, up to 16, lowered while the token tiles would not all be resident in
// one wave of clusters.
int moe_router_tc_splits(int d, int T) {
  const int nst = d / moe::kBK;
  const int cap = nst < moe::kMaxCluster ? nst : moe::kMaxCluster;
  const int tiles = (T + moe::kTM - 1) / moe::kTM;
  for (int c = cap; c >= 1; --c)
    if (tiles <= max_active_clusters(c)) return c;
  return 1;
}

cudaError_t moe_launch_router_tc(const moe::RouterArgs& a, const CUtensorMap& tm_x, int EP,
                                 cudaStream_t s, bool pdl) {
  const int KS = moe_router_tc_splits(a.d, a.T);
  cudaError_t err = set_attrs();
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.T + moe::kTM - 1) / moe::kTM, KS, 1);
  cfg.blockDim = dim3(moe::kTThreads, 1, 1);
  cfg.dynamicSmemBytes = moe::kTSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = KS;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, moe::router_tc_kernel, tm_x, a, EP, KS);
}
