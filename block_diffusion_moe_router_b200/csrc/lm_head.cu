// lm_head.cu -- the step after the layer stack: logits of every canvas token
// over the whole vocabulary, reduced on chip to what the entropy-bound
// sampler needs (fucina docs "DiffusionGemma 26B-A4B -- block text-diffusion":
// the runner denoises 256-token canvases with the entropy-bound sampler,
// temperature 0.8 -> 0.4, bound 0.1; auto-round pull request:
// EntropyBoundSamplerConfig entropy_bound 0.1).
//
// For each token t (h_t bf16 [d], W bf16 [V, d]):
//   z_v = h_t . W[v], optionally c * tanh(z_v / c);  u_v = z_v / temperature
//   logZ = log sum_v exp(u_v);  H = logZ - sum_v softmax(u)_v u_v
//   token = argmax_v z_v (lowest index on ties)
// and, over the still-masked positions, entropy-bounded acceptance: sorted
// by (H, position), the longest prefix whose entropies, all but the last,
// sum to at most the bound.
//
// Kernels:
//   lmhead_gemm_pair_kernel: persistent, on pairs of CTAs (2-CTA clusters,
//     one CTA per SM); a unit is (256 vocabulary rows, chunk of <= 256
//     tokens).  One tcgen05 UMMA of M = 256 tokens (128 in each CTA) by
//     N = 256 vocabulary rows (128 in each CTA's shared memory) per K = 16
//     step, so W streams from HBM once and each SM reads half the operand
//     bytes per multiply-add a 1-CTA M = 128 UMMA would.  Warp 0 streams W
//     (TMA, evict-first), warp 6 streams h (evict-last), warp 1 of the even
//     CTA issues the UMMAs into two 256-column TMEM accumulators per CTA,
//     warps 2..5 reduce them: the TMEM lane is the token, so each thread
//     folds its token's 256 logits in registers into (max, sum exp, sum
//     exp * u, argmax) and writes one float4 per (token, 256-row tile).  The
//     logits never reach HBM or shared memory.
//   lmhead_finalize_kernel: one CTA per token folds its V/256 partials in a
//     fixed order (deterministic) into logZ, H and the argmax.
//   lmhead_accept_kernel: one CTA ranks the masked positions by (H, t) and
//     walks them in that order summing the entropies in fp64.
// Every wait is bounded like the expert kernels' (MOE_ERR_TIMEOUT).
#include "expert_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 224;
constexpr int kRingBytes = 224 * 1024;
enum { kWhereLmA = 40, kWhereLmB, kWhereLmMma, kWhereLmEpi };

struct Stat {
  float m, s, q;
  int i;
};

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kPastV = -1.0e30f;  // scaled logit of a row past V

// 2^x by the hardware approximation (relative error ~2^-22; 2^-1e30 = 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Fold b into a: running max, sums rescaled to the new max, lowest index
// among equal maxima.  An empty side has m = -inf.
__device__ __forceinline__ void fold(Stat& a, const Stat& b) {
  if (b.m == -INFINITY) return;
  if (a.m == -INFINITY) {
    a = b;
    return;
  }
  if (b.m > a.m || (b.m == a.m && b.i < a.i)) {
    const float r = expf(a.m - b.m);
    a.s = b.s + a.s * r;
    a.q = b.q + a.q * r;
    a.m = b.m;
    a.i = b.i;
  } else {
    const float r = expf(b.m - a.m);
    a.s += b.s * r;
    a.q += b.q * r;
  }
}

// ---------------------------------------------------------------- CTA pairs
// The GEMM runs on pairs of CTAs (a 2-CTA cluster): one UMMA of M = 256
// covers both CTAs' 128 W rows against N tokens whose B rows are split
// between the two CTAs' shared memory, so each SM reads half the B operand
// per multiply-add that a 1-CTA M = 128 UMMA reads (at N = 256 the 1-CTA
// kernel is bound by those shared-memory reads at ~50% of the tensor peak).
// The even CTA of the pair issues the UMMAs and owns the full barriers; both
// CTAs' TMA copies complete on them (the .cta_group::2 form allows the peer
// CTA's barrier), and the UMMA commits arrive on both CTAs' barriers.

constexpr int kPairMaxA = 6;                 // h stages (L2)
constexpr int kPairMaxB = 8;                 // W stages (HBM)
constexpr int kPairTok = 128;                // token rows per CTA (UMMA M / 2)
constexpr int kPairV = 256;                  // vocabulary rows per unit (UMMA N)
constexpr int kPairStage = kPairTok * kBK * 2;  // 16 KB, also a CTA's half of a W stage
constexpr int kPairBarBytes = 8 * (2 * kPairMaxA + 2 * kPairMaxB + 4 + 1);
constexpr int kPairSmemBytes = 1024 + kRingBytes + kPairBarBytes + 256;

// A unit of a pair is (256 vocabulary rows, chunk of <= 256 tokens).  The
// UMMA is M = 256 tokens (128 per CTA: A = h, from each CTA's own smem) by
// N = 256 vocabulary rows (B = W, 128 rows in each CTA's smem), so W is
// streamed from HBM exactly once and each SM reads 4 KB of A and 4 KB of B
// per K = 16 step.  The accumulator lane is the token: each epilogue thread
// folds its own token's 256 logits in registers (online max / sums), with no
// shared-memory transpose and no barriers, and writes one partial per
// (token, 256-row tile).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    lmhead_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                            const __grid_constant__ CUtensorMap tm_h, LmHeadArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + kRingBytes);
  uint64_t* emptyA = fullA + kPairMaxA;
  uint64_t* fullB = emptyA + kPairMaxA;
  uint64_t* emptyB = fullB + kPairMaxB;
  uint64_t* tfull = emptyB + kPairMaxB;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  Ctl* ctl = a.ctl;

  if (threadIdx.x == 0) {
    // The full barriers of the leader collect both CTAs' copies: the leader
    // arms them with both CTAs' bytes, and a peer's copy for a stage is only
    // issued after that stage's previous use was consumed, so it always
    // lands in the phase the leader arms (a peer arrival is not needed).
    for (int i = 0; i < kPairMaxA; ++i) {
      mbar_init(&fullA[i], 1);
      mbar_init(&emptyA[i], 1);  // the pair's UMMA commit
    }
    for (int i = 0; i < kPairMaxB; ++i) {
      mbar_init(&fullB[i], 1);
      mbar_init(&emptyB[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // four epilogue warps of each CTA (leader's copy used)
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_h);
  }
  tc_fence_before();
  cluster_barrier();  // both CTAs' barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();

  const int VT2 = (a.V + kPairV - 1) / kPairV;
  const int NC = (a.T + 2 * kPairTok - 1) / (2 * kPairTok);
  const int U = VT2 * NC;
  const int nclus = gridDim.x / 2;
  const int clus = blockIdx.x / 2;
  const int nkb = a.d / kBK;
  uint8_t* ringA = ring;                          // h
  uint8_t* ringB = ring + kPairMaxA * kPairStage;  // W

  if (warp == 0) {
    // ------------------------------------------------------------ W producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = clus; u < U && ok; u += nclus) {
        const int vt2 = u % VT2;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyB[stage], phase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmA)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&fullB[stage], 2 * kPairStage);
          tma_load_2d_pair(ringB + stage * kPairStage, &tm_w, kb * kBK,
                           vt2 * kPairV + (int)rank * kPairTok,
                           mapa_rank(smem_u32(&fullB[stage]), 0), pol_w);
          if (++stage == kPairMaxB) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ h producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = clus; u < U && ok; u += nclus) {
        const int ch = u / VT2;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyA[stage], phase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmB)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&fullA[stage], 2 * kPairStage);
          tma_load_2d_pair(ringA + stage * kPairStage, &tm_h, kb * kBK,
                           ch * 2 * kPairTok + (int)rank * kPairTok,
                           mapa_rank(smem_u32(&fullA[stage]), 0), pol_act);
          if (++stage == kPairMaxA) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer (leader)
    if (leader && lane == 0) {
      int sa_i = 0, sb_i = 0;
      uint32_t pa = 0, pb = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32(2 * kPairTok, kPairV);
      for (int u = clus; u < U && ok; u += nclus) {
        if (!mbar_wait(&tempty[acc], aphase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmMma)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * kPairV);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&fullA[sa_i], pa, s_abort, ctl, a.timeout_ns, kWhereLmMma) ||
              !mbar_wait(&fullB[sb_i], pb, s_abort, ctl, a.timeout_ns, kWhereLmMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ringA + sa_i * kPairStage);
          const uint32_t sb = smem_u32(ringB + sb_i * kPairStage);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma_pair_bf16(dt, sdesc_k_sw128(sa + kk * kUmmaK * 2),
                           sdesc_k_sw128(sb + kk * kUmmaK * 2), idesc, (kb | kk) ? 1u : 0u);
          umma_pair_commit(&emptyA[sa_i], 3);
          umma_pair_commit(&emptyB[sb_i], 3);
          if (++sa_i == kPairMaxA) {
            sa_i = 0;
            pa ^= 1;
          }
          if (++sb_i == kPairMaxB) {
            sb_i = 0;
            pb ^= 1;
          }
        }
        if (!ok) break;
        umma_pair_commit(&tfull[acc], 3);
        acc ^= 1;
        if (acc == 0) aphase ^= 1;
      }
      umma_pair_commit(drain, 1);
      mbar_wait_drain(drain, 0, ctl, a.timeout_ns);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q4 = warp & 3;
    const int tl = q4 * 32 + lane;  // token inside this CTA's 128 (TMEM lane)
    const float c2 = a.inv_temp * 1.4426950408889634f;  // log2(e) / temperature
    const uint32_t tempty_l0 = mapa_rank(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_l1 = mapa_rank(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t aphase = 0;
    for (int u = clus; u < U; u += nclus) {
      if (!mbar_wait(&tfull[acc], aphase, s_abort, ctl, a.timeout_ns, kWhereLmEpi)) break;
      tc_fence_after();
      const int vt2 = u % VT2, ch = u / VT2;
      const int tok = ch * 2 * kPairTok + (int)rank * kPairTok + tl;
      const int v0 = vt2 * kPairV;
      const uint32_t tbase = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * kPairV);
      Stat st;
      st.m = -INFINITY;
      st.s = 0.f;
      st.q = 0.f;
      st.i = 0;
      for (int c0 = 0; c0 < kPairV; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + c0, v);
        tmem_wait_ld();
        // base-2 scaled logits w = u * log2(e); rows past V get a finite
        // sentinel (so that 2^(w - max) * w is 0, not 0 * -inf)
        float x[32];
        float cm = kPastV;
        int ci = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float z = __uint_as_float(v[i]);
          if (a.softcap > 0.f) z = a.softcap * tanhf(z / a.softcap);
          x[i] = (v0 + c0 + i < a.V) ? z * c2 : kPastV;
          if (x[i] > cm) {
            cm = x[i];
            ci = v0 + c0 + i;
          }
        }
        if (cm == kPastV) continue;  // the whole slice is past V
        float s2 = 0.f, q2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float e = ex2_approx(x[i] - cm);
          s2 += e;
          q2 = fmaf(e, x[i], q2);
        }
        Stat b;  // back to natural units: max u, sum e^(u - max), sum e^(u - max) u
        b.m = cm * kLn2;
        b.s = s2;
        b.q = q2 * kLn2;
        b.i = ci;
        fold(st, b);
      }
      if (tok < a.T) a.part[(size_t)tok * VT2 + vt2] = make_float4(st.m, st.s, st.q, __int_as_float(st.i));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc ? tempty_l1 : tempty_l0);
      acc ^= 1;
      if (acc == 0) aphase ^= 1;
    }
  }

  // Neither CTA leaves (or frees TMEM) while the pair's UMMAs may still read
  // its shared memory or write its TMEM: the leader drained them above.
  tc_fence_before();
  cluster_barrier();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// One CTA per token: fold its VT partials (thread-strided, then a fixed
// tree), so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) lmhead_finalize_kernel(LmHeadArgs a) {
  __shared__ Stat sh[256];
  pdl_wait();
  const int t = blockIdx.x;
  const int VT = (a.V + kPairV - 1) / kPairV;  // partials per token (256-row tiles)
  Stat st;
  st.m = -INFINITY;
  st.s = st.q = 0.f;
  st.i = 0;
  for (int j = threadIdx.x; j < VT; j += 256) {
    const float4 p = a.part[(size_t)t * VT + j];
    Stat b;
    b.m = p.x;
    b.s = p.y;
    b.q = p.z;
    b.i = __float_as_int(p.w);
    fold(st, b);
  }
  sh[threadIdx.x] = st;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      Stat x = sh[threadIdx.x];
      fold(x, sh[threadIdx.x + w]);
      sh[threadIdx.x] = x;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const Stat r = sh[0];
    const float lz = r.m + logf(r.s);
    a.logz[t] = lz;
    a.entropy[t] = fmaxf(lz - r.q / r.s, 0.f);
    a.token[t] = r.i;
  }
  pdl_launch_dependents();
}

// Entropy-bounded acceptance over the masked positions: rank by (H, t),
// then one thread walks the ranks summing entropies in fp64.  Entropies and
// the mask are staged in shared memory first (each rank reads all of them).
__global__ void __launch_bounds__(1024) lmhead_accept_kernel(LmHeadArgs a) {
  extern __shared__ int s_order[];  // [T] position at each rank (-1: none), then H [T], mask [T]
  float* s_h = reinterpret_cast<float*>(s_order + a.T);
  uint8_t* s_m = reinterpret_cast<uint8_t*>(s_h + a.T);
  pdl_wait();
  const int T = a.T;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    s_order[t] = -1;
    s_h[t] = a.entropy[t];
    s_m[t] = a.masked ? (a.masked[t] != 0) : 1;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    a.accept[t] = 0;
    if (!s_m[t]) continue;
    const float ht = s_h[t];
    int rank = 0;
    for (int q = 0; q < T; ++q) {
      const float hs = s_h[q];
      rank += (s_m[q] && (hs < ht || (hs == ht && q < t))) ? 1 : 0;
    }
    s_order[rank] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double below = 0.0;
    for (int r = 0; r < T; ++r) {
      const int t = s_order[r];
      if (t < 0 || below > (double)a.bound) break;
      a.accept[t] = 1;
      below += (double)s_h[t];
    }
  }
}

}  // namespace

}  // namespace moe

cudaError_t moe_launch_lmhead_gemm(const moe::LmHeadArgs& a, const CUtensorMap& tm_w,
                                   const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl) {
  static_assert(moe::kPairSmemBytes <= 232448, "lm_head kernel smem above the sm_100 limit");
  cudaError_t err = cudaFuncSetAttribute(moe::lmhead_gemm_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         moe::kPairSmemBytes);
  if (err != cudaSuccess) return err;
  // as many CTA pairs as can be resident at once (one CTA per SM), but no
  // more than there are units
  static int max_pairs[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && max_pairs[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(moe::kThreads, 1, 1);
    cfg.dynamicSmemBytes = moe::kPairSmemBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, moe::lmhead_gemm_pair_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs[dev] = n > 0 ? n : 1;
  }
  const int VT2 = (a.V + moe::kPairV - 1) / moe::kPairV;
  const int U = VT2 * ((a.T + 2 * moe::kPairTok - 1) / (2 * moe::kPairTok));
  const int pairs = min(min(dev < 64 ? max_pairs[dev] : num_sms / 2, num_sms / 2), U);
  return moe::launch_pdl(moe::lmhead_gemm_pair_kernel, dim3(2 * pairs), dim3(moe::kThreads),
                         (size_t)moe::kPairSmemBytes, s, pdl, tm_w, tm_h, a);
}

cudaError_t moe_launch_lmhead_tail(const moe::LmHeadArgs& a, cudaStream_t s, bool pdl) {
  cudaError_t err = moe::launch_pdl(moe::lmhead_finalize_kernel, dim3(a.T), dim3(256), 0, s, pdl, a);
  if (err != cudaSuccess) return err;
  return moe::launch_pdl(moe::lmhead_accept_kernel, dim3(1), dim3(1024),
                         (size_t)a.T * (sizeof(int) + sizeof(float) + 1), s, pdl, a);
}
