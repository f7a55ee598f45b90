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
//   lmhead_gemm_kernel: persistent, one CTA per SM; a unit is (128-row tile
//     of W, chunk of <= 256 tokens).  Swap-AB as in the expert kernels: W
//     rows are the UMMA M, tokens N, so W streams from HBM once; h is
//     re-read from L2 by every unit.  Warp 0 streams W (TMA, evict-first),
//     warp 6 streams h (evict-last), warp 1 issues the tcgen05 UMMAs into
//     two 256-column TMEM accumulators, warps 2..5 reduce each accumulator:
//     the 128 x 32 tile of a 32-token slice goes through shared memory so
//     that each thread folds 32 rows of one token into (max, sum exp, sum
//     exp * u, argmax); four such partials per token are folded again and
//     written as one float4 per (token, tile).  The logits never reach HBM.
//   lmhead_finalize_kernel: one CTA per token folds its V/128 partials in a
//     fixed order (deterministic) into logZ, H and the argmax.
//   lmhead_accept_kernel: one CTA ranks the masked positions by (H, t) and
//     walks them in that order summing the entropies in fp64.
// Every wait is bounded like the expert kernels' (MOE_ERR_TIMEOUT).
#include "expert_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 224;
constexpr int kMaxA = 12;
constexpr int kMaxB = 6;
constexpr int kRingBytes = 200 * 1024;
constexpr int kABytes = kBM * kBK * 2;    // 16 KB
constexpr int kTileCols = 32;             // tokens per epilogue slice
constexpr int kStatBytes = kBM * (kTileCols + 1) * 4 + 4 * kTileCols * 16;
constexpr int kBarBytes = 8 * (2 * kMaxA + 2 * kMaxB + 4 + 1);
constexpr int kSmemBytes = 1024 + kRingBytes + kStatBytes + kBarBytes + 256;
enum { kWhereLmA = 40, kWhereLmB, kWhereLmMma, kWhereLmEpi };

struct Stat {
  float m, s, q;
  int i;
};

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

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_h, LmHeadArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* tile = reinterpret_cast<float*>(smem + kRingBytes);   // [128][33] u values
  Stat* part = reinterpret_cast<Stat*>(tile + kBM * (kTileCols + 1));  // [4][32]
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + kRingBytes + kStatBytes);
  uint64_t* emptyA = fullA + kMaxA;
  uint64_t* fullB = emptyA + kMaxA;
  uint64_t* emptyB = fullB + kMaxB;
  uint64_t* tfull = emptyB + kMaxB;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_bcast = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  Ctl* ctl = a.ctl;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxA; ++i) {
      mbar_init(&fullA[i], 1);
      mbar_init(&emptyA[i], 1);
    }
    for (int i = 0; i < kMaxB; ++i) {
      mbar_init(&fullB[i], 1);
      mbar_init(&emptyB[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_h);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // h may come from the previous kernel
  pdl_launch_dependents();

  // Units: u = chunk * VT + tile, taken round-robin (they all cost the same).
  const int VT = (a.V + kBM - 1) / kBM;
  const int NC = (a.T + kMaxN - 1) / kMaxN;
  const int U = VT * NC;
  const int nkb = a.d / kBK;
  const int NB = (min(a.T, kMaxN) + kBRows - 1) / kBRows * kBRows;
  const int b_bytes = NB * kBK * 2;
  const int SB = min(kMaxB, max(2, (kRingBytes / 3) / b_bytes));
  const int SA = min(kMaxA, (kRingBytes - SB * b_bytes) / kABytes);
  uint8_t* ringA = ring;
  uint8_t* ringB = ring + SA * kABytes;

  if (warp == 0) {
    // ------------------------------------------------------------ W producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const int vt = u % VT;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyA[stage], phase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmA)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&fullA[stage], kABytes);
          tma_load_2d(ringA + stage * kABytes, &tm_w, kb * kBK, vt * kBM, &fullA[stage], pol_w);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == SA) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s2 = 0; s2 < SA; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&fullA[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ h producer
    if (lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const int ch = u / VT;
        const int n = min(kMaxN, a.T - ch * kMaxN);
        const int nbox = (n + kBRows - 1) / kBRows;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyB[stage], phase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmB)) {
            ok = false;
            break;
          }
          uint8_t* sb = ringB + stage * b_bytes;
          mbar_arrive_expect_tx(&fullB[stage], nbox * kBRows * kBK * 2);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(sb + bx * kBRows * kBK * 2, &tm_h, kb * kBK, ch * kMaxN + bx * kBRows,
                        &fullB[stage], pol_act);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == SB) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s2 = 0; s2 < SB; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&fullB[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      int sa_i = 0, sb_i = 0;
      uint32_t pa = 0, pb = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const int ch = u / VT;
        const int n = min(kMaxN, a.T - ch * kMaxN);
        const uint32_t idesc = idesc_bf16_f32(kBM, (n + 15) & ~15);
        if (!mbar_wait(&tempty[acc], aphase ^ 1, s_abort, ctl, a.timeout_ns, kWhereLmMma)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * kMaxN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&fullA[sa_i], pa, s_abort, ctl, a.timeout_ns, kWhereLmMma) ||
              !mbar_wait(&fullB[sb_i], pb, s_abort, ctl, a.timeout_ns, kWhereLmMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ringA + sa_i * kABytes);
          const uint32_t sb = smem_u32(ringB + sb_i * b_bytes);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma_bf16(dt, sdesc_k_sw128(sa + kk * kUmmaK * 2), sdesc_k_sw128(sb + kk * kUmmaK * 2),
                      idesc, (kb | kk) ? 1u : 0u);
          umma_commit(&emptyA[sa_i]);
          umma_commit(&emptyB[sb_i]);
          if (++sa_i == SA) {
            sa_i = 0;
            pa ^= 1;
          }
          if (++sb_i == SB) {
            sb_i = 0;
            pb ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aphase ^= 1;
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0, ctl, a.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;           // TMEM lane quarter
    const int row = q4 * 32 + lane;    // W row inside the tile (TMEM lane)
    const int et = threadIdx.x - 64;   // 0..127
    const int col = et & 31;           // token inside the slice (reduction phase)
    const int rq = et >> 5;            // row quarter it folds
    int acc = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < U; u += gridDim.x) {
      if (et == 0)
        *s_bcast = mbar_wait(&tfull[acc], aphase, s_abort, ctl, a.timeout_ns, kWhereLmEpi) ? 1 : 0;
      named_barrier(1, 128);
      if (*s_bcast == 0) break;
      tc_fence_after();
      const int vt = u % VT, ch = u / VT;
      const int n = min(kMaxN, a.T - ch * kMaxN);
      const int vrow = vt * kBM + row;
      const bool valid = vrow < a.V;
      const uint32_t tbase = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * kMaxN);
      for (int c0 = 0; c0 < n; c0 += kTileCols) {
        uint32_t v[32];
        tmem_ld32(tbase + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float z = __uint_as_float(v[i]);
          if (a.softcap > 0.f) z = a.softcap * tanhf(z / a.softcap);
          tile[row * (kTileCols + 1) + i] = valid ? z * a.inv_temp : -INFINITY;
        }
        named_barrier(1, 128);
        // thread (rq, col): rows [32 rq, 32 rq + 32) of token column col
        Stat st;
        st.m = -INFINITY;
        st.i = 0;
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
          const float x = tile[(rq * 32 + r) * (kTileCols + 1) + col];
          if (x > st.m) {
            st.m = x;
            st.i = vt * kBM + rq * 32 + r;
          }
        }
        st.s = 0.f;
        st.q = 0.f;
        if (st.m != -INFINITY) {
#pragma unroll 8
          for (int r = 0; r < 32; ++r) {
            const float x = tile[(rq * 32 + r) * (kTileCols + 1) + col];
            if (x != -INFINITY) {  // rows past V (0 * -inf would poison q)
              const float e = expf(x - st.m);
              st.s += e;
              st.q = fmaf(e, x, st.q);
            }
          }
        }
        part[rq * kTileCols + col] = st;
        named_barrier(1, 128);
        if (rq == 0) {
          Stat t = part[col];
          for (int k2 = 1; k2 < 4; ++k2) fold(t, part[k2 * kTileCols + col]);
          const int tok = ch * kMaxN + c0 + col;
          if (c0 + col < n)
            a.part[(size_t)tok * VT + vt] = make_float4(t.m, t.s, t.q, __int_as_float(t.i));
        }
        named_barrier(1, 128);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aphase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// One CTA per token: fold its VT partials (thread-strided, then a fixed
// tree), so the result does not depend on scheduling.
__global__ void __launch_bounds__(256) lmhead_finalize_kernel(LmHeadArgs a) {
  __shared__ Stat sh[256];
  pdl_wait();
  const int t = blockIdx.x;
  const int VT = (a.V + kBM - 1) / kBM;
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
// then one thread walks the ranks summing entropies in fp64.
__global__ void __launch_bounds__(1024) lmhead_accept_kernel(LmHeadArgs a) {
  extern __shared__ int s_order[];  // [T] position at each rank (-1: none)
  pdl_wait();
  const int T = a.T;
  for (int t = threadIdx.x; t < T; t += blockDim.x) s_order[t] = -1;
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    a.accept[t] = 0;
    if (a.masked && !a.masked[t]) continue;
    const float ht = a.entropy[t];
    int rank = 0;
    for (int s = 0; s < T; ++s) {
      if (a.masked && !a.masked[s]) continue;
      const float hs = a.entropy[s];
      rank += (hs < ht || (hs == ht && s < t)) ? 1 : 0;
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
      below += (double)a.entropy[t];
    }
  }
}

}  // namespace

}  // namespace moe

cudaError_t moe_launch_lmhead_gemm(const moe::LmHeadArgs& a, const CUtensorMap& tm_w,
                                   const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl) {
  static_assert(moe::kSmemBytes <= 232448, "lm_head kernel smem above the sm_100 limit");
  cudaError_t err = cudaFuncSetAttribute(moe::lmhead_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         moe::kSmemBytes);
  if (err != cudaSuccess) return err;
  const int VT = (a.V + moe::kBM - 1) / moe::kBM;
  const int U = VT * ((a.T + moe::kMaxN - 1) / moe::kMaxN);
  return moe::launch_pdl(moe::lmhead_gemm_kernel, dim3(min(num_sms, U)), dim3(moe::kThreads),
                         (size_t)moe::kSmemBytes, s, pdl, tm_w, tm_h, a);
}

cudaError_t moe_launch_lmhead_tail(const moe::LmHeadArgs& a, cudaStream_t s, bool pdl) {
  cudaError_t err = moe::launch_pdl(moe::lmhead_finalize_kernel, dim3(a.T), dim3(256), 0, s, pdl, a);
  if (err != cudaSuccess) return err;
  return moe::launch_pdl(moe::lmhead_accept_kernel, dim3(1), dim3(1024),
                         (size_t)a.T * sizeof(int), s, pdl, a);
}
