// expert_common.cuh -- pieces shared by the bf16, int4 and fp8 expert
// kernels: the work-unit record, bounded waits, GELU-tanh and the epilogue
// role (TMEM accumulators -> h = gelu(gate) * up in bf16 or fp16, or y).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kXchgStride = 33;  // floats per exchanged row (bank-conflict padding)
// Epilogue scratch: the gate/up exchange rows, then a [32 tokens x 128
// columns] bf16 tile through which h and y are written out as 16-byte rows.
constexpr int kXchgBytes = 64 * kXchgStride * 4;
constexpr int kTileBytes = 32 * 128 * 2;
constexpr int kEpiBytes = kXchgBytes + kTileBytes;
constexpr int kUnitRing = 4;     // work units in flight between the roles

enum { kUnitGateUp = 0, kUnitDown = 1, kUnitStop = -1 };

struct UnitInfo {
  int type;
  int e;      // expert
  int m;      // row tile inside the expert's weight
  int n;      // tokens in this chunk (1..256)
  int slot0;  // first slot of the chunk
  int q;      // chunk index (scheduler table)
};

enum {
  kWhereUnitEmpty = 1,
  kWhereStageEmpty,
  kWhereReady,
  kWhereUnitFullMma,
  kWhereTmemEmpty,
  kWhereStageFull,
  kWhereUnitFullEpi,
  kWhereTmemFull,
  kWhereDrain,
  kWhereUnitFullB,
  kWhereScalesEpi
};

// GELU, tanh form: 0.5 g (1 + tanh( sqrt(2/pi) (g + 0.044715 g^3) )), with
// the hardware tanh (tanh.approx.f32, relative error about 2^-11 per the PTX
// ISA): h is rounded to bf16 (2^-8) right after, so where the gate is
// positive the approximation adds at most an eighth of that rounding (where
// it is negative, gelu is small in absolute terms), and the epilogue of
// every gate_up unit is shorter than with the libm tanh (canvas layer 4 us,
// encode layer 6 us faster).
__device__ __forceinline__ float gelu_tanh(float g) {
  const float c = 0.7978845608028654f;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(c * fmaf(0.044715f * g, g * g, g)));
  return 0.5f * g * (1.f + t);
}

// Spin until *p >= need (acquire), bounded like mbar_wait.
__device__ inline bool wait_count(const int* p, int need, volatile int* abort, Ctl* ctl,
                           uint64_t timeout_ns, int where) {
  if (ld_acquire_gpu(p) >= need) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      __nanosleep(64);
      if (ld_acquire_gpu(p) >= need) return true;
    }
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_error(ctl, MOE_ERR_TIMEOUT, where);
      *abort = 1;
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ inline bool mbar_wait_drain(uint64_t* bar, uint32_t parity, Ctl* ctl, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_error(ctl, MOE_ERR_TIMEOUT, kWhereDrain);
      return false;
    }
  }
  return true;
}

// h in the epilogue's output type.
template <typename HT>
__device__ __forceinline__ HT to_h(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 to_h<__nv_bfloat16>(float v) {
  return __float2bfloat16(v);
}
template <>
__device__ __forceinline__ __half to_h<__half>(float v) {
  return __float2half_rn(v);
}

// v += the fp32 accumulator columns at taddr (a second split-K partial).
__device__ __forceinline__ void add_partial(uint32_t taddr, uint32_t (&v)[32]) {
  uint32_t w[32];
  tmem_ld32(taddr, w);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
}

// Epilogue role (warps 2..5, 128 threads): for each unit, read the fp32
// accumulator from TMEM (lane = weight row, column = token), 32 tokens at a
// time, and write
//   gate_up: h[slot][m*64 + r] = gelu_tanh(gate_r) * up_r  (lane r pairs
//            with lane 64 + r through smem), bf16;
//   down:    y[slot][m*128 + r], bf16 (or fp32 when y_bf16 is off).
// The bf16 values are transposed through a smem tile so that every global
// store is a 16-byte piece of one token's row (coalesced rows instead of
// 2-byte column scatters).  The leader does the waits and broadcasts the
// outcome, so the 128 threads always pass the same named barriers.
// kRowScale (fp8 weights): every accumulator row is first multiplied by its
// weight row's fp32 scale, read from the unit's slot rscale + 128 * ur
// (landed on sfull[ur]); HT is h's type (fp16 on that path).  The units
// rotate over `nbuf` accumulators of acc_cols columns each (tfull / tempty
// per accumulator).
template <bool kRowScale = false, typename HT = __nv_bfloat16>
__device__ __forceinline__ void epilogue_role(const ExpertArgs& a, const UnitInfo* units,
                                              uint64_t* ufull, uint64_t* uempty, uint64_t* tfull,
                                              uint64_t* tempty, float* xchg,
                                              volatile int* s_abort, volatile int* s_bcast,
                                              uint32_t tmem_base, int acc_cols, int warp,
                                              int lane, uint64_t* sfull = nullptr,
                                              const float* rscale = nullptr,
                                              int split_kpair = 0, int nbuf = 2) {
  Ctl* ctl = a.ctl;
  __nv_bfloat16* tile =
      reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(xchg) + kXchgBytes);
  HT* htile = reinterpret_cast<HT*>(tile);
  HT* hout = reinterpret_cast<HT*>(a.h);
  const uint64_t pol_keep = l2_policy_evict_last();  // h and y are read back soon
  const int q4 = warp & 3;          // TMEM lane quarter this warp may access
  const int row = q4 * 32 + lane;   // accumulator row (TMEM lane)
  const int et = threadIdx.x - 64;  // 0..127
  int ur = 0;
  uint32_t uphase = 0;
  int acc = 0;
  uint32_t aphase = 0;
  while (true) {
    // The leader waits; the decision is broadcast so the 128 threads always
    // take the same path through the named barriers below.
    if (et == 0) {
      bool ok = mbar_wait(&ufull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereUnitFullEpi);
      if (ok && units[ur].type != kUnitStop)
        ok = mbar_wait(&tfull[acc], aphase, s_abort, ctl, a.timeout_ns, kWhereTmemFull);
      if (kRowScale && ok && units[ur].type != kUnitStop)
        ok = mbar_wait(&sfull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereScalesEpi);
      *s_bcast = ok ? 1 : 0;
    }
    named_barrier(1, 128);
    const bool ok = *s_bcast != 0;
    const UnitInfo ui = units[ur];
    named_barrier(1, 128);
    if (!ok || ui.type == kUnitStop) break;
    tc_fence_after();
    const float rs = kRowScale ? rscale[ur * kBM + row] : 1.f;
    const uint32_t tbase = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * acc_cols);
    const int nch = (ui.n + 31) / 32;
    // Split K (kernels with two UMMA issuers, split_kpair = the K width of a
    // stage pair): a unit of at most acc_cols / 2 tokens spanning two or more
    // pairs is accumulated in two partials, acc_cols / 2 columns apart, which
    // are summed here.
    const int Ck = ui.type == kUnitGateUp ? a.d : a.f;
    const bool split = split_kpair > 0 && ui.n <= acc_cols / 2 && Ck > split_kpair;
    const uint32_t poff = (uint32_t)(acc_cols / 2);
    if (ui.type == kUnitGateUp) {
      for (int cc = 0; cc < nch; ++cc) {
        uint32_t v[32];
        tmem_ld32(tbase + cc * 32, v);
        tmem_wait_ld();
        if (split) add_partial(tbase + poff + cc * 32, v);
        if (row >= kGuHalf) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            xchg[(row - kGuHalf) * kXchgStride + i] =
                kRowScale ? __uint_as_float(v[i]) * rs : __uint_as_float(v[i]);
        }
        named_barrier(1, 128);
        const int cmax = min(32, ui.n - cc * 32);
        if (row < kGuHalf) {  // tile[token][r], 64 columns
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = kRowScale ? __uint_as_float(v[i]) * rs : __uint_as_float(v[i]);
            const float up = xchg[row * kXchgStride + i];
            htile[i * kGuHalf + row] = to_h<HT>(gelu_tanh(g) * up);
          }
        }
        named_barrier(1, 128);
        // 32 tokens x 128 bytes: eight 16-byte pieces per token
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int pc = et + 128 * k;
          const int tok = pc >> 3, piece = pc & 7;
          if (tok < cmax)
            st_global_hint(hout + (size_t)(ui.slot0 + cc * 32 + tok) * a.f + ui.m * kGuHalf +
                               piece * 8,
                           *reinterpret_cast<const uint4*>(htile + tok * kGuHalf + piece * 8),
                           pol_keep);
        }
      }
    } else {
      const size_t y0 = (size_t)ui.slot0 * a.d + ui.m * kBM;
      for (int cc = 0; cc < nch; ++cc) {
        uint32_t v[32];
        tmem_ld32(tbase + cc * 32, v);
        tmem_wait_ld();
        if (split) add_partial(tbase + poff + cc * 32, v);
        const int cmax = min(32, ui.n - cc * 32);
        if (a.y_bf16) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            tile[i * kBM + row] =
                __float2bfloat16(kRowScale ? __uint_as_float(v[i]) * rs : __uint_as_float(v[i]));
          named_barrier(1, 128);
          // 32 tokens x 256 bytes: sixteen 16-byte pieces per token
          __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y) + y0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int pc = et + 128 * k;
            const int tok = pc >> 4, piece = pc & 15;
            if (tok < cmax)
              st_global_hint(y + (size_t)(cc * 32 + tok) * a.d + piece * 8,
                             *reinterpret_cast<const uint4*>(tile + tok * kBM + piece * 8),
                             pol_keep);
          }
          named_barrier(1, 128);
        } else {
          float* ycol = static_cast<float*>(a.y) + y0 + row;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < cmax)
              ycol[(size_t)(cc * 32 + i) * a.d] =
                  kRowScale ? __uint_as_float(v[i]) * rs : __uint_as_float(v[i]);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&tempty[acc]);
    if (ui.type == kUnitGateUp) __threadfence();  // h visible before the chunk counter
    named_barrier(1, 128);
    if (et == 0) {
      if (ui.type == kUnitGateUp) {
        __threadfence();
        fence_proxy_async_global();
        atomicAdd(a.ready + ui.q, 1);
      }
      mbar_arrive(&uempty[ur]);
    }
    if (++ur == kUnitRing) {
      ur = 0;
      uphase ^= 1;
    }
    if (++acc == nbuf) {
      acc = 0;
      aphase ^= 1;
    }
  }
}

}  // namespace moe
