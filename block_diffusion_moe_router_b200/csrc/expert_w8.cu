// expert_w8.cu -- grouped expert GEMMs with 8-bit floating-point expert
// weights: OFP8 E4M3 codes (OCP 8-bit Floating Point Specification) with one
// fp32 scale per weight row.  The Hugging Face card
// "kingjones777/DiffusionGemma-26B-A4B-it-ROCmFP4-GGUF" ships FP4 / FP8
// builds of these weights and finds that, at a 256-token canvas, the 8-bit
// build steps faster than the 4-bit one.
//
// Same work units, scheduler, unit ring, B operands and epilogue as the bf16
// and int4 kernels; the A operand (weights) is decoded in TMEM:
//   - a code producer brings each 128-wide K stage of codes (128 rows x 128
//     bytes, 128-byte swizzled) into a ring of its own by TMA; a B producer
//     brings the matching activation tiles into a second ring.  A code stage
//     is free again as soon as the dequant warps hold it in registers, so
//     the code ring, which carries the HBM stream, is not held up by the
//     UMMAs (a shared ring kept each stage ~3x longer and the stream at
//     ~1,150 cycles per stage, latency-bound);
//   - 8 dequant warps widen the codes with the hardware E4M3 -> f16x2
//     conversion (exact: every E4M3 value is an fp16 value) and store the
//     fp16 pairs straight into TMEM (tcgen05.st), one stage per group, both
//     stages of a pair per hand-over;
//   - the UMMA (kind::f16 with A and B both fp16) reads A from TMEM and the
//     activations from shared memory: on this path x_perm and h are fp16;
//   - the epilogue multiplies each accumulator row by its weight row's fp32
//     scale before GELU-tanh(gate) * up (gate_up) or before writing y (down).
// A unit's 128 row scales come in by bulk copy into the unit's slot when the
// code producer publishes the unit.  Per weight the SM moves one byte through
// shared memory and two bytes into TMEM, with one conversion per two weights.
//
// TMEM (512 columns): two 128-column fp32 accumulators (a unit holds at most
// 128 tokens) and two A slots of 128 columns (two K stages each).

#include "expert_common.cuh"

namespace moe {

namespace {

// warps: 0 code producer, 1 UMMA (partial 0), 2-5 epilogue, 6-13 dequant,
// 14 B producer, 15 UMMA (partial 1)
constexpr int kThreads = 512;
constexpr int kDqWarp0 = 6;
constexpr int kDqGroups = 2;              // dequant groups, each owning one stage of every pair
constexpr int kDqWarps = 4 * kDqGroups;   // a group is one warp per TMEM lane quarter
constexpr int kBWarp = kDqWarp0 + kDqWarps;
constexpr int kMmaWarp2 = kBWarp + 1;
constexpr int kChunkN = 128;                 // tokens per unit
constexpr int kBK8 = 128;                    // K per stage
constexpr int kCodeBytes = kBM * kBK8;       // 16 KB of codes per stage
// TMEM A: two slots, each holding a pair of consecutive 128-wide K stages
// (2 x 64 columns of f16x2).  The UMMA issuer and the dequant warps hand A
// over once per pair: half the barrier round trips of one per stage.
constexpr int kASlots = 2;
constexpr int kACols = kBK8 / 2;             // 64 columns of f16x2 per K stage
constexpr int kASlotCols = 2 * kACols;
constexpr int kAColBase = 2 * kChunkN;       // A slots after the accumulators
constexpr int kMaxCS = 10;                   // code stages
constexpr int kMaxBS = 6;                    // B stages
constexpr int kRingBytes = 192 * 1024;       // code ring + B ring
// One row-scale slot per unit-ring entry: the unit's 128 fp32 row scales
// (gate rows then up rows for gate_up, as the TMEM lanes hold them).
constexpr int kScaleSlot = kBM * 4;
constexpr int kScaleBytes = kUnitRing * kScaleSlot;
constexpr int kBarBytes = 8 * (2 * kMaxCS + 2 * kMaxBS + 2 * kASlots + 4 + 3 * kUnitRing + 3);
constexpr int kSmemBytes =
    1024 + kRingBytes + kScaleBytes + kEpiBytes + kBarBytes + 256;
static_assert(kAColBase + kASlots * kASlotCols <= kTmemCols, "TMEM budget");

enum { kWhereAFull = 20, kWhereAEmpty, kWhereDqFull, kWhereBFull };

// Instruction descriptor, kind::f16 with fp16 A and B (formats 0), fp32 D:
// [4,6) D format = 1 (f32), [7,10) A = 0, [10,13) B = 0, K-major both,
// [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory (16-byte aligned
// addresses, size a multiple of 16), completing `bytes` on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// One lane of a converged warp, chosen by elect.sync (the lowest active
// lane, so the same lane every time the whole warp is active).  The UMMA
// issuer runs with the whole warp converged and lets the elected lane issue
// each tcgen05 instruction, which keeps the descriptor arithmetic
// warp-uniform (measured: 72 instead of 93 cycles per UMMA with A in TMEM).
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\t"
      "elect.sync rx|px, 0xffffffff;\n\t"
      "@px mov.u32 %0, 1;\n\t}"
      : "+r"(pred));
  return pred != 0;
}

// umma_commit from the elected lane (the lane that issued the UMMAs).
__device__ __forceinline__ void umma_commit_elect(uint64_t* bar) {
  if (elect_one()) umma_commit(bar);
}

// mbar_wait by every lane of a warp; the verdict is the same in all lanes.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity,
                                               volatile int* abort, Ctl* ctl,
                                               uint64_t timeout_ns, int where) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, ctl, timeout_ns, where)) != 0;
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 inputs (per the instruction
// descriptor), fp32 accumulate.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Four E4M3 codes (byte i = element i) -> two f16x2 words holding elements
// (0,1) and (2,3), the lower element in the lower half (the hardware
// conversion widens the two bytes of a 16-bit half in place).
__device__ __forceinline__ void widen4(uint32_t w, uint32_t* out) {
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(out[0]), "=r"(out[1])
      : "r"(w));
}

__global__ void __launch_bounds__(kThreads, 1)
    expert_w8_kernel(const __grid_constant__ CUtensorMap tm_cgu,
                     const __grid_constant__ CUtensorMap tm_cd,
                     const __grid_constant__ CUtensorMap tm_xp,
                     const __grid_constant__ CUtensorMap tm_h, ExpertArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;  // [CS code stages][BS B stages]
  float* rsc = reinterpret_cast<float*>(smem + kRingBytes);  // [kUnitRing][128] row scales
  float* xchg = reinterpret_cast<float*>(smem + kRingBytes + kScaleBytes);
  uint64_t* cfull = reinterpret_cast<uint64_t*>(smem + kRingBytes + kScaleBytes + kEpiBytes);
  uint64_t* cempty = cfull + kMaxCS;
  uint64_t* bfull = cempty + kMaxCS;
  uint64_t* bempty = bfull + kMaxBS;
  uint64_t* afull = bempty + kMaxBS;
  uint64_t* aempty = afull + kASlots;
  uint64_t* tfull = aempty + kASlots;
  uint64_t* tempty = tfull + 2;
  uint64_t* ufull = tempty + 2;
  uint64_t* uempty = ufull + kUnitRing;
  uint64_t* sfull = uempty + kUnitRing;  // the unit's row scales have landed
  uint64_t* drain = sfull + kUnitRing;
  uint64_t* uend = drain + 2;  // both UMMA warps are done with a unit's A slots
  UnitInfo* units = reinterpret_cast<UnitInfo*>(drain + 3);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(units + kUnitRing);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_bcast = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* s_dqbc = reinterpret_cast<volatile int*>(tmem_slot + 3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int GU = a.f / kGuHalf;
  const int DN = a.d / kBM;
  Ctl* ctl = a.ctl;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxCS; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], 4);  // the dequant group's four warps hold the codes
    }
    for (int i = 0; i < kMaxBS; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);  // UMMA commit
    }
    for (int i = 0; i < kASlots; ++i) {
      mbar_init(&afull[i], 8);  // both dequant groups' warps (one stage each)
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 2);  // one commit from each UMMA warp
      mbar_init(&tempty[i], 4);
    }
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&ufull[i], 1);
      // both UMMA warps, epilogue leader, B producer and every dequant warp
      mbar_init(&uempty[i], 4 + kDqWarps);
      mbar_init(&sfull[i], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(uend, 2);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_cgu);
    tma_prefetch_desc(&tm_cd);
    tma_prefetch_desc(&tm_xp);
    tma_prefetch_desc(&tm_h);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();

  const int maxn = max(1, min(kChunkN, ctl->max_chunk));
  const int NB = (maxn + kBRows - 1) / kBRows * kBRows;
  const int b_bytes = 4 * NB * kBK * 2;  // a stage pair: four 64-wide B sub-tiles of NB rows
  const int BS = min(kMaxBS, max(2, (kRingBytes / 3) / b_bytes));
  const int CS = min(kMaxCS, (kRingBytes - BS * b_bytes) / kCodeBytes);
  uint8_t* ringB = ring + CS * kCodeBytes;
  const int n_chunks = ctl->n_chunks;
  const int U = n_chunks * (GU + DN);

  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    // Claims and publishes the units (with their row scales), then streams
    // each unit's codes.
    const uint64_t pol_w = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    int ur = 0;
    uint32_t uphase = 0;
    uint32_t issued = 0, issued_par = 0;
    uint32_t sissued = 0, spar = 0;  // scale slots with a copy issued, and its parity
    // The first unit of CTA b is unit b; later ones come from the counter
    // (offset by the grid), so every unit is claimed exactly once.  The next
    // claim is issued as soon as a unit is taken, so the atomic's round trip
    // overlaps this unit's copies.
    int u_next = (int)blockIdx.x;
    while (true) {
      UnitInfo ui;
      ui.type = kUnitStop;
      ui.e = ui.m = ui.n = ui.slot0 = ui.q = 0;
      int go = 0;
      if (lane == 0 && !*s_abort) {
        go = 1;
        const int u = u_next;
        if (u < U) u_next = (int)gridDim.x + atomicAdd(&ctl->work_next, 1);
        if (u < U) {
          int q, m;
          if (u < n_chunks * GU) {
            ui.type = kUnitGateUp;
            q = u / GU;
            m = u - q * GU;
          } else {
            const int v = u - n_chunks * GU;
            ui.type = kUnitDown;
            q = v / DN;
            m = v - q * DN;
          }
          const int4 ci = a.chunk_info[q];  // one load: expert, first slot, tokens
          ui.e = ci.x;
          ui.m = m;
          ui.q = q;
          ui.slot0 = ci.y;
          ui.n = ci.z;
          if (ui.n < 1 || ui.n > NB) {
            record_error(ctl, MOE_ERR_DEVICE_CHECK, 201);
            *s_abort = 1;
            go = 0;
          }
        }
        if (go && mbar_wait(&uempty[ur], uphase ^ 1, s_abort, ctl, a.timeout_ns,
                            kWhereUnitEmpty)) {
          if (ui.type != kUnitStop) {
            // the unit's 128 row scales into its slot by bulk copy (the
            // gate and up blocks are 64 contiguous fp32 each: 256 bytes at
            // 256-byte offsets; a down block is 512 bytes)
            float* slot = rsc + ur * kBM;
            if (ui.type == kUnitGateUp) {
              const size_t r0 = (size_t)ui.e * 2 * a.f + (size_t)ui.m * kGuHalf;
              mbar_arrive_expect_tx(&sfull[ur], kGuHalf * 4 * 2);
              bulk_g2s(slot, a.rows_gu + r0, kGuHalf * 4, &sfull[ur]);
              bulk_g2s(slot + kGuHalf, a.rows_gu + r0 + a.f, kGuHalf * 4, &sfull[ur]);
            } else {
              const size_t r0 = (size_t)ui.e * a.d + (size_t)ui.m * kBM;
              mbar_arrive_expect_tx(&sfull[ur], kBM * 4);
              bulk_g2s(slot, a.rows_d + r0, kBM * 4, &sfull[ur]);
            }
            sissued |= 1u << ur;
            spar = (spar & ~(1u << ur)) | (uphase << ur);
          }
          units[ur] = ui;
          mbar_arrive(&ufull[ur]);
        } else {
          go = 0;
        }
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      ui.type = __shfl_sync(0xffffffffu, ui.type, 0);
      ui.e = __shfl_sync(0xffffffffu, ui.e, 0);
      ui.m = __shfl_sync(0xffffffffu, ui.m, 0);
      if (!go || ui.type == kUnitStop) break;
      if (++ur == kUnitRing) {
        ur = 0;
        uphase ^= 1;
      }
      int ok = 1;
      if (lane == 0) {
        const int C = (ui.type == kUnitGateUp) ? a.d : a.f;
        const int nkb = (C + kBK8 - 1) / kBK8;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&cempty[stage], phase ^ 1, s_abort, ctl, a.timeout_ns,
                         kWhereStageEmpty)) {
            ok = 0;
            break;
          }
          uint8_t* sa = ring + stage * kCodeBytes;
          mbar_arrive_expect_tx(&cfull[stage], kCodeBytes);
          const int cx = kb * kBK8;  // byte column of the codes
          if (ui.type == kUnitGateUp) {
            const int r0 = ui.e * 2 * a.f + ui.m * kGuHalf;
            tma_load_2d(sa, &tm_cgu, cx, r0, &cfull[stage], pol_w);
            tma_load_2d(sa + kCodeBytes / 2, &tm_cgu, cx, r0 + a.f, &cfull[stage], pol_w);
          } else {
            tma_load_2d(sa, &tm_cd, cx, ui.e * a.d + ui.m * kBM, &cfull[stage], pol_w);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == CS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    if (lane == 0) {
      for (int s2 = 0; s2 < CS; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&cfull[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
      for (int s2 = 0; s2 < kUnitRing; ++s2)
        if ((sissued >> s2) & 1u)
          mbar_wait_drain(&sfull[s2], (spar >> s2) & 1u, ctl, a.timeout_ns);
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------------------ B producer
    // Follows the unit ring; a down unit's h tiles wait for every gate_up
    // unit of the chunk (the codes of the down unit stream meanwhile).
    if (lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int ur = 0;
      uint32_t uphase = 0;
      uint32_t issued = 0, issued_par = 0;
      while (true) {
        if (!mbar_wait(&ufull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereUnitFullB)) break;
        const UnitInfo ui = units[ur];
        if (ui.type == kUnitStop) break;
        if (ui.type == kUnitDown) {
          const int need = GU + (a.test_stall ? (1 << 30) : 0);
          if (!wait_count(a.ready + ui.q, need, s_abort, ctl, a.timeout_ns, kWhereReady)) break;
          fence_proxy_async_global();
        }
        const int C = (ui.type == kUnitGateUp) ? a.d : a.f;
        const int nkb = (C + kBK8 - 1) / kBK8;
        const int nbox = (ui.n + kBRows - 1) / kBRows;
        const CUtensorMap* tb = (ui.type == kUnitGateUp) ? &tm_xp : &tm_h;
        bool ok = true;
        for (int kb0 = 0; kb0 < nkb; kb0 += 2) {  // one B stage per K-stage pair
          const int nst = min(2, nkb - kb0);
          if (!mbar_wait(&bempty[stage], phase ^ 1, s_abort, ctl, a.timeout_ns,
                         kWhereStageEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sb = ringB + stage * b_bytes;
          mbar_arrive_expect_tx(&bfull[stage], nst * 2 * nbox * kBRows * kBK * 2);
          for (int t = 0; t < 2 * nst; ++t)  // 64-wide sub-tiles
            for (int bx = 0; bx < nbox; ++bx)
              tma_load_2d(sb + t * NB * kBK * 2 + bx * kBRows * kBK * 2, tb, kb0 * kBK8 + t * kBK,
                          ui.slot0 + bx * kBRows, &bfull[stage], pol_act);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == BS) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mbar_arrive(&uempty[ur]);
        if (++ur == kUnitRing) {
          ur = 0;
          uphase ^= 1;
        }
      }
      for (int s2 = 0; s2 < BS; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&bfull[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
    }
  } else if (warp == 1 || warp == kMmaWarp2) {
    // ------------------------------------------------------------ UMMA issuers
    // Each warp runs the loop whole (warp-uniform descriptors); the elected
    // lane issues the tcgen05 instructions.  An UMMA costs its issuing warp
    // ~70-110 cycles whatever N is (small N here), and issuers in different
    // warps overlap, so two warps split K: for a unit of at most 64 tokens
    // with two or more stage pairs, warp 1 takes the even pairs into columns
    // [0, 64) of the accumulator and warp 15 the odd ones into [64, 128); the
    // epilogue adds the two partials.  Larger units stay with warp 1.
    // A slot s serves the pairs of global index = s (mod 2) and its full
    // barrier is waited for by parity, so a warp that takes a slot over from
    // the other must not run two phases ahead of it: at the end of every
    // unit both warps meet on `uend` (a bounded wait), after the old owner has
    // passed its last wait on each slot.
    const int mw = warp == 1 ? 0 : 1;
    uint32_t eph = 0;
    int bst = 0;
    uint32_t bph = 0;
    int asl = 0;
    uint32_t aph = 0;
    int ur = 0;
    uint32_t uphase = 0;
    int acc = 0;
    uint32_t aphase = 0;
    while (true) {
      if (!mbar_wait_warp(&ufull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereUnitFullMma)) break;
      const UnitInfo ui = units[ur];
      if (ui.type == kUnitStop) break;
      const int C = (ui.type == kUnitGateUp) ? a.d : a.f;
      const int nkb = (C + kBK8 - 1) / kBK8;
      const int N = (ui.n + 15) & ~15;
      const uint32_t idesc = idesc_f16_f32(kBM, N);
      if (!mbar_wait_warp(&tempty[acc], aphase ^ 1, s_abort, ctl, a.timeout_ns, kWhereTmemEmpty))
        break;
      tc_fence_after();
      const bool split = ui.n <= kChunkN / 2 && nkb > 2;
      const uint32_t dt = tmem_base + (uint32_t)(acc * kChunkN) + (split && mw ? kChunkN / 2 : 0);
      bool ok = true;
      uint32_t first = 1;  // the next UMMA of this warp is its first of the unit
      // one hand-over per K-stage pair: its A slot (dequant warps, which
      // also waited for the pair's B stage) and its B stage
      for (int kb0 = 0; kb0 < nkb; kb0 += 2) {
        const int nst = min(2, nkb - kb0);
        const bool mine = split ? ((kb0 >> 1) & 1) == mw : mw == 0;
        if (!mine) {  // the other warp's pair: keep the ring positions in step
          if (++bst == BS) {
            bst = 0;
            bph ^= 1;
          }
          if (++asl == kASlots) {
            asl = 0;
            aph ^= 1;
          }
          continue;
        }
        if (!mbar_wait_warp(&afull[asl], aph, s_abort, ctl, a.timeout_ns, kWhereAFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sb = smem_u32(ringB + bst * b_bytes);
        const uint32_t ta = tmem_base + (uint32_t)(kAColBase + asl * kASlotCols);
        for (int t = 0; t < nst; ++t) {
#pragma unroll
          for (int kk = 0; kk < kBK8 / kUmmaK; ++kk) {
            const uint32_t b = sb + (2 * t + (kk >> 2)) * NB * kBK * 2 + (kk & 3) * kUmmaK * 2;
            if (elect_one())
              umma_f16_ts(dt, ta + t * kACols + kk * (kUmmaK / 2), sdesc_k_sw128(b), idesc,
                          (first && t == 0 && kk == 0) ? 0u : 1u);
          }
        }
        first = 0;
        umma_commit_elect(&bempty[bst]);
        umma_commit_elect(&aempty[asl]);
        if (++bst == BS) {
          bst = 0;
          bph ^= 1;
        }
        if (++asl == kASlots) {
          asl = 0;
          aph ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) mbar_arrive(uend);
      if (!mbar_wait_warp(uend, eph, s_abort, ctl, a.timeout_ns, kWhereAFull)) break;
      eph ^= 1;
      umma_commit_elect(&tfull[acc]);
      if (lane == 0) mbar_arrive(&uempty[ur]);
      if (++ur == kUnitRing) {
        ur = 0;
        uphase ^= 1;
      }
      acc ^= 1;
      if (acc == 0) aphase ^= 1;
    }
    umma_commit_elect(&drain[mw]);
    if (lane == 0) mbar_wait_drain(&drain[mw], 0, ctl, a.timeout_ns);
    __syncwarp();
  } else if (warp < kDqWarp0) {
    epilogue_role<true, __half>(a, units, ufull, uempty, tfull, tempty, xchg, s_abort, s_bcast,
                                tmem_base, kChunkN, warp, lane, sfull, rsc, 2 * kBK8);
  } else {
    // ------------------------------------------------------------ dequant warps
    // Group g (one warp per TMEM lane quarter) takes the stages kb % 2 == g
    // of each unit, a whole 128-code row per thread, so the two stages of a
    // pair are widened at once; the pair's A slot is signalled full once both
    // groups' stores have landed (eight arrivals; for a last pair of one
    // stage group 1 arrives without data).
    const int dw = warp - kDqWarp0;        // 0..kDqWarps-1
    const int q4 = warp & 3;               // TMEM lane quarter
    const int row = q4 * 32 + lane;        // A row == TMEM lane
    const int grp = dw >> 2;
    const int dt = threadIdx.x - kDqWarp0 * 32;
    const int sw = row & 7;
    int stage = 0;
    uint32_t phase = 0;
    int asl = 0;
    uint32_t aph = 0;
    int bst = 0;  // the pair's B stage: waited for before the hand-over
    uint32_t bph = 0;
    int ur = 0;
    uint32_t uphase = 0;
    while (true) {
      if (dt == 0) {
        const bool ok = mbar_wait(&ufull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereDqFull);
        *s_dqbc = ok ? 1 : 0;
      }
      named_barrier(2, kDqWarps * 32);
      const bool uok = *s_dqbc != 0;
      const UnitInfo ui = units[ur];
      named_barrier(2, kDqWarps * 32);
      if (!uok || ui.type == kUnitStop) break;
      const int C = ui.type == kUnitGateUp ? a.d : a.f;
      const int G = (C + kBK8 - 1) / kBK8;
      bool sok = true;
      for (int kb = 0; kb < G; ++kb) {
        const bool pair_end = (kb & 1) || kb == G - 1;
        if ((kb & 1) != grp && sok && grp == 1 && kb == G - 1) {
          // a last pair of one stage: group 1 has nothing to decode but its
          // four arrivals still complete the pair's hand-over, in its phase
          sok = mbar_wait(&aempty[asl], aph ^ 1, s_abort, ctl, a.timeout_ns, kWhereAEmpty) &&
                mbar_wait(&bfull[bst], bph, s_abort, ctl, a.timeout_ns, kWhereBFull);
          __syncwarp();
          if (lane == 0 && sok) mbar_arrive(&afull[asl]);
        }
        if ((kb & 1) == grp && sok) {
          sok = mbar_wait(&aempty[asl], aph ^ 1, s_abort, ctl, a.timeout_ns, kWhereAEmpty);
          sok = sok && mbar_wait(&cfull[stage], phase, s_abort, ctl, a.timeout_ns, kWhereDqFull);
          if (sok) {
            // codes tile: 128-byte rows written by TMA with 128-byte
            // swizzling, i.e. 16-byte chunk c of row r sits at chunk c ^ (r & 7)
            const uint8_t* crow = ring + stage * kCodeBytes + row * kBK8;
            uint4 cw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
              cw[c] = *reinterpret_cast<const uint4*>(crow + ((c ^ sw) << 4));
            __syncwarp();
            if (lane == 0) mbar_arrive(&cempty[stage]);  // codes are in registers
            const uint32_t ta = tmem_base + ((uint32_t)(q4 * 32) << 16) +
                                (uint32_t)(kAColBase + asl * kASlotCols + (kb & 1) * kACols);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t v[32];  // columns 32h .. 32h+31 = codes 64h .. 64h+63
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                widen4(cw[4 * h + c].x, v + 8 * c + 0);
                widen4(cw[4 * h + c].y, v + 8 * c + 2);
                widen4(cw[4 * h + c].z, v + 8 * c + 4);
                widen4(cw[4 * h + c].w, v + 8 * c + 6);
              }
              tmem_st32(ta + h * 32, v);
            }
            {  // the pair is handed to the UMMA once both groups' stores land
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              sok = mbar_wait(&bfull[bst], bph, s_abort, ctl, a.timeout_ns, kWhereBFull);
              if (lane == 0 && sok) mbar_arrive(&afull[asl]);
            }
          }
        }
        if (++stage == CS) {
          stage = 0;
          phase ^= 1;
        }
        if (pair_end) {
          if (++asl == kASlots) {
            asl = 0;
            aph ^= 1;
          }
          if (++bst == BS) {
            bst = 0;
            bph ^= 1;
          }
        }
      }
      if (lane == 0) mbar_arrive(&uempty[ur]);  // this unit's slot is free
      if (++ur == kUnitRing) {
        ur = 0;
        uphase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

}  // namespace moe

cudaError_t moe_launch_expert_w8(const moe::ExpertArgs& a, const CUtensorMap& tm_cgu,
                                 const CUtensorMap& tm_cd, const CUtensorMap& tm_xp,
                                 const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl) {
  static_assert(moe::kSmemBytes <= 232448, "fp8 expert kernel smem above the sm_100 limit");
  cudaError_t err = cudaFuncSetAttribute(moe::expert_w8_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         moe::kSmemBytes);
  if (err != cudaSuccess) return err;
  return moe::launch_pdl(moe::expert_w8_kernel, dim3(num_sms), dim3(moe::kThreads),
                         (size_t)moe::kSmemBytes, s, pdl, tm_cgu, tm_cd, tm_xp, tm_h, a);
}
