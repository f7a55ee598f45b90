// expert.cu -- grouped expert GEMMs of the MoE FFN on tcgen05 tensor cores.
//
// One persistent kernel runs every (expert, chunk of <= 256 tokens) work unit of both
// projections (auto-round pull request "Add quantization support for
// DiffusionGemma", transformers backend test log: gate_proj / up_proj
// 2816->704, down_proj 704->2816, act GELUTanh; Quant-Tuner pull request,
// "Answers to the motivating questions": one fused 3-D gate_up projection):
//
//   gate_up unit (e, chunk, m): 64 gate rows [m*64, m*64+64) and the 64 up rows
//     [f + m*64, ...) of W_gu[e] are stacked into one 128-row A tile, so a
//     single M=128 UMMA per K step computes both for the chunk's tokens (N);
//     the epilogue pairs TMEM lane r (gate) with lane 64+r (up) and writes
//     h = gelu_tanh(gate) * up in bf16.
//   down unit (e, chunk, m): rows [m*128, m*128+128) of W_d[e] against the
//     chunk's h rows; the epilogue writes y (bf16, or fp32) per slot.
//
// "Swap-AB": weight rows are the UMMA M dimension and the tokens routed to
// the expert are N (16..256), so every weight byte is streamed from HBM once
// per chunk; the plan cuts an expert's tokens into chunks of 128 or 256
// (the host's choice), so at one canvas only a hot expert has two.
//
// Roles (256 threads): warp 0 = scheduler (claims units: its CTA index
// first, then from a global counter) and weight (A) producer, warps 1 and 7
// = UMMA issuers (warp 1 owns the TMEM allocation), warps 2..5 = epilogue
// (TMEM -> registers -> global), warp 6 = activation (B) producer.  One
// issuing thread sustains one M=128 K=16 UMMA per ~90-110 cycles whatever N
// is (below N ~ 180), which at 4 UMMAs per 64-wide K stage is slower than a
// stage's share of the weight stream once the chunks grow past ~100 tokens;
// UMMAs from two threads overlap, so for every unit of at most 128 tokens
// the two issuers split K: warp 1 takes the unit's even K stages and warp 7
// the odd ones, each into its own 128-column partial, and the epilogue adds
// the two partials (fixed order, so the result does not depend on timing).
// A larger unit's partials would not leave TMEM room for a second unit in
// flight, so warp 1 issues it alone into 256 columns.  Weights and activations have rings of their own,
// sized at run time from the largest chunk: the weight ring is deep, since
// its tiles come from HBM and are the bytes the kernel exists to stream,
// while the activation tiles come from L2.  So the weights of a unit keep
// streaming while its activations are still being produced: a down unit's
// W_d tiles are fetched before every gate_up unit of its chunk has published
// h, and only its h tiles wait (per-chunk counter, acquire/release).  TMEM
// (512 columns) holds two units' accumulators (two 128-column partials each
// when K is split, else one of 256 columns), so the epilogue of one unit
// overlaps the MMAs of the next.
//
// Every wait is bounded by %globaltimer; on expiry the kernel records
// MOE_ERR_TIMEOUT, the roles leave their loops, in-flight TMA copies and
// UMMAs are drained (again bounded) and TMEM is released.
#include "expert_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxA = 12;  // weight stages
constexpr int kMaxB = 8;   // activation stages
constexpr int kMinB = 3;  // 2 when rounded down to even
constexpr int kRingBytes = 200 * 1024;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kBarBytes = 8 * (2 * kMaxA + 2 * kMaxB + 4 + 2 * kUnitRing + 3);
constexpr int kSmemBytes = 1024 + kRingBytes + kEpiBytes + kBarBytes + 256;

__global__ void __launch_bounds__(kThreads, 1)
    expert_kernel(const __grid_constant__ CUtensorMap tm_wgu,
                  const __grid_constant__ CUtensorMap tm_wd,
                  const __grid_constant__ CUtensorMap tm_xp,
                  const __grid_constant__ CUtensorMap tm_h, ExpertArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* xchg = reinterpret_cast<float*>(smem + kRingBytes);
  uint64_t* fullA = reinterpret_cast<uint64_t*>(smem + kRingBytes + kEpiBytes);
  uint64_t* emptyA = fullA + kMaxA;
  uint64_t* fullB = emptyA + kMaxA;
  uint64_t* emptyB = fullB + kMaxB;
  uint64_t* tfull = emptyB + kMaxB;
  uint64_t* tempty = tfull + 2;
  uint64_t* ufull = tempty + 2;
  uint64_t* uempty = ufull + kUnitRing;
  uint64_t* drain = uempty + kUnitRing;
  uint64_t* meet = drain + 2;  // the two UMMA issuers' end-of-unit rendezvous
  UnitInfo* units = reinterpret_cast<UnitInfo*>(drain + 3);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(units + kUnitRing);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_bcast = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int GU = a.f / kGuHalf;
  const int DN = a.d / kBM;
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
      mbar_init(&tfull[i], 2);   // one commit per UMMA issuer
      mbar_init(&tempty[i], 4);  // one arrival per epilogue warp
    }
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 4);  // two UMMA issuers, epilogue leader, B producer
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(meet, 2);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_wgu);
    tma_prefetch_desc(&tm_wd);
    tma_prefetch_desc(&tm_xp);
    tma_prefetch_desc(&tm_h);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // routing tables: written by the preceding kernels
  pdl_launch_dependents();

  // B-operand rows per stage: the largest chunk, rounded up to the TMA box.
  // The activation ring takes kMinB..kMaxB stages (as many as fit half of
  // the ring: at 2048 tokens a chunk's B stage is larger than its A stage
  // and its L2 latency must be hidden too), the weights the rest.  Both
  // depths are even, so within a unit whose K is split a ring slot comes
  // back to the same issuer; across units the issuers' end-of-unit
  // rendezvous covers it (see there).  Without both, an issuer could wait on
  // a slot whose previous stage belongs to the other issuer and is still in
  // flight, and its parity wait would pass a phase early.
  const int maxn = max(1, min(kMaxN, ctl->max_chunk));
  const int NB = (maxn + kBRows - 1) / kBRows * kBRows;
  const int b_bytes = NB * kBK * 2;
  const int SB = min(kMaxB, max(kMinB, (kRingBytes / 2) / b_bytes)) & ~1;
  const int SA = min(kMaxA, (kRingBytes - SB * b_bytes) / kABytes) & ~1;
  uint8_t* ringA = ring;
  uint8_t* ringB = ring + SA * kABytes;
  // Accumulators: two units in flight, 256 columns each.  A unit of at most
  // 128 tokens (and two or more K stages) has its K split between the two
  // issuers, each into a 128-column partial; a larger unit is issued by warp
  // 1 alone into all 256 columns (warp 7 then only keeps the barrier
  // protocol).  The choice depends on the unit alone, so a unit's result
  // does not depend on the other units of the call.
  constexpr int W = 128;                   // columns of one partial
  constexpr int ACC = kMaxN;               // columns of one unit's accumulator
  const int NBUF = kTmemCols / ACC;        // 2
  const int n_chunks = ctl->n_chunks;
  const int U = n_chunks * (GU + DN);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 claims units, waits and issues the copies.
    const uint64_t pol_w = l2_policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    int ur = 0;
    uint32_t uphase = 0;
    uint32_t issued = 0, issued_par = 0;  // stages with a copy issued, and its parity
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
          if (ui.n < 1 || ui.n > NB) {  // corrupt plan: never index outside the ring
            record_error(ctl, MOE_ERR_DEVICE_CHECK, 200);
            *s_abort = 1;
            go = 0;
          }
        }
        if (go && mbar_wait(&uempty[ur], uphase ^ 1, s_abort, ctl, a.timeout_ns,
                            kWhereUnitEmpty)) {
          units[ur] = ui;
          mbar_arrive(&ufull[ur]);
        } else {
          go = 0;
        }
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      ui.type = __shfl_sync(0xffffffffu, ui.type, 0);
      ui.n = __shfl_sync(0xffffffffu, ui.n, 0);
      ui.slot0 = __shfl_sync(0xffffffffu, ui.slot0, 0);
      if (!go || ui.type == kUnitStop) break;
      if (++ur == kUnitRing) {
        ur = 0;
        uphase ^= 1;
      }
      int ok = 1;
      if (lane == 0) {
        const int nkb = (ui.type == kUnitGateUp) ? a.d / kBK : a.f / kBK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyA[stage], phase ^ 1, s_abort, ctl, a.timeout_ns,
                         kWhereStageEmpty)) {
            ok = 0;
            break;
          }
          uint8_t* sa = ringA + stage * kABytes;
          mbar_arrive_expect_tx(&fullA[stage], kABytes);
          const int kx = kb * kBK;
          if (ui.type == kUnitGateUp) {
            const int r0 = ui.e * 2 * a.f + ui.m * kGuHalf;
            tma_load_2d(sa, &tm_wgu, kx, r0, &fullA[stage], pol_w);
            tma_load_2d(sa + kGuHalf * kBK * 2, &tm_wgu, kx, r0 + a.f, &fullA[stage], pol_w);
          } else {
            tma_load_2d(sa, &tm_wd, kx, ui.e * a.d + ui.m * kBM, &fullA[stage], pol_w);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == SA) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    // Drain: every issued copy must land before the CTA may exit.
    if (lane == 0)
      for (int s2 = 0; s2 < SA; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&fullA[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
  } else if (warp == 1 || warp == 7) {
    // ------------------------------------------------------------ UMMA issuers
    // Issuer par (0: warp 1, 1: warp 7) takes the K stages kb % 2 == par of
    // every unit into partial par of the unit's accumulator.  Both always
    // wait for the accumulator to be free and commit its full barrier (count
    // 2), so neither can run a phase ahead of the epilogue.
    if (lane == 0) {
      const int par = warp == 1 ? 0 : 1;
      int g = 0;  // ring stages used by all earlier units
      int ur = 0;
      uint32_t uphase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      uint32_t mphase = 0;
      while (true) {
        if (!mbar_wait(&ufull[ur], uphase, s_abort, ctl, a.timeout_ns, kWhereUnitFullMma)) break;
        const UnitInfo ui = units[ur];
        if (ui.type == kUnitStop) break;
        const int nkb = (ui.type == kUnitGateUp) ? a.d / kBK : a.f / kBK;
        const int N = (ui.n + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, N);
        if (!mbar_wait(&tempty[buf], bphase ^ 1, s_abort, ctl, a.timeout_ns, kWhereTmemEmpty))
          break;
        tc_fence_after();
        // Split K by the stage's parity inside the unit (a unit's result then
        // does not depend on the order the units were claimed in): this
        // issuer's first stage and step.  A unit of one stage, or of more
        // than W tokens, is warp 1's alone, in columns [0, ACC).
        const bool splitk = nkb > 1 && N <= W;
        const int first = splitk ? par : (par == 0 ? 0 : 1 << 30);
        const int step = splitk ? 2 : 1;
        const uint32_t dt = tmem_base + (uint32_t)(buf * ACC + (splitk ? par * W : 0));
        const int g0 = g + (first < nkb ? first : 0);
        int sa_i = g0 % SA, sb_i = g0 % SB;
        uint32_t pa = (uint32_t)(g0 / SA) & 1u, pb = (uint32_t)(g0 / SB) & 1u;
        bool ok = true;
        for (int kb = first; kb < nkb; kb += step) {
          if (!mbar_wait(&fullA[sa_i], pa, s_abort, ctl, a.timeout_ns, kWhereStageFull) ||
              !mbar_wait(&fullB[sb_i], pb, s_abort, ctl, a.timeout_ns, kWhereStageFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ringA + sa_i * kABytes);
          const uint32_t sb = smem_u32(ringB + sb_i * b_bytes);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma_bf16(dt, sdesc_k_sw128(sa + kk * kUmmaK * 2), sdesc_k_sw128(sb + kk * kUmmaK * 2),
                      idesc, (kb > first || kk > 0) ? 1u : 0u);
          umma_commit(&emptyA[sa_i]);
          umma_commit(&emptyB[sb_i]);
          sa_i += step;
          if (sa_i >= SA) {
            sa_i -= SA;
            pa ^= 1;
          }
          sb_i += step;
          if (sb_i >= SB) {
            sb_i -= SB;
            pb ^= 1;
          }
        }
        if (!ok) break;
        // The two issuers meet at the end of every unit: a ring slot then
        // holds, before it comes back to an issuer, either its own stage of
        // the same unit (the depths are even) or a stage of an earlier unit
        // that both issuers have waited on, so no parity wait can be
        // satisfied by a phase two behind.
        mbar_arrive(meet);
        if (!mbar_wait(meet, mphase, s_abort, ctl, a.timeout_ns, kWhereStageFull)) break;
        mphase ^= 1;
        umma_commit(&tfull[buf]);
        mbar_arrive(&uempty[ur]);
        g += nkb;
        if (++ur == kUnitRing) {
          ur = 0;
          uphase ^= 1;
        }
        if (++buf == NBUF) {
          buf = 0;
          bphase ^= 1;
        }
      }
      // Drain: all issued UMMAs complete before TMEM is released.
      umma_commit(&drain[par]);
      mbar_wait_drain(&drain[par], 0, ctl, a.timeout_ns);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ B producer
    // Follows the unit ring; a down unit's h tiles wait for every gate_up
    // unit of the chunk.
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
        const int nkb = (ui.type == kUnitGateUp) ? a.d / kBK : a.f / kBK;
        const int nbox = (ui.n + kBRows - 1) / kBRows;
        const uint32_t tx = nbox * kBRows * kBK * 2;
        const CUtensorMap* tb = (ui.type == kUnitGateUp) ? &tm_xp : &tm_h;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&emptyB[stage], phase ^ 1, s_abort, ctl, a.timeout_ns,
                         kWhereStageEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sb = ringB + stage * b_bytes;
          mbar_arrive_expect_tx(&fullB[stage], tx);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(sb + bx * kBRows * kBK * 2, tb, kb * kBK, ui.slot0 + bx * kBRows,
                        &fullB[stage], pol_act);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == SB) {
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
      for (int s2 = 0; s2 < SB; ++s2)
        if ((issued >> s2) & 1u)
          mbar_wait_drain(&fullB[s2], (issued_par >> s2) & 1u, ctl, a.timeout_ns);
    }
  } else {
    epilogue_role(a, units, ufull, uempty, tfull, tempty, xchg, s_abort, s_bcast, tmem_base,
                  ACC, warp, lane, nullptr, nullptr, kBK, NBUF);
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

cudaError_t moe_launch_expert(const moe::ExpertArgs& a, const CUtensorMap& tm_wgu,
                              const CUtensorMap& tm_wd, const CUtensorMap& tm_xp,
                              const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl) {
  static_assert(moe::kSmemBytes <= 232448, "expert kernel smem above the sm_100 limit");
  cudaError_t err = cudaFuncSetAttribute(moe::expert_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         moe::kSmemBytes);
  if (err != cudaSuccess) return err;
  return moe::launch_pdl(moe::expert_kernel, dim3(num_sms), dim3(moe::kThreads),
                         (size_t)moe::kSmemBytes, s, pdl, tm_wgu, tm_wd, tm_xp, tm_h, a);
}
