// common.cuh -- sm_100a building blocks shared by the MoE kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (UMMA + TMEM)
// wrappers, the device status word, and launch-parameter structs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- layout constants
constexpr int kBM = 128;           // UMMA M: weight rows per tile
constexpr int kBK = 64;            // K elements per pipeline stage (bf16: 128 bytes/row)
constexpr int kUmmaK = 16;         // K of one kind::f16 UMMA
constexpr int kMaxN = 256;         // tokens per unit (UMMA N upper bound)
constexpr int kBRows = 32;         // rows per B-operand TMA box
constexpr int kGuHalf = 64;        // gate rows (and up rows) per gate_up tile
constexpr int kTmemCols = 512;     // whole TMEM: 2 accumulators x 256 columns
constexpr int kRouterTT = 8;       // tokens per router CTA
constexpr int kRouterTE = 32;      // experts per router CTA
constexpr int kMaxE = 256;
constexpr int kMaxK = 32;

// Device status / scheduler words kept by the plan (one small int array).
struct Ctl {
  int status;        // 0 or an moe_status_t, first error wins
  int where;         // code of the wait or check that failed
  int work_next;     // next unit index handed out by the expert scheduler
  int n_chunks;      // number of (expert, 256-token chunk) pairs this call
  int max_chunk;     // largest chunk (tokens) this call
  int pad[3];
};

__device__ __forceinline__ void record_error(Ctl* ctl, int code, int where) {
  if (atomicCAS(&ctl->status, 0, code) == 0) atomicExch(&ctl->where, where);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up after
// timeout_ns (records MOE_ERR_TIMEOUT with `where`) or when another role of
// the CTA has already given up (*abort != 0).  Returns true on success.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          Ctl* ctl, uint64_t timeout_ns, int where) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(a, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_error(ctl, MOE_ERR_TIMEOUT, where);
      *abort = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte global store / load with an L2 eviction-priority hint (policy from
// l2_policy_evict_*): intermediates that the next kernel reads back are kept
// in L2 while the weight stream (evict_first) flows past them.
__device__ __forceinline__ void st_global_hint(void* p, const uint4& v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w), "l"(policy)
               : "memory");
}
__device__ __forceinline__ uint4 ld_global_hint(const void* p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load (no multicast): box at element coordinates (x, y),
// x innermost.  Completes `bytes` on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Bring [p, p + bytes) into L2 (bytes a multiple of 16, p 16-byte aligned).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

// The calling CTA's share of [base, base + bytes) into L2, issued by one
// thread as 64 KB bulk prefetches (bytes and base 16-byte aligned).  A
// prefetch only fills the coherent L2, so it is safe before the grid
// dependency wait.
__device__ __forceinline__ void prefetch_l2_grid(const void* base, uint64_t bytes) {
  if (threadIdx.x != 0) return;
  const uint64_t nblk = (uint64_t)gridDim.x * gridDim.y;
  const uint64_t me = (uint64_t)blockIdx.y * gridDim.x + blockIdx.x;
  const uint64_t share = ((bytes + nblk - 1) / nblk + 15) & ~uint64_t(15);
  const uint64_t lo = me * share;
  const uint64_t hi = lo + share < bytes ? lo + share : bytes;
  const char* b = static_cast<const char*>(base);
  for (uint64_t o = lo; o < hi; o += 65536) {
    const uint64_t n = hi - o < 65536 ? hi - o : 65536;
    prefetch_l2_bulk(b + o, (uint32_t)n);
  }
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every UMMA issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D.
//   [4,6) D format = 1 (f32), [7,10) A = 1 (bf16), [10,13) B = 1 (bf16),
//   [15] A major = 0 (K), [16] B major = 0 (K), [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with
// 128-byte swizzling: rows of 128 bytes, 8-row swizzle atoms 1024 bytes
// apart (SBO), leading offset unused for swizzled K-major (1), version 1,
// layout type 2 (SWIZZLE_128B).  The atom base must be 1024-byte aligned;
// stepping K inside the 128-byte row adds bytes to the start address.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// 32 lanes x 32 bit, 32 consecutive columns: thread i of the warp gets TMEM
// lane (warp's quarter base + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- CTA pairs
// Kernels on pairs of CTAs (2-CTA clusters, one CTA per SM): one
// tcgen05.mma.cta_group::2 of M = 256 reads 128 A rows from each CTA's shared
// memory and N/2 B rows from each, and writes 128 TMEM lanes x N columns in
// each CTA.  The even CTA issues the UMMAs and owns the full barriers; both
// CTAs' TMA copies complete on them, and the UMMA commits arrive on both
// CTAs' barriers.

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// plain arrive on a barrier given by its shared::cluster address
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr)
               : "memory");
}

// TMA tile into this CTA's shared memory, completing on the pair's barrier
// at `bar_cl` (a shared::cluster address, possibly in the peer CTA)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* m, int x, int y,
                                                 uint32_t bar_cl, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar_cl), "l"(policy)
      : "memory");
}

// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T, M = 256
__device__ __forceinline__ void umma_pair_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at the same offset in every CTA of `mask` when
// the pair's UMMAs issued so far are done.
__device__ __forceinline__ void umma_pair_commit(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Programmatic dependent launch: wait until the preceding grid in the stream
// has completed and its memory is visible (a no-op when the kernel was not
// launched with the attribute), and let the next grid begin launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- launch params
struct RouterArgs {
  int T, E, k, d;
  float eps;
  const __nv_bfloat16* x;
  const float* router_w;
  const float* gamma;
  const float* bias;
  int32_t* idx;
  float* w;
  float* gap;
  Ctl* ctl;
  const void* l2_prefetch;      // bytes to pull into L2 while routing (or NULL)
  uint64_t l2_prefetch_bytes;
};

struct PlanArgs {
  int T, E, k, d, f;
  int chunk;             // tokens per scheduler chunk (256 bf16, 128 int4)
  const int32_t* idx;    // [T*k]
  int32_t* offsets;      // [E+1]
  int32_t* perm;         // [T*k] slot -> token
  int32_t* slot_of;      // [T*k] assignment -> slot
  int4* chunk_info;      // [max_chunks] chunk -> {expert, first slot, tokens, index in expert}
  int32_t* ready;        // [max_chunks] gate_up tiles finished per chunk
  Ctl* ctl;
};


struct GatherArgs {
  int rows, d;
  float eps;
  const float* gamma2;   // expert-side (1 + gamma2) RMSNorm, or NULL for raw x
  const int32_t* perm;
  const __nv_bfloat16* x;
  __nv_bfloat16* x_perm;  // bf16, or fp16 bits when xf16 is set
  int xf16;               // write x_perm as fp16 (the fp8-weight path's B operand)
};

struct CombineArgs {
  int T, k, d;
  const int32_t* slot_of;
  const float* w;      // [T, k], or NULL: every weight 1
  const void* y;       // fp32 or bf16 [rows, d]
  int y_bf16;
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int rows = 0;        // rows of y: a slot outside [0, rows) is clamped and reported
  Ctl* ctl = nullptr;
};

struct ExpertArgs {
  int T, E, k, d, f;
  const int32_t* perm;     // slot -> token
  const int32_t* offsets;
  const int4* chunk_info;  // [max_chunks] {expert, first slot, tokens, index in expert}
  int32_t* ready;
  const __half* scales_gu;  // int4: [E, 2f, ceil(d/128)]
  const __half* scales_d;   // int4: [E, d, ceil(f/128)]
  const float* rows_gu;     // fp8: one fp32 scale per weight row [E, 2f]
  const float* rows_d;      // fp8: [E, d]
  __nv_bfloat16* h;   // [T*k, f] (fp16 bits on the fp8 path)
  void* y;            // [T*k, d], fp32 or (y_bf16) bf16
  int y_bf16;
  Ctl* ctl;
  uint64_t timeout_ns;
  int test_stall;
};


// lm_head over the canvas: statistics of softmax(z / temperature) per token
// and entropy-bounded acceptance (lm_head.cu).
struct LmHeadArgs {
  int T, V, d;
  float inv_temp;        // 1 / temperature
  float softcap;         // z -> softcap * tanh(z / softcap) when > 0
  float bound;           // entropy bound of the acceptance step
  const uint8_t* masked; // [T] 1 = still masked (NULL: all)
  float4* part;          // [T, ceil(V/256)] per-tile (max, sum exp, sum exp*u, argmax)
  int32_t* token;        // [T] argmax
  float* entropy;        // [T]
  float* logz;           // [T]
  uint8_t* accept;       // [T]
  Ctl* ctl;
  uint64_t timeout_ns;
};

// ---------------------------------------------------------------- top-k
// Order-preserving map of a float to an unsigned key (-0 is folded into +0
// first, so equal floats get equal keys).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f == 0.f ? 0.f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k of one token's logits, held C per lane (lane l: experts l + 32c, NaN
// already mapped to -inf).  Selection order is (logit desc, index asc); each
// round takes the warp's best by two redux.sync reductions (largest key,
// then lowest index among the lanes holding it).  Writes idx[j] and the
// routing weights w[j] = exp(z_j - z_0) / sum (softmax over the selected
// logits, i.e. the full softmax renormalised over the set), and gap =
// z_(k) - z_(k+1) (+inf when k == E).
template <int C>
__device__ __forceinline__ void warp_topk(const float (&v)[C], int E, int k, int lane,
                                          int32_t* idx, float* w, float* gap) {
  // Each lane first orders its C candidates (logit desc, index asc; the
  // indices lane + 32c rise with c, so an odd-even transposition sort that
  // swaps only on a strictly larger key keeps equal keys in index order).
  // Every round then compares lane heads only: the warp maximum of the key,
  // the lowest index among the lanes holding it, and that lane pops its head.
  uint32_t key[C];
  int id[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int ee = lane + 32 * c;
    key[c] = ee < E ? float_key(v[c]) : 0u;
    id[c] = ee < E ? ee : 0x7fffffff;
  }
#pragma unroll
  for (int pass = 0; pass < C; ++pass) {
#pragma unroll
    for (int c = pass & 1; c + 1 < C; c += 2) {
      const bool sw = key[c + 1] > key[c];
      const uint32_t ka = sw ? key[c + 1] : key[c], kb = sw ? key[c] : key[c + 1];
      const int ia = sw ? id[c + 1] : id[c], ib = sw ? id[c] : id[c + 1];
      key[c] = ka;
      key[c + 1] = kb;
      id[c] = ia;
      id[c + 1] = ib;
    }
  }
  float my_sel = -INFINITY;
  int my_idx = 0;
  float next_v = -INFINITY;
  const int rounds = (k < E) ? k + 1 : k;
  for (int j = 0; j < rounds; ++j) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
    const uint32_t cand = (key[0] == m) ? (uint32_t)id[0] : 0xffffffffu;
    const int bi = (int)__reduce_min_sync(0xffffffffu, cand);
    const float val = key_float(m);
    if (j < k) {
      if (id[0] == bi) {  // pop the head
#pragma unroll
        for (int c = 0; c + 1 < C; ++c) {
          key[c] = key[c + 1];
          id[c] = id[c + 1];
        }
        key[C - 1] = 0u;
        id[C - 1] = 0x7fffffff;
      }
      if (lane == j) {
        my_sel = val;
        my_idx = bi;
      }
    } else {
      next_v = val;
    }
  }
  const float top = __shfl_sync(0xffffffffu, my_sel, 0);
  const float ex = (lane < k) ? expf(my_sel - top) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    idx[lane] = my_idx;
    w[lane] = ex / sum;
  }
  const float last = __shfl_sync(0xffffffffu, my_sel, k - 1);
  if (lane == 0 && gap) *gap = (k < E) ? (last - next_v) : INFINITY;
}

// Launch with programmatic stream serialization (when pdl is set) so the
// kernel's launch and prologue overlap the tail of the previous kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace moe

// Host-side launchers (one per kernel file).
cudaError_t moe_launch_router(const moe::RouterArgs& a, const CUtensorMap& tm_rw, cudaStream_t s,
                              bool pdl);
size_t moe_router_smem_bytes(int d);
int moe_router_tc_splits(int d, int T);
cudaError_t moe_launch_router_tc(const moe::RouterArgs& a, const CUtensorMap& tm_x, int EP,
                                 cudaStream_t s, bool pdl);
cudaError_t moe_launch_plan(const moe::PlanArgs& a, cudaStream_t s, bool pdl);
cudaError_t moe_launch_gather(const moe::GatherArgs& a, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_plan_gather(const moe::PlanArgs& a, const moe::GatherArgs& g, int num_sms,
                                   cudaStream_t s, bool pdl);
cudaError_t moe_launch_combine(const moe::CombineArgs& a, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_ep_keys(const int32_t* idx, int A, int E, int per, int32_t* keys,
                               moe::Ctl* ctl, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_ep_meta(const int32_t* idx, const int32_t* pos, const int32_t* offsets,
                               int A, int E, int per, int ranks, int32_t* send_expert,
                               int32_t* send_counts, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_expert(const moe::ExpertArgs& a, const CUtensorMap& tm_wgu,
                              const CUtensorMap& tm_wd, const CUtensorMap& tm_xp,
                              const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_expert_w4(const moe::ExpertArgs& a, const CUtensorMap& tm_cgu,
                                 const CUtensorMap& tm_cd, const CUtensorMap& tm_xp,
                                 const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_lmhead_gemm(const moe::LmHeadArgs& a, const CUtensorMap& tm_w,
                                   const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl);
cudaError_t moe_launch_lmhead_tail(const moe::LmHeadArgs& a, cudaStream_t s, bool pdl);
cudaError_t moe_launch_expert_w8(const moe::ExpertArgs& a, const CUtensorMap& tm_cgu,
                                 const CUtensorMap& tm_cd, const CUtensorMap& tm_xp,
                                 const CUtensorMap& tm_h, int num_sms, cudaStream_t s, bool pdl);
