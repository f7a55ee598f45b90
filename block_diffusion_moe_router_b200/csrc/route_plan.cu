// route_plan.cu -- from the router's top-k indices to expert-contiguous work:
//   counts[e], offsets = exclusive scan, and a STABLE scatter: assignment
//   a = t*k + j of expert e gets slot offsets[e] + (number of earlier
//   assignments with the same expert).  Also the chunk table of the expert
//   kernel's scheduler (one chunk = up to 256 tokens of one expert) and the
//   reset of its counters; the gather of x rows into slot order; and the
//   fixed-order weighted combine.
//
// A cluster of CTAs of 32 warps (one per 2048 assignments, up to 16) does the
// counting sort: each warp owns a contiguous range of assignments, ranks
// equal experts inside each 32-wide step (the lanes with the same id, found
// with one ballot per id bit), and per-(warp, expert) and per-(CTA, expert)
// counts are scanned in order, so the result is independent of timing
// (bitwise deterministic).
#include <algorithm>

#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kRegIters = 16;  // 32-wide steps per warp held in registers (16K assignments)
constexpr int kRegRange = kPlanWarps * 32 * kRegIters;  // per-CTA range kept in registers
constexpr int kPlanMaxCluster = 16;
constexpr int kPlanPerCta = 2048;  // assignments per CTA before another joins the cluster

// Lanes of `mask` whose expert id equals this lane's: one ballot per bit of
// the id (ids < 2^nbits), each narrowing the set to the lanes that agree on
// that bit.  Cheaper than a match instruction and just as exact.
__device__ __forceinline__ unsigned peer_lanes(unsigned mask, int e, int nbits) {
  unsigned peers = mask;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    if (b < nbits) {
      const unsigned ones = __ballot_sync(0xffffffffu, (e >> b) & 1);
      peers &= ((e >> b) & 1) ? ones : ~ones;
    }
  }
  return peers;
}

// The counting sort, on a cluster of NC CTAs: CTA r owns assignments
// [r*A/NC, (r+1)*A/NC), warp w of it a contiguous sub-range.  Ranks inside a
// warp's 32-wide steps come from ballots; per-(warp, expert) counts are
// scanned in warp order, per-(CTA, expert) totals in rank order through
// distributed shared memory, so every slot is independent of timing.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs a) {
  extern __shared__ int s_perm[];  // [A] on a single CTA: perm built here, written in order
  __shared__ int cnt[kPlanWarps][kMaxE];  // per-warp counts, then per-warp bases
  __shared__ int ctot[kMaxE];             // this CTA's per-expert totals (read by peers)
  __shared__ int base[kMaxE];             // the expert's assignments in lower ranks
  __shared__ int tot[kMaxE];
  __shared__ int off[kMaxE + 1];
  __shared__ int cst[kMaxE + 1];
  __shared__ int wsum[2][kMaxE / 32];
  __shared__ int s_maxc;
  cg::cluster_group cluster = cg::this_cluster();
  const int NC = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int E = a.E;
  const int A = a.T * a.k;
  const int nbits = E > 1 ? 32 - __clz(E - 1) : 0;  // bits of an expert id (E <= 256)

  for (int i = tid; i < kPlanWarps * kMaxE; i += kPlanThreads) (&cnt[0][0])[i] = 0;
  if (tid == 0) s_maxc = 0;
  // The gather may launch at once: it waits for this grid to complete.
  pdl_launch_dependents();
  pdl_wait();  // idx comes from the router
  __syncthreads();

  const int clo = (int)((long long)A * rank / NC);
  const int chi = (int)((long long)A * (rank + 1) / NC);
  const int per = (chi - clo + kPlanWarps - 1) / kPlanWarps;
  const int lo = min(chi, clo + warp * per);
  const int hi = min(chi, lo + per);

  // ---- local ranks.  With at most kRegIters 32-wide steps per warp the
  // expert ids and ranks stay in registers; longer ranges keep the rank in
  // slot_of until the bases are known.
  const int iters = (hi - lo + 31) / 32;
  // uniform over the CTA: a range of <= kRegRange gives every warp <= kRegIters steps
  const bool in_regs = chi - clo <= kRegRange;
  int e_r[kRegIters], r_r[kRegIters];
  if (in_regs) {
    // every load of the warp's range in flight before the first use
#pragma unroll
    for (int it = 0; it < kRegIters; ++it) {
      const int as = lo + 32 * it + lane;
      e_r[it] = (it < iters && as < hi) ? __ldg(a.idx + as) : 0;
    }
#pragma unroll
    for (int it = 0; it < kRegIters; ++it) {
      if (it >= iters) break;  // warp-uniform
      const int as = lo + 32 * it + lane;
      const bool act = as < hi;
      int e = e_r[it];
      const unsigned mask = __ballot_sync(0xffffffffu, act);
      if (act && (e < 0 || e >= E)) {
        record_error(a.ctl, MOE_ERR_DEVICE_CHECK, 100);
        e = 0;
      }
      const unsigned peers = peer_lanes(mask, e, nbits);  // all lanes take part
      int rk = 0;
      if (act) {
        const int r = __popc(peers & ((1u << lane) - 1u));
        const int b = cnt[warp][e];
        __syncwarp(mask);
        if (r == 0) cnt[warp][e] = b + __popc(peers);
        rk = b + r;
      }
      __syncwarp();
      e_r[it] = e;
      r_r[it] = rk;
    }
  } else {
    for (int b0 = lo; b0 < hi; b0 += 32) {
      const int as = b0 + lane;
      const bool act = as < hi;
      const unsigned mask = __ballot_sync(0xffffffffu, act);
      int e = act ? __ldg(a.idx + as) : 0;
      if (act && (e < 0 || e >= E)) {
        record_error(a.ctl, MOE_ERR_DEVICE_CHECK, 100);
        e = 0;
      }
      const unsigned peers = peer_lanes(mask, e, nbits);  // all lanes take part
      if (act) {
        const int r = __popc(peers & ((1u << lane) - 1u));
        const int b = cnt[warp][e];
        __syncwarp(mask);
        if (r == 0) cnt[warp][e] = b + __popc(peers);
        a.slot_of[as] = b + r;
      }
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- per-expert bases: warps of this CTA, then the CTAs of the cluster
  if (tid < E) {
    int run = 0;
#pragma unroll 8
    for (int w = 0; w < kPlanWarps; ++w) {
      const int c = cnt[w][tid];
      cnt[w][tid] = run;
      run += c;
    }
    ctot[tid] = run;
  }
  if (NC > 1)
    cluster.sync();
  else
    __syncthreads();
  if (tid < E) {
    int b = 0, t = 0;
    for (int q = 0; q < NC; ++q) {
      const int c = (q == rank) ? ctot[tid] : *cluster.map_shared_rank(&ctot[tid], q);
      if (q < rank) b += c;
      t += c;
    }
    base[tid] = b;
    tot[tid] = t;
    atomicMax(&s_maxc, min(t, a.chunk));
  }
  __syncthreads();
  // ---- exclusive scans of the totals (slots) and of the chunk counts,
  // warp-level inclusive scans then a scan of the warp sums (E <= 256)
  {
    const int n = (tid < E) ? tot[tid] : 0;
    const int c = (n + a.chunk - 1) / a.chunk;
    int sn = n, sc = c;
    if (tid < kMaxE) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yn = __shfl_up_sync(0xffffffffu, sn, o);
        const int yc = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) {
          sn += yn;
          sc += yc;
        }
      }
      if (lane == 31) {
        wsum[0][warp] = sn;
        wsum[1][warp] = sc;
      }
    }
    __syncthreads();
    if (tid < kMaxE) {
      int bn = 0, bc = 0;
      for (int w = 0; w < warp; ++w) {
        bn += wsum[0][w];
        bc += wsum[1][w];
      }
      if (tid < E) {
        off[tid + 1] = bn + sn;
        cst[tid + 1] = bc + sc;
      }
      if (tid == 0) {
        off[0] = 0;
        cst[0] = 0;
      }
    }
  }
  __syncthreads();
  if (rank == 0) {
    if (tid == 0) {
      a.ctl->n_chunks = cst[E];
      a.ctl->max_chunk = s_maxc;
      a.ctl->work_next = 0;
    }
    if (tid <= E) a.offsets[tid] = off[tid];
    if (tid < E) {
      for (int q = cst[tid]; q < cst[tid + 1]; ++q) {
        const int c = q - cst[tid];
        a.chunk_info[q] = make_int4(tid, off[tid] + c * a.chunk, min(a.chunk, tot[tid] - c * a.chunk), c);
        a.ready[q] = 0;
      }
    }
  }

  // ---- final slots.  perm is a scatter; a single CTA builds it in shared
  // memory and writes it out in order (coalesced), since every store then
  // goes through one SM.
  if (in_regs) {
    const bool staged = NC == 1;
#pragma unroll
    for (int it = 0; it < kRegIters; ++it) {
      if (it >= iters) break;
      const int as = lo + 32 * it + lane;
      if (as < hi) {
        const int e = e_r[it];
        const int slot = off[e] + base[e] + cnt[warp][e] + r_r[it];
        a.slot_of[as] = slot;
        if (staged)
          s_perm[slot] = as / a.k;
        else
          a.perm[slot] = as / a.k;
      }
    }
    if (staged) {
      __syncthreads();
      for (int i = tid; i < A; i += kPlanThreads) a.perm[i] = s_perm[i];
    }
  } else {
    for (int as = lo + lane; as < hi; as += 32) {
      int e = __ldg(a.idx + as);
      if (e < 0 || e >= E) e = 0;
      const int slot = off[e] + base[e] + cnt[warp][e] + a.slot_of[as];
      a.slot_of[as] = slot;
      a.perm[slot] = as / a.k;
    }
  }
  if (NC > 1) cluster.sync();  // peers may still be reading ctot
}

// x rows in slot order: x_perm[s] = x[perm[s]], or, with gamma2, the
// expert-side norm bf16(x / sqrt(mean(x^2) + eps) * (1 + gamma2)) of that row
// (the model's pre-FFN norm, whose only consumer is the fused gate_up).  One
// warp per row, 16-byte moves, every load of the row issued before any use.
// With xf16 the row is written as fp16 instead (exact for bf16 values of
// magnitude 2^-14 .. 65504; the normed row is rounded once, to fp16).
constexpr int kGatherVec = 16;  // uint4 per lane held in registers (d <= 4096)
constexpr int kGatherMaxD = 4096;

// One row (warp-wide, lane owns 16-byte pieces lane + 32j), in passes of
// VEC pieces per lane with every load of a pass issued before any use.  With
// the expert norm, the row's sum of squares is taken first (an extra read
// when the row needs more than one pass); g1, when given, holds 1 + gamma2
// (in shared memory), else gamma2 is read from global memory.
template <int VEC>
__device__ __forceinline__ void gather_row(const GatherArgs& a, int row, int t, int lane,
                                           const float* g1 = nullptr) {
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
  uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (size_t)row * a.d);
  const int n = a.d / 8;
  const bool one_pass = n <= 32 * VEC;
  float inv = 1.f;
  uint4 v[VEC];
  if (a.gamma2) {
    float ss = 0.f;
    for (int p0 = 0; p0 < n; p0 += 32 * VEC) {
#pragma unroll
      for (int j = 0; j < VEC; ++j)
        if (p0 + lane + 32 * j < n) v[j] = __ldg(src + p0 + lane + 32 * j);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        if (p0 + lane + 32 * j < n) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h2[q]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    inv = 1.0f / sqrtf(ss / (float)a.d + a.eps);
  }
  for (int p0 = 0; p0 < n; p0 += 32 * VEC) {
    if (!(a.gamma2 && one_pass)) {  // a single-pass row is still in v
#pragma unroll
      for (int j = 0; j < VEC; ++j)
        if (p0 + lane + 32 * j < n) v[j] = __ldg(src + p0 + lane + 32 * j);
    }
    if (a.gamma2) {
      const float4* g4 = reinterpret_cast<const float4*>(a.gamma2);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        const int i = p0 + lane + 32 * j;
        if (i < n) {
          float g[8];  // 1 + gamma2 of the piece's eight columns
          if (g1) {
            const float4 ga = reinterpret_cast<const float4*>(g1)[2 * i];
            const float4 gb = reinterpret_cast<const float4*>(g1)[2 * i + 1];
            g[0] = ga.x; g[1] = ga.y; g[2] = ga.z; g[3] = ga.w;
            g[4] = gb.x; g[5] = gb.y; g[6] = gb.z; g[7] = gb.w;
          } else {
            const float4 ga = __ldg(g4 + 2 * i), gb = __ldg(g4 + 2 * i + 1);
            g[0] = 1.f + ga.x; g[1] = 1.f + ga.y; g[2] = 1.f + ga.z; g[3] = 1.f + ga.w;
            g[4] = 1.f + gb.x; g[5] = 1.f + gb.y; g[6] = 1.f + gb.z; g[7] = 1.f + gb.w;
          }
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&v[j]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h2[q]);
            const float y0 = (f.x * inv) * g[2 * q];
            const float y1 = (f.y * inv) * g[2 * q + 1];
            if (a.xf16)
              *reinterpret_cast<__half2*>(&h2[q]) = __floats2half2_rn(y0, y1);
            else
              h2[q] = __floats2bfloat162_rn(y0, y1);
          }
        }
      }
    } else if (a.xf16) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        if (p0 + lane + 32 * j < n) {
          __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&v[j]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h2[q]);
            *reinterpret_cast<__half2*>(&h2[q]) = __floats2half2_rn(f.x, f.y);
          }
        }
      }
    }
    const uint64_t pol_keep = l2_policy_evict_last();  // the expert kernel reads it next
#pragma unroll
    for (int j = 0; j < VEC; ++j)
      if (p0 + lane + 32 * j < n) st_global_hint(dst + p0 + lane + 32 * j, v[j], pol_keep);
  }
}

__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a) {
  // The expert kernel may launch at once (its prologue then overlaps this
  // grid); it waits for this grid to complete before reading the tables.
  pdl_launch_dependents();
  pdl_wait();
  // grid-stride over rows: at most a few CTAs per SM, all resident at once
  for (int row = blockIdx.x * 8 + (threadIdx.x >> 5); row < a.rows; row += gridDim.x * 8)
    gather_row<kGatherVec>(a, row, __ldg(a.perm + row), threadIdx.x & 31);
}


// Plan and gather in one launch for one canvas (T <= 256 tokens, T*k <=
// 2048 assignments): every CTA runs the whole counting sort redundantly in
// shared memory, CTA 0 alone writes the tables out, and each CTA then
// gathers its share of rows straight from its own copy of perm.  This saves
// the plan kernel's launch and one hand-off on the layer's critical path.
//
// Stable ranks from a token bitmap: thread t owns token t; bit t of row e is
// set when token t chose expert e (a token's k experts are distinct).  The
// rank of (t, e) among expert e's assignments in (t, j) order is the number
// of set bits of row e below t: a per-word exclusive prefix of the row's
// popcounts plus one masked popcount.
constexpr int kSmallT = 256;   // tokens (= threads)
constexpr int kSmallA = 2048;  // assignments
constexpr int kSmallK = 8;     // experts per token
constexpr int kSmallWords = kSmallT / 32;

__global__ void __launch_bounds__(kSmallT) plan_gather_small_kernel(PlanArgs a, GatherArgs g) {
  // word-major, so that lanes holding different experts hit different banks
  __shared__ uint32_t bits[kSmallWords][kMaxE];  // 8 KB at E = 256
  __shared__ int pre[kSmallWords][kMaxE];        // exclusive prefix popcounts per row
  __shared__ int tot[kMaxE];
  __shared__ int off[kMaxE + 1];
  __shared__ int cst[kMaxE + 1];
  __shared__ int wsum[2][kMaxE / 32];
  __shared__ int s_maxc;
  __shared__ int s_bad;
  __shared__ int s_perm[kSmallA];
  __shared__ __align__(16) float s_g1[kGatherMaxD];  // 1 + gamma2 (expert norm)
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int E = a.E;
  const int T = a.T;
  const int K = a.k;
  const int A = T * K;
  const bool writer = blockIdx.x == 0;

  for (int i = tid; i < kMaxE * kSmallWords; i += kSmallT) (&bits[0][0])[i] = 0u;
  if (tid == 0) {
    s_maxc = 0;
    s_bad = 0;
  }
  // The expert kernel may launch at once: it waits for this grid to complete.
  pdl_launch_dependents();
  pdl_wait();  // idx comes from the router
  // the expert norm's 1 + gamma2 into shared memory; its loads overlap the
  // plan below (the gather, after the plan's barriers, reads it)
  if (g.gamma2)
    for (int i = tid; i < g.d; i += kSmallT) s_g1[i] = 1.f + __ldg(g.gamma2 + i);
  __syncthreads();

  int ev[kSmallK];
  const bool own = tid < T;
  if (own) {
#pragma unroll
    for (int j = 0; j < kSmallK; ++j) {
      if (j < K) {
        int e = __ldg(a.idx + tid * K + j);
        if (e < 0 || e >= E) {
          s_bad = 1;
          e = 0;
        }
        ev[j] = e;
      }
    }
#pragma unroll
    for (int j = 0; j < kSmallK; ++j)
      if (j < K) atomicOr(&bits[warp][ev[j]], 1u << lane);
  }
  __syncthreads();
  if (tid < E) {  // row popcounts: exclusive prefix over the words, total
    int run = 0;
#pragma unroll
    for (int w = 0; w < kSmallWords; ++w) {
      pre[w][tid] = run;
      run += __popc(bits[w][tid]);
    }
    tot[tid] = run;
    atomicMax(&s_maxc, min(run, a.chunk));
  }
  __syncthreads();
  {  // exclusive scans of the totals and of the chunk counts (E <= 256 = threads)
    const int n = (tid < E) ? tot[tid] : 0;
    const int c = (n + a.chunk - 1) / a.chunk;
    int sn = n, sc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yn = __shfl_up_sync(0xffffffffu, sn, o);
      const int yc = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= o) {
        sn += yn;
        sc += yc;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = sn;
      wsum[1][warp] = sc;
    }
    __syncthreads();
    int bn = 0, bc = 0;
    for (int w = 0; w < warp; ++w) {
      bn += wsum[0][w];
      bc += wsum[1][w];
    }
    if (tid < E) {
      off[tid + 1] = bn + sn;
      cst[tid + 1] = bc + sc;
    }
    if (tid == 0) {
      off[0] = 0;
      cst[0] = 0;
    }
  }
  __syncthreads();
  if (writer) {
    if (tid == 0) {
      // a repeated expert in a token's set (or an id out of range) breaks
      // the count; slots stay in range, the status word reports it
      if (s_bad || off[E] != A) record_error(a.ctl, MOE_ERR_DEVICE_CHECK, 101);
      a.ctl->n_chunks = cst[E];
      a.ctl->max_chunk = s_maxc;
      a.ctl->work_next = 0;
    }
    if (tid <= E) a.offsets[tid] = off[tid];
    if (tid < E) {
      for (int q = cst[tid]; q < cst[tid + 1]; ++q) {
        const int c = q - cst[tid];
        a.chunk_info[q] =
            make_int4(tid, off[tid] + c * a.chunk, min(a.chunk, tot[tid] - c * a.chunk), c);
        a.ready[q] = 0;
      }
    }
  }
  if (own) {
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kSmallK; ++j) {
      if (j >= K) break;
      const int e = ev[j];
      const int slot = min(A - 1, off[e] + pre[warp][e] + __popc(bits[warp][e] & below));
      if (writer) a.slot_of[tid * K + j] = slot;
      s_perm[slot] = tid;
    }
  }
  __syncthreads();
  if (writer)
    for (int i = tid; i < A; i += kSmallT) a.perm[i] = s_perm[i];
  // this CTA's rows of x_perm (a warp per row)
  for (int row = blockIdx.x * (kSmallT / 32) + warp; row < A; row += gridDim.x * (kSmallT / 32))
    gather_row<kGatherVec>(g, row, s_perm[row], lane, g.gamma2 ? s_g1 : nullptr);
}

// out[t] = residual[t] + sum_j w[t,j] * y[slot_of[t,j]]   (j order, fp32, one
// rounding; w NULL: every weight 1, so with k = 1 a row is copied exactly).  One token per CTA step (grid-stride over tokens, a few CTAs per
// SM, so the whole grid is resident at once); a thread owns up to kCombCols
// 16-byte column groups of the row and issues the loads of up to kCombK
// contributions per column group before accumulating them.  slot_of and w of
// the token are read by every thread (the same addresses: one L1 line).  y is
// fp32 (4 values per load) or bf16 (8 values per load, widened exactly).
constexpr int kCombThreads = 128;
constexpr int kCombK = 8;         // contributions in flight per column group
constexpr int kCombMaxD = 4096;   // d a CTA of kCombThreads covers

template <typename YT>
struct YVec {
  static constexpr int n = 16 / (int)sizeof(YT);             // values per 16-byte load
  static constexpr int cols = kCombMaxD / (kCombThreads * n);  // column groups per thread
};

__device__ __forceinline__ void widen(const uint4& r, const float*, float (&v)[4]) {
  v[0] = __uint_as_float(r.x);
  v[1] = __uint_as_float(r.y);
  v[2] = __uint_as_float(r.z);
  v[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void widen(const uint4& r, const __nv_bfloat16*, float (&v)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// A slot outside the y rows is clamped (and reported) instead of read.
__device__ __forceinline__ int checked_slot(const CombineArgs& a, int sl) {
  if (a.rows > 0 && (sl < 0 || sl >= a.rows)) {
    if (a.ctl) record_error(a.ctl, MOE_ERR_DEVICE_CHECK, 120);
    return sl < 0 ? 0 : a.rows - 1;
  }
  return sl;
}

template <typename YT>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineArgs a) {
  constexpr int V = YVec<YT>::n;
  constexpr int kCombCols = YVec<YT>::cols;
  const YT* y = static_cast<const YT*>(a.y);
  // slot_of and w of the CTA's first token before the wait: they come from
  // the router and the plan, which completed before the expert kernel (this
  // grid's predecessor) could let this grid launch.
  int sl0[kCombK];
  float wt0[kCombK];
  {
    const int t = blockIdx.x;
#pragma unroll
    for (int j = 0; j < kCombK; ++j) {
      const bool in = t < a.T && j < a.k;
      sl0[j] = in ? checked_slot(a, __ldg(a.slot_of + (size_t)t * a.k + j)) : 0;
      wt0[j] = in ? (a.w ? __ldg(a.w + (size_t)t * a.k + j) : 1.f) : 0.f;
    }
  }
  pdl_wait();  // y comes from the expert kernel
  pdl_launch_dependents();
  const int ncol = a.d / V;  // 16-byte column groups per row
  const uint64_t pol_drop = l2_policy_evict_first();
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
    float acc[kCombCols][V];
#pragma unroll
    for (int q = 0; q < kCombCols; ++q)
#pragma unroll
      for (int i = 0; i < V; ++i) acc[q][i] = 0.f;
    for (int j0 = 0; j0 < a.k; j0 += kCombK) {
      int sl[kCombK];
      float wt[kCombK];
      const bool pre = t == (int)blockIdx.x && j0 == 0;
#pragma unroll
      for (int j = 0; j < kCombK; ++j) {
        sl[j] = pre ? sl0[j]
                    : (j0 + j < a.k) ? checked_slot(a, __ldg(a.slot_of + (size_t)t * a.k + j0 + j))
                                     : 0;
        wt[j] = pre ? wt0[j]
                    : (j0 + j < a.k) ? (a.w ? __ldg(a.w + (size_t)t * a.k + j0 + j) : 1.f) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < kCombCols; ++q) {
        const int col = threadIdx.x + kCombThreads * q;
        if (col >= ncol) break;
        uint4 r[kCombK];
#pragma unroll
        for (int j = 0; j < kCombK; ++j)
          if (j0 + j < a.k)  // read once: let it leave L2
            r[j] = ld_global_hint(reinterpret_cast<const uint4*>(y + (size_t)sl[j] * a.d) + col,
                                  pol_drop);
#pragma unroll
        for (int j = 0; j < kCombK; ++j) {
          if (j0 + j < a.k) {
            float v[V];
            widen(r[j], y, v);
#pragma unroll
            for (int i = 0; i < V; ++i) acc[q][i] = fmaf(wt[j], v[i], acc[q][i]);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kCombCols; ++q) {
      const int col = threadIdx.x + kCombThreads * q;
      if (col >= ncol) break;
      const size_t o = (size_t)t * a.d + (size_t)V * col;
      if (a.residual) {
#pragma unroll
        for (int i = 0; i < V; i += 4) {
          const uint2 rr = *reinterpret_cast<const uint2*>(a.residual + o + i);
          const float2 r0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rr.x));
          const float2 r1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rr.y));
          acc[q][i] = r0.x + acc[q][i];
          acc[q][i + 1] = r0.y + acc[q][i + 1];
          acc[q][i + 2] = r1.x + acc[q][i + 2];
          acc[q][i + 3] = r1.y + acc[q][i + 3];
        }
      }
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        __nv_bfloat162 o0 = __floats2bfloat162_rn(acc[q][i], acc[q][i + 1]);
        __nv_bfloat162 o1 = __floats2bfloat162_rn(acc[q][i + 2], acc[q][i + 3]);
        uint2 ov;
        ov.x = *reinterpret_cast<uint32_t*>(&o0);
        ov.y = *reinterpret_cast<uint32_t*>(&o1);
        *reinterpret_cast<uint2*>(a.out + o + i) = ov;
      }
    }
  }
}

// ---------------------------------------------------------------- expert parallel
// Dispatch of the token-expert assignments to the ranks that own the experts
// (rank r owns experts [r * per, (r + 1) * per)): the assignments are sorted
// by owner with the plan kernel, keyed by owner instead of expert, so each
// owner's rows are contiguous and in (token, j) order.

// keys[a] = idx[a] / per (the owner of the assignment's expert).
__global__ void __launch_bounds__(256) ep_keys_kernel(const int32_t* idx, int A, int E, int per,
                                                      int32_t* keys, Ctl* ctl) {
  pdl_wait();
  pdl_launch_dependents();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < A; i += gridDim.x * blockDim.x) {
    int e = idx[i];
    if (e < 0 || e >= E) {
      record_error(ctl, MOE_ERR_DEVICE_CHECK, 110);
      e = 0;
    }
    keys[i] = e / per;
  }
}

// send_expert[pos[a]] = idx[a] % per (the expert's index on its owner), and
// send_counts[r] = rows for owner r.
__global__ void __launch_bounds__(256) ep_meta_kernel(const int32_t* idx, const int32_t* pos,
                                                      const int32_t* offsets, int A, int E, int per,
                                                      int ranks, int32_t* send_expert,
                                                      int32_t* send_counts) {
  pdl_wait();
  pdl_launch_dependents();
  const int i0 = blockIdx.x * blockDim.x + threadIdx.x;
  if (i0 < ranks) send_counts[i0] = offsets[i0 + 1] - offsets[i0];
  for (int i = i0; i < A; i += gridDim.x * blockDim.x) {
    int e = idx[i];
    if (e < 0 || e >= E) e = 0;
    const int p = pos[i];
    if (p >= 0 && p < A) send_expert[p] = e % per;
  }
}

}  // namespace

}  // namespace moe

cudaError_t moe_launch_plan(const moe::PlanArgs& a, cudaStream_t s, bool pdl) {
  const int A = a.T * a.k;
  int nc = (A + moe::kPlanPerCta - 1) / moe::kPlanPerCta;
  nc = std::max(1, std::min(nc, moe::kPlanMaxCluster));
  if (nc > 8) {
    const cudaError_t err = cudaFuncSetAttribute(
        moe::plan_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  // a single CTA stages perm in shared memory (the whole range is in registers)
  const size_t smem = (nc == 1 && A <= moe::kRegRange) ? (size_t)A * sizeof(int) : 0;
  if (smem > 0) {
    const cudaError_t err = cudaFuncSetAttribute(
        moe::plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  if (nc == 1) return moe::launch_pdl(moe::plan_kernel, dim3(1), dim3(moe::kPlanThreads), smem, s, pdl, a);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nc);
  cfg.blockDim = dim3(moe::kPlanThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nc;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, moe::plan_kernel, a);
}

cudaError_t moe_launch_plan_gather(const moe::PlanArgs& a, const moe::GatherArgs& g, int num_sms,
                                   cudaStream_t s, bool pdl) {
  const int A = a.T * a.k;
  if (a.T <= moe::kSmallT && a.k <= moe::kSmallK && g.rows == A) {  // one launch
    const int blocks = std::max(1, std::min((A + 7) / 8, 4 * std::max(num_sms, 1)));
    return moe::launch_pdl(moe::plan_gather_small_kernel, dim3(blocks), dim3(moe::kSmallT), 0, s,
                           pdl, a, g);
  }
  const cudaError_t err = moe_launch_plan(a, s, pdl);
  if (err != cudaSuccess) return err;
  return moe_launch_gather(g, num_sms, s, pdl);
}

cudaError_t moe_launch_gather(const moe::GatherArgs& a, int num_sms, cudaStream_t s, bool pdl) {
  if (a.rows == 0) return cudaSuccess;
  static_assert(moe::kGatherVec * 32 * 8 >= 4096, "gather holds a whole row in registers");
  const int blocks = std::min((a.rows + 7) / 8, 4 * std::max(num_sms, 1));
  return moe::launch_pdl(moe::gather_kernel, dim3(blocks), dim3(256), 0, s, pdl, a);
}

cudaError_t moe_launch_combine(const moe::CombineArgs& a, int num_sms, cudaStream_t s, bool pdl) {
  if (a.T == 0) return cudaSuccess;
  if (a.d > moe::kCombMaxD) return cudaErrorInvalidValue;
  const dim3 grid(std::min(a.T, 8 * std::max(num_sms, 1)));
  if (a.y_bf16)
    return moe::launch_pdl(moe::combine_kernel<__nv_bfloat16>, grid, dim3(moe::kCombThreads), 0,
                           s, pdl, a);
  return moe::launch_pdl(moe::combine_kernel<float>, grid, dim3(moe::kCombThreads), 0, s, pdl,
                         a);
}

cudaError_t moe_launch_ep_keys(const int32_t* idx, int A, int E, int per, int32_t* keys,
                               moe::Ctl* ctl, int num_sms, cudaStream_t s, bool pdl) {
  if (A == 0) return cudaSuccess;
  const int blocks = std::max(1, std::min((A + 255) / 256, 4 * std::max(num_sms, 1)));
  return moe::launch_pdl(moe::ep_keys_kernel, dim3(blocks), dim3(256), 0, s, pdl, idx, A, E, per,
                         keys, ctl);
}

cudaError_t moe_launch_ep_meta(const int32_t* idx, const int32_t* pos, const int32_t* offsets,
                               int A, int E, int per, int ranks, int32_t* send_expert,
                               int32_t* send_counts, int num_sms, cudaStream_t s, bool pdl) {
  const int n = std::max(A, ranks);
  const int blocks = std::max(1, std::min((n + 255) / 256, 4 * std::max(num_sms, 1)));
  return moe::launch_pdl(moe::ep_meta_kernel, dim3(blocks), dim3(256), 0, s, pdl, idx, pos,
                         offsets, A, E, per, ranks, send_expert, send_counts);
}
