// route_plan.cu -- from the router's top-k indices to expert-contiguous work:
//   counts[e], offsets = exclusive scan, and a STABLE scatter: assignment
//   a = t*k + j of expert e gets slot offsets[e] + (number of earlier
//   assignments with the same expert).  Also the chunk table of the expert
//   kernel's scheduler (one chunk = up to 256 tokens of one expert) and the
//   reset of its counters; and the gather of x rows into slot order.
//
// One CTA of 32 warps does the counting sort: warp w owns a contiguous range
// of assignments, ranks equal experts inside each 32-wide step with
// __match_any_sync, and per-(warp, expert) counts are scanned in warp order,
// so the result is independent of timing (bitwise deterministic).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs a) {
  __shared__ int cnt[kPlanWarps][kMaxE];  // per-warp counts, then per-warp bases
  __shared__ int off[kMaxE + 1];
  __shared__ int cst[kMaxE + 1];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int E = a.E;
  const int A = a.T * a.k;

  for (int i = tid; i < kPlanWarps * kMaxE; i += kPlanThreads) (&cnt[0][0])[i] = 0;
  __syncthreads();

  const int per = (A + kPlanWarps - 1) / kPlanWarps;
  const int lo = min(A, warp * per);
  const int hi = min(A, lo + per);

  // ---- local ranks (stored in slot_of until the bases are known)
  for (int base = lo; base < hi; base += 32) {
    const int as = base + lane;
    const bool act = as < hi;
    const unsigned mask = __ballot_sync(0xffffffffu, act);
    if (act) {
      int e = a.idx[as];
      if (e < 0 || e >= E) {
        record_error(a.ctl, MOE_ERR_DEVICE_CHECK, 100);
        e = 0;
      }
      const unsigned peers = __match_any_sync(mask, e);
      const int r = __popc(peers & ((1u << lane) - 1u));
      const int b = cnt[warp][e];
      __syncwarp(mask);
      if (r == 0) cnt[warp][e] = b + __popc(peers);
      a.slot_of[as] = b + r;
    }
    __syncwarp();
  }
  __syncthreads();

  // ---- per-expert totals; per-warp bases inside each expert's segment
  if (tid < E) {
    int run = 0;
    for (int w = 0; w < kPlanWarps; ++w) {
      const int c = cnt[w][tid];
      cnt[w][tid] = run;
      run += c;
    }
    off[tid] = run;  // total, scanned below
  }
  __syncthreads();
  if (tid == 0) {
    int o = 0, q = 0, mx = 0;
    for (int e = 0; e < E; ++e) {
      const int n = off[e];
      off[e] = o;
      cst[e] = q;
      o += n;
      q += (n + kMaxN - 1) / kMaxN;
      mx = max(mx, min(n, kMaxN));
    }
    off[E] = o;
    cst[E] = q;
    a.ctl->n_chunks = q;
    a.ctl->max_chunk = mx;
    a.ctl->work_next = 0;
  }
  __syncthreads();
  if (tid <= E) a.offsets[tid] = off[tid];
  if (tid < E) {
    for (int q = cst[tid]; q < cst[tid + 1]; ++q) {
      a.chunk_e[q] = tid;
      a.chunk_c[q] = q - cst[tid];
      a.ready[q] = 0;
    }
  }

  // ---- final slots
  for (int as = lo + lane; as < hi; as += 32) {
    int e = a.idx[as];
    if (e < 0 || e >= E) e = 0;
    const int slot = off[e] + cnt[warp][e] + a.slot_of[as];
    a.slot_of[as] = slot;
    a.perm[slot] = as / a.k;
  }
}

// x rows in slot order: x_perm[s] = x[perm[s]] (one warp per row, 16-byte moves)
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  const int t = __ldg(a.perm + row);
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
  uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (size_t)row * a.d);
  for (int i = lane; i < a.d / 8; i += 32) dst[i] = __ldg(src + i);
}

// out[t] = residual[t] + sum_j w[t,j] * y[slot_of[t,j]]   (j order, fp32)
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  __shared__ int sl[kMaxK];
  __shared__ float wt[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < a.k) {
    sl[threadIdx.x] = a.slot_of[(size_t)t * a.k + threadIdx.x];
    wt[threadIdx.x] = a.w[(size_t)t * a.k + threadIdx.x];
  }
  __syncthreads();
  for (int i = threadIdx.x * 4; i < a.d; i += blockDim.x * 4) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < a.k; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(a.y + (size_t)sl[j] * a.d + i));
      const float wj = wt[j];
      s.x = fmaf(wj, v.x, s.x);
      s.y = fmaf(wj, v.y, s.y);
      s.z = fmaf(wj, v.z, s.z);
      s.w = fmaf(wj, v.w, s.w);
    }
    if (a.residual) {
      const uint2 r = *reinterpret_cast<const uint2*>(a.residual + (size_t)t * a.d + i);
      const float2 r0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
      const float2 r1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
      s.x = r0.x + s.x;
      s.y = r0.y + s.y;
      s.z = r1.x + s.z;
      s.w = r1.y + s.w;
    }
    __nv_bfloat162 o0 = __floats2bfloat162_rn(s.x, s.y);
    __nv_bfloat162 o1 = __floats2bfloat162_rn(s.z, s.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&o0);
    o.y = *reinterpret_cast<uint32_t*>(&o1);
    *reinterpret_cast<uint2*>(a.out + (size_t)t * a.d + i) = o;
  }
}

}  // namespace

}  // namespace moe

cudaError_t moe_launch_plan(const moe::PlanArgs& a, cudaStream_t s) {
  moe::plan_kernel<<<1, moe::kPlanThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t moe_launch_gather(const moe::GatherArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  moe::gather_kernel<<<(a.rows + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t moe_launch_combine(const moe::CombineArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  moe::combine_kernel<<<a.T, 256, 0, s>>>(a);
  return cudaGetLastError();
}
