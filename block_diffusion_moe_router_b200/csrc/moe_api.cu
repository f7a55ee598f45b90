// moe_api.cu -- host side of the C ABI declared in include/moe.h: plan
// objects, argument validation, the plan-owned workspace, TMA tensor maps and
// the launch sequence router -> plan -> gather -> expert GEMMs -> combine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "moe.h"

// fp4 expert kernel (expert_w4f.cu): the fp8 launcher's arguments plus the
// block-scale tensor maps of both weights.
cudaError_t moe_launch_expert_w4f(const moe::ExpertArgs& a, const CUtensorMap& tm_cgu,
                                  const CUtensorMap& tm_cd, const CUtensorMap& tm_xp,
                                  const CUtensorMap& tm_h, const CUtensorMap& tm_bgu,
                                  const CUtensorMap& tm_bd, int num_sms, cudaStream_t s,
                                  bool pdl);

namespace {

using moe::Ctl;

struct ProfRec {
  int kernel;
  cudaEvent_t start, stop;
};

}  // namespace

struct moe_plan_s {
  int E, k, d, f;
  moe_wdtype_t wdtype;
  int device;
  int num_sms;
  float eps;
  int timeout_ms;
  int profile;
  int test_stall;
  int pdl;
  int prefetch_mb;
  int y_bf16;
  int router_sel;
  int debug;       // MOE_OPT_DEBUG: lay the next workspace out with guard blocks
  int chunk_tokens;  // MOE_OPT_CHUNK_TOKENS: 0 (by call size), 128 or 256
  int cap_T;
  int last_T;
  void* ws;  // one device allocation holding everything below
  std::vector<size_t> guards;  // offsets of the workspace's guard blocks (debug layout)
  Ctl* noalloc_ctl;            // status word of this plan's last moe_forward_noalloc call
  Ctl* ctl;
  int32_t *idx, *perm, *slot_of, *offsets, *ready;
  int4* chunk_info;
  float *w, *gap, *y;
  __nv_bfloat16 *x_perm, *h, *x_dev, *res_dev, *out_dev;
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> ev_pool;
};

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, 128-byte swizzle,
// box = box_rows x 64 columns (128 bytes).
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D fp32 tensor map over the router weight [E, d]: box = 32 rows x 128
// columns, no swizzle; rows past E read as zero.
bool make_map_router(CUtensorMap* m, const float* base, uint64_t E, uint64_t d) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {d, E};
  cuuint64_t strides[1] = {d * 4};
  cuuint32_t box[2] = {128, (cuuint32_t)moe::kRouterTE};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_codes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols_bytes,
                    uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols_bytes, rows};
  cuuint64_t strides[1] = {cols_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Tokens per scheduler chunk.  128 for the int4, fp8 and fp4 kernels (which
// keep decoded A stages in TMEM next to the accumulators).  bf16:
// MOE_OPT_CHUNK_TOKENS, by default 128 for a call of at most 256 tokens and
// 256 above.  At one canvas a hot expert then becomes chunks of at most 128
// tokens, each with two UMMA issuers and activation stages of at most 16 KB
// (a 256-token chunk sizes every stage at 32 KB and leaves two); for long
// calls, where most experts get 100-200 tokens, one 256-token chunk streams
// each expert's weights once.
int chunk_size(moe_plan_t p, int T) {
  if (p->wdtype != MOE_W_BF16) return 128;
  if (p->chunk_tokens == 128 || p->chunk_tokens == moe::kMaxN) return p->chunk_tokens;
  return T <= 256 ? 128 : moe::kMaxN;
}

size_t max_chunks(int E, size_t T, int k) { return (size_t)E + (T * (size_t)k) / 128 + 1; }

// Experts rounded up to the UMMA N granularity for the tensor-core router.
int router_ep(int E) { return (E + 15) / 16 * 16; }

// Router path: the tensor-core router (E <= 128) unless the FFMA router is
// asked for; E > 128 always takes the FFMA router.
bool use_router_tc(moe_plan_t p, int T) {
  (void)T;
  return p->E <= 128 && p->router_sel != 1;
}

// 2-D byte tensor map over packed int4 codes [rows, cols_bytes]: box = box_rows
// x 64 bytes (one group of 128 codes), 64-byte swizzle.
bool make_map_codes(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols_bytes,
                    uint32_t box_rows);

// 2-D byte tensor map over fp8 codes [rows, cols]: box = box_rows x 128 bytes
// (one 128-wide K stage), 128-byte swizzle.
bool make_map_fp8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D byte tensor map over packed fp4 codes [rows, cols_bytes]: box =
// box_rows x 128 bytes (two 128-wide K stages), 128-byte swizzle.
bool make_map_codes_pair(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols_bytes,
                         uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols_bytes, rows};
  cuuint64_t strides[1] = {cols_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D byte tensor map over the E4M3 block scales of fp4 scale records: the
// records are {fp32 s[R]; uint8 block[NB][R]} back to back, so the block
// scales form an [E][NB][R] array with row stride R and expert stride equal to
// the record size.  Box = box_rows x 16 blocks (a pair of 128-wide K stages).
bool make_map_blk(CUtensorMap* m, const void* records, uint64_t E, uint64_t R, uint64_t NB,
                  uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {R, NB, E};
  cuuint64_t strides[2] = {R, R * (4 + NB)};
  cuuint32_t box[3] = {box_rows, 16, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  void* base = const_cast<uint8_t*>(static_cast<const uint8_t*>(records) + 4 * R);
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

moe_status_t check_device(moe_plan_t p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  return dev == p->device ? MOE_OK : MOE_ERR_INVALID_ARG;
}

constexpr size_t kGuardBytes = 256;
constexpr int kGuardByte = 0xA5;

// T within the token limits of include/moe.h.
bool tokens_ok(const moe_plan_s* p, int T) {
  return T <= MOE_MAX_T && (int64_t)T * p->k <= (int64_t)MOE_MAX_ASSIGNMENTS;
}

// Grows the workspace to hold T tokens (T within tokens_ok), stream-ordered
// on `s`: the old allocation is released with cudaFreeAsync and the new one
// taken with cudaMallocAsync and cleared with cudaMemsetAsync, so the host
// never waits.  With the debug layout a guard block of kGuardBytes follows
// every region.
moe_status_t ensure_workspace(moe_plan_t p, int T, cudaStream_t s) {
  if (p->ws && T <= p->cap_T) return MOE_OK;
  {
    // growth inside a stream capture would put allocation nodes into the
    // caller's graph: the workspace must be reserved before capturing
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return MOE_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return MOE_ERR_UNSUPPORTED;
  }
  size_t cap = p->cap_T > 0 ? (size_t)p->cap_T : 16;
  while (cap < (size_t)T) cap *= 2;
  if (cap > (size_t)MOE_MAX_T) cap = MOE_MAX_T;
  if (cap * (size_t)p->k > (size_t)MOE_MAX_ASSIGNMENTS) cap = (size_t)T;
  const size_t A = cap * p->k;
  const size_t MC = max_chunks(p->E, cap, p->k);
  const bool dbg = p->debug != 0;
  std::vector<size_t> guards;
  size_t sz = 0;
  auto take = [&](size_t bytes) {
    size_t o = sz;
    sz += align256(bytes);
    if (dbg) {
      guards.push_back(sz);
      sz += kGuardBytes;
    }
    return o;
  };
  const size_t o_ctl = take(sizeof(Ctl));
  const size_t o_idx = take(A * 4), o_w = take(A * 4), o_gap = take(cap * 4);
  const size_t o_perm = take(A * 4), o_slot = take(A * 4), o_off = take((size_t)(p->E + 1) * 4);
  const size_t o_ci = take(MC * 16), o_rd = take(MC * 4);
  const size_t o_xp = take(A * p->d * 2);
  const size_t o_h = take(A * p->f * 2), o_y = take(A * p->d * 4);
  const size_t o_xd = take(cap * p->d * 2), o_rs = take(cap * p->d * 2);
  const size_t o_od = take(cap * p->d * 2);
  if (p->ws) {
    if (cudaFreeAsync(p->ws, s) != cudaSuccess) return MOE_ERR_CUDA;
    p->ws = nullptr;
    p->cap_T = 0;
  }
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, sz, s) != cudaSuccess) {
    cudaGetLastError();
    p->cap_T = 0;
    return MOE_ERR_ALLOC;
  }
  if (cudaMemsetAsync(ws, 0, sz, s) != cudaSuccess) {
    cudaFreeAsync(ws, s);
    return MOE_ERR_CUDA;
  }
  char* b = static_cast<char*>(ws);
  for (size_t g : guards)
    if (cudaMemsetAsync(b + g, kGuardByte, kGuardBytes, s) != cudaSuccess) {
      cudaFreeAsync(ws, s);
      return MOE_ERR_CUDA;
    }
  p->ws = ws;
  p->guards.swap(guards);
  p->ctl = reinterpret_cast<Ctl*>(b + o_ctl);
  p->idx = reinterpret_cast<int32_t*>(b + o_idx);
  p->w = reinterpret_cast<float*>(b + o_w);
  p->gap = reinterpret_cast<float*>(b + o_gap);
  p->perm = reinterpret_cast<int32_t*>(b + o_perm);
  p->slot_of = reinterpret_cast<int32_t*>(b + o_slot);
  p->offsets = reinterpret_cast<int32_t*>(b + o_off);
  p->chunk_info = reinterpret_cast<int4*>(b + o_ci);
  p->ready = reinterpret_cast<int32_t*>(b + o_rd);
  p->x_perm = reinterpret_cast<__nv_bfloat16*>(b + o_xp);
  p->h = reinterpret_cast<__nv_bfloat16*>(b + o_h);
  p->y = reinterpret_cast<float*>(b + o_y);
  p->x_dev = reinterpret_cast<__nv_bfloat16*>(b + o_xd);
  p->res_dev = reinterpret_cast<__nv_bfloat16*>(b + o_rs);
  p->out_dev = reinterpret_cast<__nv_bfloat16*>(b + o_od);
  p->cap_T = (int)cap;
  return MOE_OK;
}

cudaEvent_t take_event(moe_plan_t p) {
  if (!p->ev_pool.empty()) {
    cudaEvent_t e = p->ev_pool.back();
    p->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Records an event pair around one launch when profiling is on.
struct ProfScope {
  moe_plan_t p;
  int kernel;
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(moe_plan_t p_, int k_, cudaStream_t s_) : p(p_), kernel(k_), s(s_) {
    if (p->profile && p->prof.size() < 65536) {
      a = take_event(p);
      b = take_event(p);
      if (a && b) cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    if (a && b) {
      cudaEventRecord(b, s);
      p->prof.push_back({kernel, a, b});
    }
  }
};

moe_status_t validate_route(moe_plan_t p, int T, const void* x, const float* rw,
                            const float* gamma, const float* bias) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!tokens_ok(p, T)) return MOE_ERR_UNSUPPORTED;
  if (!x || !rw || !gamma) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(rw) || !aligned16(gamma)) return MOE_ERR_INVALID_ARG;
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) return MOE_ERR_INVALID_ARG;
  return check_device(p);
}

// Bytes of the fused gate_up weight pulled into L2 during routing.
uint64_t prefetch_bytes(moe_plan_t p) {
  const uint64_t n = (uint64_t)p->E * 2 * p->f * p->d;  // weights of the fused gate_up
  const uint64_t all =
      p->wdtype == MOE_W_BF16 ? 2 * n : (p->wdtype == MOE_W_FP8_E4M3 ? n : n / 2);  // int4, fp4: n/2
  const uint64_t want = (uint64_t)p->prefetch_mb << 20;
  return want < all ? want : all;
}

moe_status_t launch_router(moe_plan_t p, int T, const void* x, const float* rw,
                           const float* gamma, const float* bias, int32_t* idx, float* w,
                           float* gap, cudaStream_t s, const void* pf = nullptr,
                           uint64_t pf_bytes = 0, Ctl* ctl = nullptr) {
  moe::RouterArgs ra;
  ra.T = T;
  ra.E = p->E;
  ra.k = p->k;
  ra.d = p->d;
  ra.eps = p->eps;
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.router_w = rw;
  ra.gamma = gamma;
  ra.bias = bias;
  ra.idx = idx;
  ra.w = w;
  ra.gap = gap;
  ra.ctl = ctl ? ctl : p->ctl;
  ra.l2_prefetch = pf_bytes ? pf : nullptr;
  ra.l2_prefetch_bytes = pf_bytes;
  const bool pdl = p->pdl != 0;
  if (use_router_tc(p, T)) {
    const int EP = router_ep(p->E);
    CUtensorMap tm_x;
    if (!make_map_bf16(&tm_x, x, (uint64_t)T, p->d, 128)) return MOE_ERR_CUDA;
    ProfScope ps(p, MOE_K_ROUTER, s);
    return moe_launch_router_tc(ra, tm_x, EP, s, pdl) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  CUtensorMap tm_rw;
  if (!make_map_router(&tm_rw, rw, p->E, p->d)) return MOE_ERR_CUDA;
  ProfScope ps(p, MOE_K_ROUTER, s);
  return moe_launch_router(ra, tm_rw, s, pdl) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* moe_status_str(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: bad pointer, size, alignment or aliasing";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or dtype outside the kernels' limits";
    case MOE_ERR_ALLOC: return "MOE_ERR_ALLOC: workspace allocation failed";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or launch failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a device-side bounded wait ran out";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a kernel saw an out-of-range index";
  }
  return "unknown moe_status_t";
}

moe_status_t moe_plan_create(int E, int k, int d, int f, moe_wdtype_t wdtype, moe_plan_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (E < 1 || E > moe::kMaxE || k < 1 || k > E || k > moe::kMaxK) return MOE_ERR_UNSUPPORTED;
  if (d < 128 || d > 4096 || d % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (f < 64 || f > 4096 || f % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (wdtype != MOE_W_BF16 && wdtype != MOE_W_INT4_G128 && wdtype != MOE_W_FP8_E4M3 &&
      wdtype != MOE_W_FP4_E2M1)
    return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe_plan_s* p = new moe_plan_s();
  p->E = E;
  p->k = k;
  p->d = d;
  p->f = f;
  p->wdtype = wdtype;
  p->device = dev;
  p->num_sms = sms;
  p->eps = 1e-6f;
  p->timeout_ms = 1000;
  p->profile = 0;
  p->test_stall = 0;
  p->pdl = 1;
  p->prefetch_mb = 0;
  p->y_bf16 = 1;
  p->router_sel = 0;
  p->debug = 0;
  p->chunk_tokens = 0;
  p->cap_T = 0;
  p->last_T = 0;
  p->ws = nullptr;
  p->noalloc_ctl = nullptr;
  *out = p;
  return MOE_OK;
}

moe_status_t moe_plan_set_option(moe_plan_t p, int key, double value) {
  if (!p) return MOE_ERR_INVALID_ARG;
  switch (key) {
    case MOE_OPT_EPS:
      if (!(value >= 0.0)) return MOE_ERR_INVALID_ARG;
      p->eps = (float)value;
      return MOE_OK;
    case MOE_OPT_TIMEOUT_MS:
      if (!(value >= 1.0 && value <= 600000.0)) return MOE_ERR_INVALID_ARG;
      p->timeout_ms = (int)value;
      return MOE_OK;
    case MOE_OPT_PROFILE:
      p->profile = value != 0.0;
      return MOE_OK;
    case MOE_OPT_TEST_STALL:
      p->test_stall = value != 0.0;
      return MOE_OK;
    case MOE_OPT_PDL:
      p->pdl = value != 0.0;
      return MOE_OK;
    case MOE_OPT_ROUTER:
      if (!(value == 0.0 || value == 1.0 || value == 2.0)) return MOE_ERR_INVALID_ARG;
      p->router_sel = (int)value;
      return MOE_OK;
    case MOE_OPT_L2_PREFETCH_MB:
      if (!(value >= 0.0 && value <= 4096.0)) return MOE_ERR_INVALID_ARG;
      p->prefetch_mb = (int)value;
      return MOE_OK;
    case MOE_OPT_Y_BF16:
      p->y_bf16 = value != 0.0;
      return MOE_OK;
    case MOE_OPT_DEBUG:
      p->debug = value != 0.0;
      return MOE_OK;
    case MOE_OPT_CHUNK_TOKENS:
      if (value != 0.0 && value != 128.0 && value != (double)moe::kMaxN) return MOE_ERR_INVALID_ARG;
      p->chunk_tokens = (int)value;
      return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

moe_status_t moe_plan_reserve(moe_plan_t p, int max_T) {
  if (!p || max_T < 0) return MOE_ERR_INVALID_ARG;
  if (!tokens_ok(p, max_T)) return MOE_ERR_UNSUPPORTED;
  moe_status_t st = check_device(p);
  if (st != MOE_OK) return st;
  st = ensure_workspace(p, max_T > 0 ? max_T : 1, nullptr);
  if (st != MOE_OK) return st;
  return cudaStreamSynchronize(nullptr) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_route(moe_plan_t p, int T, const void* x, const float* router_w,
                       const float* router_gamma, const float* router_bias, int32_t* idx_out,
                       float* w_out, float* gap_out, void* stream) {
  moe_status_t st = validate_route(p, T, x, router_w, router_gamma, router_bias);
  if (st != MOE_OK || T == 0) return st;
  if (!idx_out || !w_out) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx_out) & 3u) || (reinterpret_cast<uintptr_t>(w_out) & 3u) ||
      (gap_out && (reinterpret_cast<uintptr_t>(gap_out) & 3u)))
    return MOE_ERR_INVALID_ARG;
  st = ensure_workspace(p, 1, static_cast<cudaStream_t>(stream));
  if (st != MOE_OK) return st;
  return launch_router(p, T, x, router_w, router_gamma, router_bias, idx_out, w_out, gap_out,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// The layer, or (row_expert != NULL) its expert part alone: rows x[t] routed
// to expert row_expert[t] with weight 1 (a plan with k == 1), no router.
// The router arguments are validated by the caller.
moe_status_t forward_impl(moe_plan_t p, int T, const void* x, const float* router_w,
                          const float* router_gamma, const float* router_bias,
                          const int32_t* row_expert, const float* expert_gamma,
                          const void* w_gate_up, const void* w_down, const void* scales_gate_up,
                          const void* scales_down, const void* residual, void* out,
                          cudaStream_t s) {
  moe_status_t st = MOE_OK;
  if (!w_gate_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (expert_gamma && !aligned16(expert_gamma)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  if (p->wdtype == MOE_W_BF16) {
    if (scales_gate_up || scales_down) return MOE_ERR_INVALID_ARG;
  } else {
    if (!scales_gate_up || !scales_down) return MOE_ERR_INVALID_ARG;
    if (!aligned16(scales_gate_up) || !aligned16(scales_down)) return MOE_ERR_INVALID_ARG;
  }
  const size_t act = (size_t)T * p->d * 2;
  if (overlap(out, act, x, act)) return MOE_ERR_INVALID_ARG;
  if (residual && residual != out && overlap(out, act, residual, act)) return MOE_ERR_INVALID_ARG;
  st = ensure_workspace(p, T, s);
  if (st != MOE_OK) return st;

  const int A = T * p->k;  // <= MOE_MAX_ASSIGNMENTS
  const bool w4 = p->wdtype == MOE_W_INT4_G128;
  const bool w8 = p->wdtype == MOE_W_FP8_E4M3;
  const bool w4f = p->wdtype == MOE_W_FP4_E2M1;
  CUtensorMap tm_wgu, tm_wd, tm_x, tm_h, tm_bgu, tm_bd;
  bool maps_ok;
  if (w4f)
    maps_ok = make_map_codes_pair(&tm_wgu, w_gate_up, (uint64_t)p->E * 2 * p->f, p->d / 2,
                                  moe::kGuHalf) &&
              make_map_codes_pair(&tm_wd, w_down, (uint64_t)p->E * p->d, p->f / 2, moe::kBM) &&
              make_map_blk(&tm_bgu, scales_gate_up, p->E, 2 * p->f, p->d / 16, moe::kGuHalf) &&
              make_map_blk(&tm_bd, scales_down, p->E, p->d, p->f / 16, moe::kBM);
  else if (w4)
    maps_ok = make_map_codes(&tm_wgu, w_gate_up, (uint64_t)p->E * 2 * p->f, p->d / 2, moe::kGuHalf) &&
              make_map_codes(&tm_wd, w_down, (uint64_t)p->E * p->d, p->f / 2, moe::kBM);
  else if (w8)
    maps_ok = make_map_fp8(&tm_wgu, w_gate_up, (uint64_t)p->E * 2 * p->f, p->d, moe::kGuHalf) &&
              make_map_fp8(&tm_wd, w_down, (uint64_t)p->E * p->d, p->f, moe::kBM);
  else
    maps_ok = make_map_bf16(&tm_wgu, w_gate_up, (uint64_t)p->E * 2 * p->f, p->d, moe::kGuHalf) &&
              make_map_bf16(&tm_wd, w_down, (uint64_t)p->E * p->d, p->f, moe::kBM);
  // x_perm and h (bf16, or fp16 on the fp8 and fp4 paths: 2-byte elements either way)
  maps_ok = maps_ok && make_map_bf16(&tm_x, p->x_perm, (uint64_t)A, p->d, moe::kBRows) &&
            make_map_bf16(&tm_h, p->h, (uint64_t)A, p->f, moe::kBRows);
  if (!maps_ok) return MOE_ERR_CUDA;

  if (!row_expert) {
    st = launch_router(p, T, x, router_w, router_gamma, router_bias, p->idx, p->w, p->gap, s,
                       w_gate_up, prefetch_bytes(p));
    if (st != MOE_OK) return st;
  }

  moe::PlanArgs pa;
  pa.T = T;
  pa.E = p->E;
  pa.k = p->k;
  pa.d = p->d;
  pa.f = p->f;
  pa.chunk = chunk_size(p, T);
  pa.idx = row_expert ? row_expert : p->idx;
  pa.offsets = p->offsets;
  pa.perm = p->perm;
  pa.slot_of = p->slot_of;
  pa.chunk_info = p->chunk_info;
  pa.ready = p->ready;
  pa.ctl = p->ctl;

  moe::GatherArgs ga;
  ga.rows = A;
  ga.d = p->d;
  ga.eps = p->eps;
  ga.gamma2 = expert_gamma;
  ga.perm = p->perm;
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.x_perm = p->x_perm;
  ga.xf16 = (w8 || w4f) ? 1 : 0;
  {
    ProfScope ps(p, MOE_K_PLAN, s);
    if (moe_launch_plan_gather(pa, ga, p->num_sms, s, p->pdl != 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  moe::ExpertArgs ea;
  ea.T = T;
  ea.E = p->E;
  ea.k = p->k;
  ea.d = p->d;
  ea.f = p->f;
  ea.perm = p->perm;
  ea.offsets = p->offsets;
  ea.chunk_info = p->chunk_info;
  ea.ready = p->ready;
  ea.h = p->h;
  ea.y = p->y;
  ea.y_bf16 = p->y_bf16;
  ea.ctl = p->ctl;
  ea.timeout_ns = (uint64_t)p->timeout_ms * 1000000ull;
  ea.test_stall = p->test_stall;
  ea.scales_gu = w4 ? static_cast<const __half*>(scales_gate_up) : nullptr;
  ea.scales_d = w4 ? static_cast<const __half*>(scales_down) : nullptr;
  // fp8: the fp32 row scales; fp4: the scale records, which open with them
  ea.rows_gu = (w8 || w4f) ? static_cast<const float*>(scales_gate_up) : nullptr;
  ea.rows_d = (w8 || w4f) ? static_cast<const float*>(scales_down) : nullptr;
  {
    ProfScope ps(p, MOE_K_EXPERT, s);
    const cudaError_t le =
        w4 ? moe_launch_expert_w4(ea, tm_wgu, tm_wd, tm_x, tm_h, p->num_sms, s, p->pdl != 0)
        : w8 ? moe_launch_expert_w8(ea, tm_wgu, tm_wd, tm_x, tm_h, p->num_sms, s, p->pdl != 0)
        : w4f ? moe_launch_expert_w4f(ea, tm_wgu, tm_wd, tm_x, tm_h, tm_bgu, tm_bd, p->num_sms, s,
                                      p->pdl != 0)
             : moe_launch_expert(ea, tm_wgu, tm_wd, tm_x, tm_h, p->num_sms, s, p->pdl != 0);
    if (le != cudaSuccess) return MOE_ERR_CUDA;
  }

  moe::CombineArgs ca;
  ca.T = T;
  ca.k = p->k;
  ca.d = p->d;
  ca.slot_of = p->slot_of;
  ca.w = row_expert ? nullptr : p->w;
  ca.y = p->y;
  ca.y_bf16 = p->y_bf16;
  ca.residual = static_cast<const __nv_bfloat16*>(residual);
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.rows = A;
  ca.ctl = p->ctl;
  {
    ProfScope ps(p, MOE_K_COMBINE, s);
    if (moe_launch_combine(ca, p->num_sms, s, p->pdl != 0) != cudaSuccess) return MOE_ERR_CUDA;
  }

  p->last_T = T;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_forward(moe_plan_t p, int T, const void* x, const float* router_w,
                         const float* router_gamma, const float* router_bias,
                         const float* expert_gamma, const void* w_gate_up, const void* w_down,
                         const void* scales_gate_up, const void* scales_down, const void* residual,
                         void* out, void* stream) {
  moe_status_t st = validate_route(p, T, x, router_w, router_gamma, router_bias);
  if (st != MOE_OK || T == 0) return st;
  return forward_impl(p, T, x, router_w, router_gamma, router_bias, nullptr, expert_gamma,
                      w_gate_up, w_down, scales_gate_up, scales_down, residual, out,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_rows(moe_plan_t p, int R, const void* x_rows, const int32_t* row_expert,
                             const float* expert_gamma, const void* w_gate_up, const void* w_down,
                             const void* scales_gate_up, const void* scales_down, void* y_rows,
                             void* stream) {
  if (!p || R < 0) return MOE_ERR_INVALID_ARG;
  if (p->k != 1) return MOE_ERR_INVALID_ARG;
  if (R == 0) return MOE_OK;
  if (!tokens_ok(p, R)) return MOE_ERR_UNSUPPORTED;
  if (!x_rows || !row_expert || !aligned16(x_rows) ||
      (reinterpret_cast<uintptr_t>(row_expert) & 3u))
    return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device(p);
  if (st != MOE_OK) return st;
  return forward_impl(p, R, x_rows, nullptr, nullptr, nullptr, row_expert, expert_gamma,
                      w_gate_up, w_down, scales_gate_up, scales_down, nullptr, y_rows,
                      static_cast<cudaStream_t>(stream));
}

moe_status_t moe_ep_dispatch(moe_plan_t p, int T, const void* x, const int32_t* idx, int n_ranks,
                             const float* expert_gamma, void* send_rows, int32_t* send_expert,
                             int32_t* pos, int32_t* send_counts, void* stream) {
  if (!p || T < 0) return MOE_ERR_INVALID_ARG;
  if (n_ranks < 1 || n_ranks > p->E || n_ranks > moe::kMaxE || p->E % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (!send_counts || (reinterpret_cast<uintptr_t>(send_counts) & 3u)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    moe_status_t st = check_device(p);
    if (st != MOE_OK) return st;
    return cudaMemsetAsync(send_counts, 0, (size_t)n_ranks * 4, s) == cudaSuccess ? MOE_OK
                                                                                    : MOE_ERR_CUDA;
  }
  if (!tokens_ok(p, T)) return MOE_ERR_UNSUPPORTED;
  if (!x || !idx || !send_rows || !send_expert || !pos) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(send_rows) || (expert_gamma && !aligned16(expert_gamma)) ||
      ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(send_expert) |
        reinterpret_cast<uintptr_t>(pos)) & 3u))
    return MOE_ERR_INVALID_ARG;
  const size_t A = (size_t)T * p->k;
  if (overlap(send_rows, A * p->d * 2, x, (size_t)T * p->d * 2)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device(p);
  if (st != MOE_OK) return st;
  st = ensure_workspace(p, T, s);
  if (st != MOE_OK) return st;
  const bool pdl = p->pdl != 0;
  const int per = p->E / n_ranks;
  // owner keys into the plan workspace, then the plan keyed by owner: pos is
  // the plan's slot of every assignment, perm the token of every send row
  if (moe_launch_ep_keys(idx, (int)A, p->E, per, p->idx, p->ctl, p->num_sms, s, pdl) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  moe::PlanArgs pa;
  pa.T = T;
  pa.E = n_ranks;
  pa.k = p->k;
  pa.d = p->d;
  pa.f = p->f;
  pa.chunk = chunk_size(p, T);
  pa.idx = p->idx;
  pa.offsets = p->offsets;
  pa.perm = p->perm;
  pa.slot_of = pos;
  pa.chunk_info = p->chunk_info;
  pa.ready = p->ready;
  pa.ctl = p->ctl;
  if (moe_launch_plan(pa, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
  moe::GatherArgs ga;
  ga.rows = (int)A;
  ga.d = p->d;
  ga.eps = p->eps;
  ga.gamma2 = expert_gamma;
  ga.perm = p->perm;
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.x_perm = static_cast<__nv_bfloat16*>(send_rows);
  ga.xf16 = 0;
  if (moe_launch_gather(ga, p->num_sms, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe_launch_ep_meta(idx, pos, p->offsets, (int)A, p->E, per, n_ranks, send_expert,
                         send_counts, p->num_sms, s, pdl) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_combine_rows(moe_plan_t p, int T, const void* y_rows, const int32_t* pos,
                              const float* w, const void* residual, void* out, void* stream) {
  if (!p || T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!tokens_ok(p, T)) return MOE_ERR_UNSUPPORTED;
  if (!y_rows || !pos || !w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_rows) || !aligned16(out) || (residual && !aligned16(residual)) ||
      ((reinterpret_cast<uintptr_t>(pos) | reinterpret_cast<uintptr_t>(w)) & 3u))
    return MOE_ERR_INVALID_ARG;
  const size_t act = (size_t)T * p->d * 2;
  const size_t A = (size_t)T * p->k;
  if (overlap(out, act, y_rows, A * p->d * 2)) return MOE_ERR_INVALID_ARG;
  if (residual && residual != out && overlap(out, act, residual, act)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device(p);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = ensure_workspace(p, 1, s);  // the status word
  if (st != MOE_OK) return st;
  moe::CombineArgs ca;
  ca.T = T;
  ca.k = p->k;
  ca.d = p->d;
  ca.slot_of = pos;
  ca.w = w;
  ca.y = y_rows;
  ca.y_bf16 = 1;
  ca.residual = static_cast<const __nv_bfloat16*>(residual);
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.rows = (int)A;
  ca.ctl = p->ctl;
  return moe_launch_combine(ca, p->num_sms, s, p->pdl != 0) == cudaSuccess ? MOE_OK
                                                                           : MOE_ERR_CUDA;
}

moe_status_t moe_forward_host(moe_plan_t p, int T, const void* x_host, const float* router_w,
                              const float* router_gamma, const float* router_bias,
                              const float* expert_gamma, const void* w_gate_up, const void* w_down,
                              const void* scales_gate_up, const void* scales_down,
                              const void* residual_host, void* out_host, void* stream) {
  if (!p || T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!tokens_ok(p, T)) return MOE_ERR_UNSUPPORTED;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device(p);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = ensure_workspace(p, T, s);
  if (st != MOE_OK) return st;
  const size_t act = (size_t)T * p->d * 2;
  if (cudaMemcpyAsync(p->x_dev, x_host, act, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (residual_host &&
      cudaMemcpyAsync(p->res_dev, residual_host, act, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = moe_forward(p, T, p->x_dev, router_w, router_gamma, router_bias, expert_gamma, w_gate_up,
                   w_down,
                   scales_gate_up, scales_down, residual_host ? p->res_dev : nullptr, p->out_dev,
                   stream);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, p->out_dev, act, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_plan_routing(moe_plan_t p, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                              void* stream) {
  if (!p || !p->ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t A = (size_t)p->last_T * p->k;
  if (offsets && cudaMemcpyAsync(offsets, p->offsets, (p->E + 1) * 4, cudaMemcpyDeviceToDevice,
                                 s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (perm && A && cudaMemcpyAsync(perm, p->perm, A * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (slot_of && A &&
      cudaMemcpyAsync(slot_of, p->slot_of, A * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_plan_sync_status(moe_plan_t p, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int status = 0;
  // The plan's own word first, then the word its last noalloc call left in
  // the library's array; each is cleared once read.
  Ctl* words[2] = {p->ws ? p->ctl : nullptr, p->noalloc_ctl};
  for (Ctl* w : words) {
    if (!w) continue;
    int c[2] = {0, 0};
    if (cudaMemcpy(c, w, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (c[0] != 0) {
      if (status == 0) status = c[0];
      const int zero[2] = {0, 0};
      if (cudaMemcpy(w, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
  }
  if (p->ws && !p->guards.empty()) {
    unsigned char g[kGuardBytes];
    for (size_t off : p->guards) {
      if (cudaMemcpy(g, static_cast<char*>(p->ws) + off, kGuardBytes, cudaMemcpyDeviceToHost) !=
          cudaSuccess)
        return MOE_ERR_CUDA;
      for (size_t i = 0; i < kGuardBytes; ++i)
        if (g[i] != (unsigned char)kGuardByte) {
          if (status == 0) status = MOE_ERR_DEVICE_CHECK;
          break;
        }
    }
  }
  return static_cast<moe_status_t>(status);
}

moe_status_t moe_plan_profile(moe_plan_t p, int kernel, double* total_ms, int* launches) {
  if (!p || !total_ms || !launches || kernel < 0 || kernel >= MOE_K_COUNT)
    return MOE_ERR_INVALID_ARG;
  double tot = 0.0;
  int n = 0;
  std::vector<ProfRec> keep;
  for (const ProfRec& r : p->prof) {
    if (r.kernel != kernel) {
      keep.push_back(r);
      continue;
    }
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return MOE_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return MOE_ERR_CUDA;
    tot += ms;
    ++n;
    p->ev_pool.push_back(r.start);
    p->ev_pool.push_back(r.stop);
  }
  p->prof.swap(keep);
  *total_ms = tot;
  *launches = n;
  return MOE_OK;
}

void moe_plan_destroy(moe_plan_t p) {
  if (!p) return;
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != p->device) cudaSetDevice(p->device);
  if (p->ws) {
    cudaDeviceSynchronize();
    cudaFree(p->ws);
  }
  for (const ProfRec& r : p->prof) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  for (cudaEvent_t e : p->ev_pool) cudaEventDestroy(e);
  if (prev >= 0 && prev != p->device) cudaSetDevice(prev);
  delete p;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_forward_noalloc: the moe_forward launch sequence with every
// intermediate carved from one file-scope device array, for callers that
// cannot allocate device memory (a host that pre-assigns all GPU memory, or a
// loop that must never enter the allocator).  Nothing here calls cudaMalloc,
// cudaFree or any allocating routine.

static __device__ __align__(256) unsigned char moe_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[128] = {};

// Device address of the array on device `dev` (must be current).  In host
// code the array's name is only a stand-in, so it is never passed to a kernel
// directly.  The address is looked up again on every call whose stream is
// not capturing (a device reset reloads the module and moves the array);
// during a capture, which must not trigger a module load, the last address
// looked up on the device is used.
void* noalloc_scratch(int dev, cudaStream_t s) {
  if (dev < 0 || dev >= 128) return nullptr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, moe_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" moe_status_t moe_forward_noalloc(moe_plan_t p, int T, const void* x,
                                            const float* router_w, const float* router_gamma,
                                            const float* router_bias, const float* expert_gamma,
                                            const void* w_gate_up,
                                            const void* w_down, const void* scales_gate_up,
                                            const void* scales_down, const void* residual,
                                            void* out, int32_t* status_out, void* stream) {
  moe_status_t st = validate_route(p, T, x, router_w, router_gamma, router_bias);
  if (st != MOE_OK || T == 0) return st;
  if (!w_gate_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (expert_gamma && !aligned16(expert_gamma)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)) return MOE_ERR_INVALID_ARG;
  if (p->wdtype == MOE_W_BF16) {
    if (scales_gate_up || scales_down) return MOE_ERR_INVALID_ARG;
  } else {
    return MOE_ERR_UNSUPPORTED;
  }
  const size_t act = (size_t)T * p->d * 2;
  if (overlap(out, act, x, act)) return MOE_ERR_INVALID_ARG;
  if (residual && residual != out && overlap(out, act, residual, act)) return MOE_ERR_INVALID_ARG;

  // Carve the intermediates for T tokens; refuse what does not fit.
  const size_t A = (size_t)T * p->k;
  const size_t MC = max_chunks(p->E, T, p->k);
  size_t sz = 0;
  auto take = [&](size_t bytes) {
    size_t o = sz;
    sz += align256(bytes);
    return o;
  };
  const size_t o_ctl = take(sizeof(Ctl));
  const size_t o_idx = take(A * 4), o_w = take(A * 4), o_gap = take((size_t)T * 4);
  const size_t o_perm = take(A * 4), o_slot = take(A * 4), o_off = take((size_t)(p->E + 1) * 4);
  const size_t o_ci = take(MC * 16), o_rd = take(MC * 4);
  const size_t o_xp = take(A * p->d * 2);
  const size_t o_h = take(A * p->f * 2), o_y = take(A * p->d * 4);
  if (sz > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* b = static_cast<char*>(noalloc_scratch(p->device, s));
  if (!b) return MOE_ERR_CUDA;
  Ctl* ctl = reinterpret_cast<Ctl*>(b + o_ctl);
  int32_t* idx = reinterpret_cast<int32_t*>(b + o_idx);
  float* w = reinterpret_cast<float*>(b + o_w);
  float* gap = reinterpret_cast<float*>(b + o_gap);
  int32_t* perm = reinterpret_cast<int32_t*>(b + o_perm);
  int32_t* slot_of = reinterpret_cast<int32_t*>(b + o_slot);
  int32_t* offsets = reinterpret_cast<int32_t*>(b + o_off);
  int4* chunk_info = reinterpret_cast<int4*>(b + o_ci);
  int32_t* ready = reinterpret_cast<int32_t*>(b + o_rd);
  __nv_bfloat16* x_perm = reinterpret_cast<__nv_bfloat16*>(b + o_xp);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(b + o_h);
  float* y = reinterpret_cast<float*>(b + o_y);

  CUtensorMap tm_wgu, tm_wd, tm_x, tm_h;
  if (!make_map_bf16(&tm_wgu, w_gate_up, (uint64_t)p->E * 2 * p->f, p->d, moe::kGuHalf) ||
      !make_map_bf16(&tm_wd, w_down, (uint64_t)p->E * p->d, p->f, moe::kBM) ||
      !make_map_bf16(&tm_x, x_perm, (uint64_t)A, p->d, moe::kBRows) ||
      !make_map_bf16(&tm_h, h, (uint64_t)A, p->f, moe::kBRows))
    return MOE_ERR_CUDA;

  // The status word must start at zero; the plan kernel resets the scheduler
  // counters and chunk tables itself on every call.
  if (cudaMemsetAsync(ctl, 0, sizeof(Ctl), s) != cudaSuccess) return MOE_ERR_CUDA;
  p->noalloc_ctl = ctl;  // moe_plan_sync_status reads this call's status here

  {
    const bool prof = p->profile != 0;
    p->profile = 0;  // no event records on this path
    const moe_status_t rs =
        launch_router(p, T, x, router_w, router_gamma, router_bias, idx, w, gap, s, w_gate_up,
                      prefetch_bytes(p), ctl);
    p->profile = prof;
    if (rs != MOE_OK) return rs;
  }

  moe::PlanArgs pa;
  pa.T = T;
  pa.E = p->E;
  pa.k = p->k;
  pa.d = p->d;
  pa.f = p->f;
  pa.chunk = chunk_size(p, T);
  pa.idx = idx;
  pa.offsets = offsets;
  pa.perm = perm;
  pa.slot_of = slot_of;
  pa.chunk_info = chunk_info;
  pa.ready = ready;
  pa.ctl = ctl;

  moe::GatherArgs ga;
  ga.rows = (int)A;
  ga.d = p->d;
  ga.eps = p->eps;
  ga.gamma2 = expert_gamma;
  ga.perm = perm;
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.x_perm = x_perm;
  ga.xf16 = 0;
  if (moe_launch_plan_gather(pa, ga, p->num_sms, s, p->pdl != 0) != cudaSuccess)
    return MOE_ERR_CUDA;

  moe::ExpertArgs ea;
  ea.T = T;
  ea.E = p->E;
  ea.k = p->k;
  ea.d = p->d;
  ea.f = p->f;
  ea.perm = perm;
  ea.offsets = offsets;
  ea.chunk_info = chunk_info;
  ea.ready = ready;
  ea.h = h;
  ea.y = y;
  ea.y_bf16 = p->y_bf16;
  ea.ctl = ctl;
  ea.timeout_ns = (uint64_t)p->timeout_ms * 1000000ull;
  ea.test_stall = p->test_stall;
  ea.scales_gu = nullptr;
  ea.scales_d = nullptr;
  ea.rows_gu = nullptr;
  ea.rows_d = nullptr;
  if (moe_launch_expert(ea, tm_wgu, tm_wd, tm_x, tm_h, p->num_sms, s, p->pdl != 0) !=
      cudaSuccess)
    return MOE_ERR_CUDA;

  moe::CombineArgs ca;
  ca.T = T;
  ca.k = p->k;
  ca.d = p->d;
  ca.slot_of = slot_of;
  ca.w = w;
  ca.y = y;
  ca.y_bf16 = p->y_bf16;
  ca.residual = static_cast<const __nv_bfloat16*>(residual);
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.rows = (int)A;
  ca.ctl = ctl;
  if (moe_launch_combine(ca, p->num_sms, s, p->pdl != 0) != cudaSuccess) return MOE_ERR_CUDA;

  if (status_out && cudaMemcpyAsync(status_out, &ctl->status, sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
