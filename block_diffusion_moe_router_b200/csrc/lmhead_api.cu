// lmhead_api.cu -- C ABI of the lm_head / entropy-bound acceptance step
// (declared in moe.h): argument checks, workspace, tensor maps, launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "moe.h"

struct moe_lmhead_s {
  int V, d;
  int device;
  int num_sms;
  int timeout_ms;
  int cap_T;
  void* ws;  // Ctl, then the per-(token, tile) partials
  moe::Ctl* ctl;
  float4* part;
  int profile;  // record CUDA events around the GEMM launch
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof;
};

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// bf16 [rows, cols] row-major, 128-byte swizzle, box = box_rows x 64 columns.
bool map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

constexpr int kMaxT = 4096;

}  // namespace

extern "C" {

moe_status_t moe_lmhead_create(int V, int d, moe_lmhead_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (V < 1 || V > (1 << 24) || d < 64 || d > 8192 || d % 64 != 0) return MOE_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe_lmhead_s* p = new moe_lmhead_s();
  p->V = V;
  p->d = d;
  p->device = dev;
  p->num_sms = sms;
  p->timeout_ms = 1000;
  p->cap_T = 0;
  p->ws = nullptr;
  p->ctl = nullptr;
  p->part = nullptr;
  p->profile = 0;
  *out = p;
  return MOE_OK;
}

moe_status_t moe_lmhead_forward(moe_lmhead_t p, int T, const void* h, const void* w,
                                float temperature, float softcap, const uint8_t* masked,
                                float entropy_bound, int32_t* token_out, float* entropy_out,
                                float* logz_out, uint8_t* accept_out, void* stream) {
  if (!p || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!h || !w || !token_out || !entropy_out || !accept_out) return MOE_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(w, 16) || !aligned(token_out, 4) || !aligned(entropy_out, 4) ||
      (logz_out && !aligned(logz_out, 4)))
    return MOE_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !std::isfinite(temperature) || !(softcap >= 0.f) ||
      !std::isfinite(softcap) || !(entropy_bound >= 0.f))
    return MOE_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev != p->device) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int VT = (p->V + 255) / 256;  // partials per token: one per 256-row tile
  if (!p->ws || T > p->cap_T) {
    // stream-ordered growth: the host does not wait for earlier calls
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return MOE_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return MOE_ERR_UNSUPPORTED;
    int cap = p->cap_T > 0 ? p->cap_T : 64;
    while (cap < T) cap *= 2;
    if (cap > kMaxT) cap = kMaxT;
    const size_t bytes = 256 + (size_t)cap * VT * sizeof(float4) + (size_t)cap * 4;
    if (p->ws) {
      if (cudaFreeAsync(p->ws, s) != cudaSuccess) return MOE_ERR_CUDA;
      p->ws = nullptr;
      p->cap_T = 0;
    }
    if (cudaMallocAsync(&p->ws, bytes, s) != cudaSuccess) {
      cudaGetLastError();
      p->ws = nullptr;
      p->cap_T = 0;
      return MOE_ERR_ALLOC;
    }
    p->ctl = static_cast<moe::Ctl*>(p->ws);
    p->part = reinterpret_cast<float4*>(static_cast<uint8_t*>(p->ws) + 256);
    p->cap_T = cap;
    if (cudaMemsetAsync(p->ctl, 0, sizeof(moe::Ctl), s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // logZ goes to the caller's array, else to scratch after the partials
  float* logz = logz_out ? logz_out
                         : reinterpret_cast<float*>(p->part + (size_t)p->cap_T * VT);
  CUtensorMap tm_w, tm_h;
  if (!map_bf16(&tm_w, w, (uint64_t)p->V, (uint64_t)p->d, moe::kBM) ||
      !map_bf16(&tm_h, h, (uint64_t)T, (uint64_t)p->d, 128))
    return MOE_ERR_CUDA;
  moe::LmHeadArgs a;
  a.T = T;
  a.V = p->V;
  a.d = p->d;
  a.inv_temp = 1.0f / temperature;
  a.softcap = softcap;
  a.bound = entropy_bound;
  a.masked = masked;
  a.part = p->part;
  a.token = token_out;
  a.entropy = entropy_out;
  a.logz = logz;
  a.accept = accept_out;
  a.ctl = p->ctl;
  a.timeout_ns = (uint64_t)p->timeout_ms * 1000000ull;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (p->profile) {
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess)
      return MOE_ERR_CUDA;
    cudaEventRecord(e0, s);
  }
  if (moe_launch_lmhead_gemm(a, tm_w, tm_h, p->num_sms, s, !p->profile) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->profile) {
    cudaEventRecord(e1, s);
    p->prof.emplace_back(e0, e1);
  }
  return moe_launch_lmhead_tail(a, s, !p->profile) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_lmhead_set_profile(moe_lmhead_t p, int on) {
  if (!p) return MOE_ERR_INVALID_ARG;
  p->profile = on != 0;
  return MOE_OK;
}

moe_status_t moe_lmhead_profile(moe_lmhead_t p, double* gemm_ms, int* launches) {
  if (!p || !gemm_ms || !launches) return MOE_ERR_INVALID_ARG;
  double tot = 0.0;
  for (auto& e : p->prof) {
    float ms = 0.f;
    if (cudaEventSynchronize(e.second) != cudaSuccess ||
        cudaEventElapsedTime(&ms, e.first, e.second) != cudaSuccess)
      return MOE_ERR_CUDA;
    tot += ms;
    cudaEventDestroy(e.first);
    cudaEventDestroy(e.second);
  }
  *gemm_ms = tot;
  *launches = (int)p->prof.size();
  p->prof.clear();
  return MOE_OK;
}

moe_status_t moe_lmhead_sync_status(moe_lmhead_t p, void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  if (!p->ws) return MOE_OK;
  moe::Ctl c;
  if (cudaMemcpy(&c, p->ctl, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (c.status != 0) {
    const int zero[2] = {0, 0};
    if (cudaMemcpy(p->ctl, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return static_cast<moe_status_t>(c.status);
}

void moe_lmhead_destroy(moe_lmhead_t p) {
  if (!p) return;
  for (auto& e : p->prof) {
    cudaEventDestroy(e.first);
    cudaEventDestroy(e.second);
  }
  if (p->ws) {
    cudaDeviceSynchronize();
    cudaFree(p->ws);
  }
  delete p;
}

}  // extern "C"
