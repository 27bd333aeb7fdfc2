// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument
// validation, TMA descriptor construction, persistent-grid sizing and kernel
// launches.  Every step of the computation runs in the kernels; this file
// only prepares launches.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fa.h"
#include "bwd_kernel.cuh"
#include "fwd_kernel.cuh"

namespace {

// Per-device status word the kernels OR error bits into.
__device__ int g_fa_status;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int major = 0;
  int minor = 0;
  int* status = nullptr;  // device address of g_fa_status
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Fills *info for the current device (once per device).
int device_info(DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_LAUNCH;
    if (d.major != 10) return FA_ERR_ARCH;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_fa_status) != cudaSuccess)
      return FA_ERR_LAUNCH;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_LAUNCH;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *info = &d;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
  const long long elems = static_cast<long long>(B) * H * N * d;
  if (elems >= (1ll << 31)) return FA_ERR_SHAPE;
  return FA_OK;
}

int check_scale(float scale) {
  if (!std::isfinite(scale) || scale < 0.f) return FA_ERR_ARG;
  return FA_OK;
}

// 3-D view [B*H][N][d] of a bf16 tensor, boxes of 128 rows x 64 columns with
// 128-byte swizzle.  Rows past N read as zero (the third dimension keeps
// one head's ragged tail from reading the next head's rows).
int make_tmap(CUtensorMap* m, const void* base, int BH, int N, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

int fwd_units(int B, int H, int N) { return B * H * ((N + 255) / 256); }

template <int D, bool CAUSAL>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const fa::FwdParams& p, int ctas, cudaStream_t stream) {
  auto kern = fa::fa_fwd_kernel<D, CAUSAL>;
  const int smem = fa::FwdLayout<D>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  kern<<<ctas, 384, smem, stream>>>(tq, tk, tv, p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace

extern "C" {

const char* fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_SHAPE: return "invalid shape (B, H, N must be >= 1 and B*H*N*d < 2^31)";
    case FA_ERR_UNSUPPORTED_D: return "unsupported head dimension (d must be 64 or 128)";
    case FA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "workspace smaller than fa_bwd_workspace_size()";
    case FA_ERR_LAUNCH: return "the CUDA runtime rejected a launch or query";
    case FA_ERR_TIMEOUT: return "a device-side wait timed out";
    case FA_ERR_DEVICE_ASSERT: return "a device-side consistency check failed";
    case FA_ERR_ARCH: return "the current device is not an sm_100 (B200-class) GPU";
    case FA_ERR_ARG: return "invalid argument (scale must be finite and >= 0; grad_dtype 0 or 1)";
    default: return "unknown status";
  }
}

int fa_launch_shape(int pass, int B, int H, int N, int d, int causal, int* ctas, int* work_units) {
  (void)causal;
  if (!ctas || !work_units) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  DeviceInfo* info = nullptr;
  s = device_info(&info);
  if (s != FA_OK) return s;
  const int units = pass == 0 ? fwd_units(B, H, N) : fa::bwd_units(B, H, N);
  *work_units = units;
  *ctas = units < info->sms ? units : info->sms;
  return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_ALIGN;
  DeviceInfo* info = nullptr;
  if ((s = device_info(&info)) != FA_OK) return s;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (make_tmap(&tq, q, BH, N, d) != FA_OK || make_tmap(&tk, k, BH, N, d) != FA_OK ||
      make_tmap(&tv, v, BH, N, d) != FA_OK)
    return FA_ERR_LAUNCH;
  fa::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.BH = BH;
  p.N = N;
  p.n_qt2 = (N + 255) / 256;
  p.n_units = fwd_units(B, H, N);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = info->status;
  const int ctas = p.n_units < info->sms ? p.n_units : info->sms;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_fwd<64, true>(tq, tk, tv, p, ctas, st)
                  : launch_fwd<64, false>(tq, tk, tv, p, ctas, st);
  return causal ? launch_fwd<128, true>(tq, tk, tv, p, ctas, st)
                : launch_fwd<128, false>(tq, tk, tv, p, ctas, st);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != FA_OK) return 0;
  return fa::bwd_workspace_bytes(B, H, N, d);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
           const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
           int causal, void* workspace, size_t workspace_bytes, int grad_dtype,
           fa_stream_t stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (grad_dtype != 0 && grad_dtype != 1) return FA_ERR_ARG;
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (workspace_bytes < fa::bwd_workspace_bytes(B, H, N, d)) return FA_ERR_WORKSPACE;
  DeviceInfo* info = nullptr;
  if ((s = device_info(&info)) != FA_OK) return s;
  return fa::launch_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal != 0,
                        workspace, grad_dtype, info->sms, info->status,
                        reinterpret_cast<cudaStream_t>(stream), g_encode);
}

int fa_check_device_errors(fa_stream_t stream) {
  DeviceInfo* info = nullptr;
  int s = device_info(&info);
  if (s != FA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_LAUNCH;
  int host = 0;
  if (cudaMemcpyFromSymbol(&host, g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_LAUNCH;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_LAUNCH;
  if (host & fa::kDevTimeout) return FA_ERR_TIMEOUT;
  if (host & fa::kDevAssert) return FA_ERR_DEVICE_ASSERT;
  return FA_OK;
}

}  // extern "C"
