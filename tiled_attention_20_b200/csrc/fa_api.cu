// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument
// validation, TMA descriptor construction, persistent-grid and split
// planning, and kernel launches.  Every step of the computation runs in the
// kernels (the *_kernel.cuh headers); this file only prepares launches, and
// holds the one-thread kernel of the failure-detection self-test.
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fa.h"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "dq_kernel.cuh"
#include "gemm_kernel.cuh"
#include "fwd_kernel.cuh"

namespace {

// Per-device status word the kernels OR error bits into.
__device__ int g_fa_status;

// Failure-detection self-test: one thread waits, with the given bound, on an
// mbarrier that nothing will ever arrive on.  The bounded wait gives up,
// latches the timeout bit and the kernel returns normally.
__global__ void fa_selftest_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    fa::fence_barrier_init();
    fa::mbar_wait(&bar, 0, status, limit_ns);  // phase 0 never completes
  }
}

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

// ---------------------------------------------------------------- tracing
// Opt-in per-kernel timing: while enabled, every launch is bracketed by a
// pair of CUDA events on its stream.  On a stream that is being captured into
// a CUDA graph the events are recorded as external event nodes, so every
// replay of the graph stamps them (a plain record during capture would only
// order the captured work).
enum { kKernFwd = 0, kKernBwdPrep = 1, kKernBwd = 2, kKernBwdConvert = 3, kKernDq = 4,
       kKernDecode = 5, kKernGemm = 6, kKernGemmPack = 7, kNumKernels = 8 };
const char* const kKernelNames[kNumKernels] = {"fa_fwd_kernel", "fa_bwd_prep", "fa_bwd_kernel",
                                               "fa_bwd_dq_convert", "fa_dq_kernel",
                                               "fa_decode_kernel", "fa_gemm_kernel",
                                               "fa_gemm_pack"};
struct TraceRec {
  int kernel;
  int device;
  cudaEvent_t start, stop;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
unsigned g_trace_mask = 0;  // bit k set: kernel id k is bracketed
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool[kMaxDevices];
size_t g_event_used[kMaxDevices];

cudaEvent_t trace_event(int dev) {
  if (g_event_used[dev] == g_event_pool[dev].size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_event_pool[dev].push_back(e);
  }
  return g_event_pool[dev][g_event_used[dev]++];
}

// Brackets one launch when tracing is on.
class LaunchTrace {
 public:
  LaunchTrace(int kernel, cudaStream_t s) : stream_(s) {
    std::lock_guard<std::mutex> lock(g_trace_mu);
    if (!g_trace_on || !((g_trace_mask >> kernel) & 1u)) return;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
    rec_.kernel = kernel;
    rec_.device = dev;
    rec_.start = trace_event(dev);
    rec_.stop = trace_event(dev);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return;
    flags_ = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    if (rec_.start && rec_.stop && cudaEventRecordWithFlags(rec_.start, s, flags_) == cudaSuccess)
      active_ = true;
  }
  ~LaunchTrace() {
    if (!active_) return;
    std::lock_guard<std::mutex> lock(g_trace_mu);
    if (cudaEventRecordWithFlags(rec_.stop, stream_, flags_) == cudaSuccess) g_trace.push_back(rec_);
  }

 private:
  cudaStream_t stream_;
  TraceRec rec_{};
  unsigned flags_ = cudaEventRecordDefault;
  bool active_ = false;
};

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

int make_tmap_rows(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows);

// Forward schedule (fwd_item).  Causal heads with an even number P >= 8 of
// tile pairs are dealt as merged complementary pairs, except for the last
// R = (P / 2) << shift heads, left as single pairs; shift is the smallest
// that gives those at least two rounds of the persistent grid.  Returns h1
// (the number of merged heads) and sets the decode's divisor and shift.
int fwd_schedule(int BH, int N, int causal, int sms, int* item_div, int* tail_shift) {
  const int P = (N + 255) / 256;
  *item_div = BH;
  *tail_shift = 0;
  if (!causal || P < 8 || (P & 1)) return 0;
  const int half = P / 2;
  int shift = 0;
  while ((static_cast<long long>(half) << shift) * P < 2LL * sms) ++shift;
  const long long R = static_cast<long long>(half) << shift;
  if (BH <= R) return 0;
  *item_div = half;
  *tail_shift = shift;
  return BH - static_cast<int>(R);
}
int fwd_items(int BH, int N, int h1) {
  const int P = (N + 255) / 256;
  return h1 * (P / 2) + (BH - h1) * P;  // h1 > 0 only when P is even
}

template <int D, bool CAUSAL, bool FP8 = false>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const fa::FwdParams& p, int ctas, cudaStream_t stream) {
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, FP8>;
  const int smem = fa::FwdLayout<D, FP8>::kSmemBytes;
  // The kernel moves registers between warpgroups; its split assumes the
  // launch allocation it was compiled for.  Refuse to launch otherwise
  // (a larger request than the block holds would never be granted).
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess || attr.numRegs != fa::kFwdLaunchRegs)
    return FA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  LaunchTrace trace(kKernFwd, stream);
  kern<<<ctas, 384, smem, stream>>>(tq, tk, tv, p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// ---------------------------------------------------------------- backward launches
// 3-D view [B*H][N][d] of a bf16 tensor, boxes of `box_rows` rows x 64
// columns with 128-byte swizzle.  Rows past N read as zero (the third
// dimension keeps one head's ragged tail from reading the next head's rows).
int make_tmap_rows(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

// 3-D view [B*H][N][d] of an 8-bit tensor with d = 128: boxes of `box_rows`
// rows x 128 columns (128 bytes, the 128-byte swizzle span).
int make_tmap_rows_u8(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N) * d};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

template <int D, bool CAUSAL, bool DQ>
int launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const CUtensorMap& tdo, const fa::BwdParams& p, int ctas,
                    cudaStream_t stream) {
  auto kern = fa::fa_bwd_kernel<D, CAUSAL, DQ>;
  const int smem = fa::BwdLayout<D>::kSmemBytes;
  // The register split between warpgroups assumes this launch allocation.
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess || attr.numRegs != fa::kBwdLaunchRegs)
    return FA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  LaunchTrace trace(kKernBwd, stream);
  kern<<<ctas, 512, smem, stream>>>(tq, tk, tv, tdo, p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

template <int D, bool CAUSAL>
int launch_dq(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
              const CUtensorMap& tdo, const fa::DqParams& p, int ctas, cudaStream_t stream) {
  auto kern = fa::fa_dq_kernel<D, CAUSAL>;
  const int smem = fa::DqLayout<D>::kSmemBytes;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess || attr.numRegs != fa::kDqLaunchRegs)
    return FA_ERR_LAUNCH;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  LaunchTrace trace(kKernDq, stream);
  kern<<<ctas, 384, smem, stream>>>(tq, tk, tv, tdo, p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// Backward: preprocess, then either the atomic main kernel (dQ, dK, dV) and
// the dQ conversion, or (deterministic) the main kernel without dQ and the
// query-block-major dQ kernel.
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
               float scale, bool causal, void* workspace, int grad_dtype, int sms, int* status,
               cudaStream_t stream, bool deterministic = false) {
  const int BH = B * H;
  const size_t npad = fa::bwd_npad(N);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + fa::round256(static_cast<size_t>(BH) * N * d * 4));
  float* dvec = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(lse2) +
                                         fa::round256(static_cast<size_t>(BH) * npad * 4));
  int* sched = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(dvec) +
                                      fa::round256(static_cast<size_t>(BH) * npad * 4));
  CUtensorMap tq, tk, tv, tdo;
  if (make_tmap_rows(&tq, q, BH, N, d, 64) != FA_OK || make_tmap_rows(&tdo, dO, BH, N, d, 64) != FA_OK ||
      make_tmap_rows(&tk, k, BH, N, d, 128) != FA_OK || make_tmap_rows(&tv, v, BH, N, d, 128) != FA_OK)
    return FA_ERR_LAUNCH;
  // 1. D, lse * log2(e), zeroed dQ accumulator
  {
    const long long threads = static_cast<long long>(BH) * npad * (d / 8);
    const int blocks = static_cast<int>((threads + 255) / 256);
    LaunchTrace trace(kKernBwdPrep, stream);
    if (d == 64)
      fa::fa_bwd_prep<64><<<blocks, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2,
          dvec, dq_acc, sched, BH, N, static_cast<int>(npad), deterministic ? 0 : 1, status);
    else
      fa::fa_bwd_prep<128><<<blocks, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2,
          dvec, dq_acc, sched, BH, N, static_cast<int>(npad), deterministic ? 0 : 1, status);
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  }
  // 2. tensor-core main kernel
  fa::BwdParams p;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = dq_acc;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.sched = sched;
  p.BH = BH;
  p.N = N;
  p.Npad = static_cast<int>(npad);
  p.nq = (N + 63) / 64;
  p.nkv = (N + 127) / 128;
  p.n_units = BH * p.nkv;
  p.group_heads = fa::bwd_group_heads(N, d);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  p.grad_f32 = grad_dtype;
  p.status = status;
  const int ctas = p.n_units < sms ? p.n_units : sms;
  int rc;
  if (deterministic) {
    if (d == 64)
      rc = causal ? launch_bwd_main<64, true, false>(tq, tk, tv, tdo, p, ctas, stream)
                  : launch_bwd_main<64, false, false>(tq, tk, tv, tdo, p, ctas, stream);
    else
      rc = causal ? launch_bwd_main<128, true, false>(tq, tk, tv, tdo, p, ctas, stream)
                  : launch_bwd_main<128, false, false>(tq, tk, tv, tdo, p, ctas, stream);
    if (rc != FA_OK) return rc;
    CUtensorMap tq128, tdo128;
    if (make_tmap_rows(&tq128, q, BH, N, d, 128) != FA_OK ||
        make_tmap_rows(&tdo128, dO, BH, N, d, 128) != FA_OK)
      return FA_ERR_LAUNCH;
    fa::DqParams dp;
    dp.dq = dq;
    dp.lse2 = lse2;
    dp.dvec = dvec;
    dp.BH = BH;
    dp.N = N;
    dp.Npad = static_cast<int>(npad);
    dp.nqt = (N + 127) / 128;
    dp.n_units = BH * dp.nqt;
    dp.scale_log2 = scale * 1.4426950408889634f;
    dp.scale = scale;
    dp.grad_f32 = grad_dtype;
    dp.status = status;
    const int dctas = dp.n_units < sms ? dp.n_units : sms;
    if (d == 64)
      return causal ? launch_dq<64, true>(tq128, tk, tv, tdo128, dp, dctas, stream)
                    : launch_dq<64, false>(tq128, tk, tv, tdo128, dp, dctas, stream);
    return causal ? launch_dq<128, true>(tq128, tk, tv, tdo128, dp, dctas, stream)
                  : launch_dq<128, false>(tq128, tk, tv, tdo128, dp, dctas, stream);
  }
  if (d == 64)
    rc = causal ? launch_bwd_main<64, true, true>(tq, tk, tv, tdo, p, ctas, stream)
                : launch_bwd_main<64, false, true>(tq, tk, tv, tdo, p, ctas, stream);
  else
    rc = causal ? launch_bwd_main<128, true, true>(tq, tk, tv, tdo, p, ctas, stream)
                : launch_bwd_main<128, false, true>(tq, tk, tv, tdo, p, ctas, stream);
  if (rc != FA_OK) return rc;
  // 3. dQ = scale * accumulator
  {
    const long long n8 = static_cast<long long>(BH) * N * d / 8;
    const int blocks = static_cast<int>((n8 + 255) / 256);
    LaunchTrace trace(kKernBwdConvert, stream);
    fa::fa_bwd_dq_convert<<<blocks, 256, 0, stream>>>(dq_acc, dq, n8, scale, grad_dtype);
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

}  // namespace

// ---------------------------------------------------------------- backward without allocation
// Scratch for fa_bwd_noalloc: a fixed array in the library's device image,
// present on every GPU that loads the library until the process exits.
// Host code must not hand this symbol to a kernel: on the host it names a
// stand-in, not device memory.  Its device address is looked up per device.
static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[FA_BWD_NOALLOC_MAX_SCRATCH];

namespace {
void* g_noalloc_addr[kMaxDevices];  // device address of the scratch, per device

// The scratch's device address on the current device, looked up on the first
// call there (with that device current) and remembered.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return FA_ERR_LAUNCH;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return FA_OK;
}
// ---------------------------------------------------------------- decode
constexpr int kDecMaxNq = 8;

int decode_max_chunk_tiles(int nqp) { return (4096 / nqp) / fa::kDecTileKeys; }

int decode_plan(int BH, int Nq, int Nk, int num_splits, int sms, int per_sm, int* splits,
                int* chunk) {
  const int tiles = (Nk + fa::kDecTileKeys - 1) / fa::kDecTileKeys;
  const int max_ct = decode_max_chunk_tiles(fa::dec_nqp(Nq));
  int ct;
  if (num_splits > 0) {
    ct = (tiles + num_splits - 1) / num_splits;
    ct = ct < 1 ? 1 : (ct > max_ct ? max_ct : ct);
  } else {
    // Wave quantization: the cost of a chunk size is the number of waves of
    // CTAs times the tiles each CTA streams (+1 for its fixed work).
    const long long slots = static_cast<long long>(sms) * per_sm;
    long long best = -1;
    ct = 1;
    const int top = tiles < max_ct ? tiles : max_ct;
    for (int c = 1; c <= top; ++c) {
      const long long sp = (tiles + c - 1) / c;
      const long long waves = (sp * BH + slots - 1) / slots;
      const long long cost = waves * (c + 1);
      if (best < 0 || cost <= best) {
        best = cost;
        ct = c;
      }
    }
  }
  *splits = (tiles + ct - 1) / ct;
  *chunk = ct * fa::kDecTileKeys;
  return FA_OK;
}

int check_decode_shape(int B, int H, int Nq, int Nk, int ld_kv, int d) {
  if (B < 1 || H < 1 || Nq < 1 || Nq > kDecMaxNq || Nk < 1 || ld_kv < Nk) return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
  if (static_cast<long long>(B) * H > 65535) return FA_ERR_SHAPE;
  return FA_OK;
}

size_t decode_ws_bytes(int BH, int Nq, int d, int splits) {
  if (splits <= 1) return 0;
  const size_t nqp = static_cast<size_t>(fa::dec_nqp(Nq));
  const size_t slots = static_cast<size_t>(BH) * splits * nqp;
  return fa::round256(static_cast<size_t>(BH) * 4) + fa::round256(slots * d * 4) +
         fa::round256(slots * 2 * 4);
}

template <int D, int NQP>
int decode_occupancy(int* per_sm) {
  auto kern = fa::fa_decode_kernel<D, NQP>;
  const int smem = fa::DecLayout<D, NQP>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, kern, fa::kDecThreads, smem) !=
          cudaSuccess ||
      *per_sm < 1)
    return FA_ERR_LAUNCH;
  return FA_OK;
}

int decode_occupancy_any(int d, int Nq, int* per_sm) {
  switch (fa::dec_nqp(Nq) * (d == 64 ? 1 : -1)) {
    case 1: return decode_occupancy<64, 1>(per_sm);
    case 2: return decode_occupancy<64, 2>(per_sm);
    case 4: return decode_occupancy<64, 4>(per_sm);
    case 8: return decode_occupancy<64, 8>(per_sm);
    case -1: return decode_occupancy<128, 1>(per_sm);
    case -2: return decode_occupancy<128, 2>(per_sm);
    case -4: return decode_occupancy<128, 4>(per_sm);
    default: return decode_occupancy<128, 8>(per_sm);
  }
}

template <int D, int NQP>
int launch_decode_t(const fa::DecodeParams& p, int BH, cudaStream_t stream) {
  auto kern = fa::fa_decode_kernel<D, NQP>;
  const int smem = fa::DecLayout<D, NQP>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  LaunchTrace trace(kKernDecode, stream);
  kern<<<dim3(p.splits, BH), fa::kDecThreads, smem, stream>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int launch_decode(const fa::DecodeParams& p, int BH, int d, cudaStream_t stream) {
  switch (fa::dec_nqp(p.Nq) * (d == 64 ? 1 : -1)) {
    case 1: return launch_decode_t<64, 1>(p, BH, stream);
    case 2: return launch_decode_t<64, 2>(p, BH, stream);
    case 4: return launch_decode_t<64, 4>(p, BH, stream);
    case 8: return launch_decode_t<64, 8>(p, BH, stream);
    case -1: return launch_decode_t<128, 1>(p, BH, stream);
    case -2: return launch_decode_t<128, 2>(p, BH, stream);
    case -4: return launch_decode_t<128, 4>(p, BH, stream);
    default: return launch_decode_t<128, 8>(p, BH, stream);
  }
}

// ---------------------------------------------------------------- GEMM
size_t gemm_ld8(int n) { return (static_cast<size_t>(n) + 7) / 8 * 8; }

bool gemm_needs_pack(const void* ptr, int ld) {
  return !aligned16(ptr) || (ld % 8) != 0;
}

size_t gemm_ws_bytes(const void* A, const void* B, int M, int N, int K, int lda, int ldb) {
  size_t bytes = 0;
  if (gemm_needs_pack(A, lda)) bytes += fa::round256(static_cast<size_t>(M) * gemm_ld8(K) * 2);
  if (gemm_needs_pack(B, ldb)) bytes += fa::round256(static_cast<size_t>(K) * gemm_ld8(N) * 2);
  return bytes;
}

// 2-D view [rows][cols] of a bf16 matrix with row stride `ld` elements
// (a multiple of 8), boxes of box_rows x 64 columns, 128-byte swizzle.
int make_tmap_2d(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

// Tile width: 256 columns when that still gives every SM at least one tile,
// else 128 (more, smaller tiles for small problems).
int gemm_tile_n(int M, int N, int sms) {
  const long long t256 = static_cast<long long>((M + fa::kGemmBM - 1) / fa::kGemmBM) * ((N + 255) / 256);
  return t256 >= sms ? 256 : 128;
}

template <int BN>
int launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, fa::GemmParams p, int sms,
                  cudaStream_t st) {
  p.tiles_n = (p.N + BN - 1) / BN;
  p.n_tiles = ((p.M + fa::kGemmBM - 1) / fa::kGemmBM) * p.tiles_n;
  const int ctas = p.n_tiles < sms ? p.n_tiles : sms;
  auto kern = fa::fa_gemm_kernel<BN>;
  const int smem = fa::GemmLayout<BN>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_LAUNCH;
  LaunchTrace trace(kKernGemm, st);
  kern<<<ctas, 256, smem, st>>>(ta, tb, p);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int launch_gemm_pack(const void* src, int ld_src, void* dst, int ld_dst, int rows, int cols,
                     int sms, cudaStream_t stream) {
  LaunchTrace trace(kKernGemmPack, stream);
  fa::fa_gemm_pack<<<sms * 4, 256, 0, stream>>>(static_cast<const uint16_t*>(src), ld_src,
                                                static_cast<uint16_t*>(dst), ld_dst, rows, cols);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// Split of a decode problem on the current device.
int decode_device_plan(int B, int H, int Nq, int Nk, int d, int num_splits, DeviceInfo** info,
                       int* splits, int* chunk) {
  int s = device_info(info);
  if (s != FA_OK) return s;
  int per_sm = 1;
  if ((s = decode_occupancy_any(d, Nq, &per_sm)) != FA_OK) return s;
  return decode_plan(B * H, Nq, Nk, num_splits, (*info)->sms, per_sm, splits, chunk);
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
    case FA_ERR_WORKSPACE: return "workspace smaller than the *_workspace_size() it needs";
    case FA_ERR_LAUNCH: return "the CUDA runtime rejected a launch or query";
    case FA_ERR_TIMEOUT: return "a device-side wait timed out";
    case FA_ERR_DEVICE_ASSERT: return "a device-side consistency check failed";
    case FA_ERR_ARCH: return "the current device is not an sm_100 (B200-class) GPU";
    case FA_ERR_ARG: return "invalid argument (scale must be finite and >= 0; grad_dtype 0 or 1)";
    case FA_ERR_NOALLOC_LIMIT:
      return "problem needs more backward scratch than fa_bwd_noalloc's fixed maximum";
    default: return "unknown status";
  }
}

int fa_decode_plan(int BH, int Nq, int Nk, int d, int num_splits, int sms, int ctas_per_sm,
                   int* splits, int* chunk_keys) {
  if (!splits || !chunk_keys) return FA_ERR_NULL;
  if (BH < 1 || BH > 65535 || Nq < 1 || Nq > kDecMaxNq || Nk < 1 || sms < 1 || ctas_per_sm < 1)
    return FA_ERR_SHAPE;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
  return decode_plan(BH, Nq, Nk, num_splits, sms, ctas_per_sm, splits, chunk_keys);
}

size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits) {
  if (check_decode_shape(B, H, Nq, Nk, Nk, d) != FA_OK) return 0;
  DeviceInfo* info = nullptr;
  int splits = 1, chunk = 0;
  if (decode_device_plan(B, H, Nq, Nk, d, num_splits, &info, &splits, &chunk) != FA_OK) return 0;
  return decode_ws_bytes(B * H, Nq, d, splits);
}

int fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
              const int* cache_lens, int B, int H, int Nq, int Nk, int ld_kv, int d, float scale,
              int causal, int num_splits, void* workspace, size_t workspace_bytes,
              fa_stream_t stream) {
  if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_NULL;
  int s = check_decode_shape(B, H, Nq, Nk, ld_kv, d);
  if (s != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (num_splits < 0) return FA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(lse) || (cache_lens && (reinterpret_cast<uintptr_t>(cache_lens) & 3u)))
    return FA_ERR_ALIGN;
  DeviceInfo* info = nullptr;
  int splits = 1, chunk = 0;
  if ((s = decode_device_plan(B, H, Nq, Nk, d, num_splits, &info, &splits, &chunk)) != FA_OK)
    return s;
  const int BH = B * H;
  const size_t need = decode_ws_bytes(BH, Nq, d, splits);
  if (need > 0) {
    if (!workspace) return FA_ERR_NULL;
    if (!aligned16(workspace)) return FA_ERR_ALIGN;
    if (workspace_bytes < need) return FA_ERR_WORKSPACE;
  }
  fa::DecodeParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k_cache);
  p.v = static_cast<const uint16_t*>(v_cache);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.lens = cache_lens;
  p.counter = nullptr;
  p.part_o = p.part_ml = nullptr;
  if (need > 0) {
    const size_t nqp = static_cast<size_t>(fa::dec_nqp(Nq));
    const size_t slots = static_cast<size_t>(BH) * splits * nqp;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.counter = reinterpret_cast<int*>(ws);
    p.part_o = reinterpret_cast<float*>(ws + fa::round256(static_cast<size_t>(BH) * 4));
    p.part_ml = reinterpret_cast<float*>(ws + fa::round256(static_cast<size_t>(BH) * 4) +
                                         fa::round256(slots * d * 4));
  }
  p.status = info->status;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.ld = ld_kv;
  p.splits = splits;
  p.chunk = chunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  return launch_decode(p, BH, d, reinterpret_cast<cudaStream_t>(stream));
}

int fa_launch_shape(int pass, int B, int H, int N, int d, int causal, int* ctas, int* work_units) {
  if (!ctas || !work_units) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  DeviceInfo* info = nullptr;
  s = device_info(&info);
  if (s != FA_OK) return s;
  int item_div, tail_shift;
  const int units =
      pass == 0 ? fwd_items(B * H, N, fwd_schedule(B * H, N, causal, info->sms, &item_div, &tail_shift))
                : fa::bwd_units(B, H, N);
  *work_units = units;
  *ctas = units < info->sms ? units : info->sms;
  return FA_OK;
}

int fa_fwd_schedule(int B, int H, int N, int causal, int sms, int* items, int* merged_heads,
                    int* tail_shift) {
  if (!items || !merged_heads || !tail_shift) return FA_ERR_NULL;
  if (B < 1 || H < 1 || N < 1 || sms < 1 ||
      static_cast<long long>(B) * H * ((N + 255) / 256) >= (1LL << 31))
    return FA_ERR_SHAPE;
  int item_div = 0;
  const int h1 = fwd_schedule(B * H, N, causal, sms, &item_div, tail_shift);
  *merged_heads = h1;
  *items = fwd_items(B * H, N, h1);
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
  if (make_tmap_rows(&tq, q, BH, N, d, 128) != FA_OK ||
      make_tmap_rows(&tk, k, BH, N, d, 128) != FA_OK ||
      make_tmap_rows(&tv, v, BH, N, d, 128) != FA_OK)
    return FA_ERR_LAUNCH;
  fa::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.descale_q = p.descale_k = p.descale_v = nullptr;
  p.BH = BH;
  p.N = N;
  p.n_qt2 = (N + 255) / 256;
  p.h1 = fwd_schedule(BH, N, causal, info->sms, &p.item_div, &p.tail_shift);
  p.n_units = fwd_items(BH, N, p.h1);
  // Masked scores are -inf before scaling; a zero scale would turn them into
  // NaN.  FLT_MIN keeps them at -inf while every finite score still scales
  // to zero, so scale = 0 gives exactly uniform weights.
  p.scale_log2 = std::fmax(scale * 1.4426950408889634f, FLT_MIN);
  p.status = info->status;
  const int ctas = p.n_units < info->sms ? p.n_units : info->sms;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64)
    return causal ? launch_fwd<64, true>(tq, tk, tv, p, ctas, st)
                  : launch_fwd<64, false>(tq, tk, tv, p, ctas, st);
  return causal ? launch_fwd<128, true>(tq, tk, tv, p, ctas, st)
                : launch_fwd<128, false>(tq, tk, tv, p, ctas, st);
}

size_t fa_gemm_workspace_size(const void* A, const void* B, int M, int N, int K, int lda,
                               int ldb) {
  if (M < 1 || N < 1 || K < 1 || lda < K || ldb < N) return 0;
  return gemm_ws_bytes(A, B, M, N, K, lda, ldb);
}

int fa_gemm_tiles(int M, int N, int sms, int* tile_n, int* tiles_m, int* tiles_n) {
  if (!tile_n || !tiles_m || !tiles_n) return FA_ERR_NULL;
  if (M < 1 || N < 1 || sms < 1) return FA_ERR_SHAPE;
  *tile_n = gemm_tile_n(M, N, sms);
  *tiles_m = (M + fa::kGemmBM - 1) / fa::kGemmBM;
  *tiles_n = (N + *tile_n - 1) / *tile_n;
  return FA_OK;
}

int fa_gemm(const void* A, const void* B, void* C, int M, int N, int K, int lda, int ldb, int ldc,
            void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (!A || !B || !C) return FA_ERR_NULL;
  if (M < 1 || N < 1 || K < 1 || lda < K || ldb < N || ldc < N) return FA_ERR_SHAPE;
  if (static_cast<long long>(M) * lda >= (1ll << 40) || static_cast<long long>(K) * ldb >= (1ll << 40) ||
      static_cast<long long>(M) * ldc >= (1ll << 40))
    return FA_ERR_SHAPE;
  auto al2 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 1u) == 0; };
  if (!al2(A) || !al2(B) || !al2(C)) return FA_ERR_ALIGN;
  const size_t need = gemm_ws_bytes(A, B, M, N, K, lda, ldb);
  if (need > 0) {
    if (!workspace) return FA_ERR_NULL;
    if (!aligned16(workspace)) return FA_ERR_ALIGN;
    if (workspace_bytes < need) return FA_ERR_WORKSPACE;
  }
  DeviceInfo* info = nullptr;
  int s = device_info(&info);
  if (s != FA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Operands whose rows are not 16-byte aligned go through an aligned copy.
  const void* a_use = A;
  const void* b_use = B;
  int lda_use = lda, ldb_use = ldb;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (gemm_needs_pack(A, lda)) {
    lda_use = static_cast<int>(gemm_ld8(K));
    if ((s = launch_gemm_pack(A, lda, ws, lda_use, M, K, info->sms, st)) != FA_OK) return s;
    a_use = ws;
    ws += fa::round256(static_cast<size_t>(M) * lda_use * 2);
  }
  if (gemm_needs_pack(B, ldb)) {
    ldb_use = static_cast<int>(gemm_ld8(N));
    if ((s = launch_gemm_pack(B, ldb, ws, ldb_use, K, N, info->sms, st)) != FA_OK) return s;
    b_use = ws;
  }
  CUtensorMap ta, tb;
  if (make_tmap_2d(&ta, a_use, M, K, lda_use, 128) != FA_OK ||
      make_tmap_2d(&tb, b_use, K, N, ldb_use, 64) != FA_OK)
    return FA_ERR_LAUNCH;
  fa::GemmParams p;
  p.c = static_cast<uint16_t*>(C);
  p.M = M;
  p.N = N;
  p.K = K;
  p.ldc = ldc;
  p.k_blocks = (K + fa::kGemmBK - 1) / fa::kGemmBK;
  p.status = info->status;
  return gemm_tile_n(M, N, info->sms) == 256 ? launch_gemm_t<256>(ta, tb, p, info->sms, st)
                                             : launch_gemm_t<128>(ta, tb, p, info->sms, st);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, const float* descale_q,
               const float* descale_k, const float* descale_v, void* o, float* lse, int B, int H,
               int N, int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !descale_q || !descale_k || !descale_v || !o || !lse) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  if (d != 128) return FA_ERR_UNSUPPORTED_D;
  if ((s = check_scale(scale)) != FA_OK) return s;
  auto al4 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !al4(descale_q) || !al4(descale_k) || !al4(descale_v))
    return FA_ERR_ALIGN;
  DeviceInfo* info = nullptr;
  if ((s = device_info(&info)) != FA_OK) return s;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (make_tmap_rows_u8(&tq, q, BH, N, d, 128) != FA_OK ||
      make_tmap_rows_u8(&tk, k, BH, N, d, 128) != FA_OK ||
      make_tmap_rows_u8(&tv, v, BH, N, d, 128) != FA_OK)
    return FA_ERR_LAUNCH;
  fa::FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.descale_q = descale_q;
  p.descale_k = descale_k;
  p.descale_v = descale_v;
  p.BH = BH;
  p.N = N;
  p.n_qt2 = (N + 255) / 256;
  p.h1 = fwd_schedule(BH, N, causal, info->sms, &p.item_div, &p.tail_shift);
  p.n_units = fwd_items(BH, N, p.h1);
  p.scale_log2 = scale * 1.4426950408889634f;  // the kernel folds in the descales, then clamps
  p.status = info->status;
  const int ctas = p.n_units < info->sms ? p.n_units : info->sms;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return causal ? launch_fwd<128, true, true>(tq, tk, tv, p, ctas, st)
                : launch_fwd<128, false, true>(tq, tk, tv, p, ctas, st);
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const void* dO, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, void* workspace,
                         size_t workspace_bytes, int grad_dtype, fa_stream_t stream) {
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
  return launch_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal != 0, workspace,
                    grad_dtype, info->sms, info->status, reinterpret_cast<cudaStream_t>(stream),
                    true);
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
  return launch_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal != 0, workspace,
                    grad_dtype, info->sms, info->status, reinterpret_cast<cudaStream_t>(stream));
}

int fa_selftest_wait_timeout(int limit_ms, fa_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return FA_ERR_ARG;
  DeviceInfo* info = nullptr;
  int s = device_info(&info);
  if (s != FA_OK) return s;
  fa_selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      info->status, static_cast<unsigned long long>(limit_ms) * 1000000ull);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
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

int fa_trace_start_mask(unsigned kernel_mask) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  g_trace.clear();
  for (int dev = 0; dev < kMaxDevices; ++dev) g_event_used[dev] = 0;
  g_trace_mask = kernel_mask;
  g_trace_on = true;
  return FA_OK;
}

int fa_trace_start(void) { return fa_trace_start_mask(~0u); }

int fa_trace_stop(int n_kernels, int* launches, double* total_ms) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  g_trace_on = false;
  if (n_kernels < 0 || (n_kernels > 0 && (!launches || !total_ms))) return FA_ERR_NULL;
  for (int k = 0; k < n_kernels; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.0;
  }
  int rc = FA_OK;
  for (const TraceRec& r : g_trace) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      rc = FA_ERR_LAUNCH;
      continue;
    }
    if (r.kernel < n_kernels) {
      launches[r.kernel] += 1;
      total_ms[r.kernel] += ms;
    }
  }
  g_trace.clear();
  return rc;
}

const char* fa_trace_kernel_name(int kernel) {
  return (kernel >= 0 && kernel < kNumKernels) ? kKernelNames[kernel] : "unknown";
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, int grad_dtype, fa_stream_t stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_NULL;
  int s = check_shape(B, H, N, d);
  if (s != FA_OK) return s;
  if ((s = check_scale(scale)) != FA_OK) return s;
  if (grad_dtype != 0 && grad_dtype != 1) return FA_ERR_ARG;
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_ALIGN;
  if (fa::bwd_workspace_bytes(B, H, N, d) > FA_BWD_NOALLOC_MAX_SCRATCH) return FA_ERR_NOALLOC_LIMIT;
  DeviceInfo* info = nullptr;
  if ((s = device_info(&info)) != FA_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  // The preprocess kernel rewrites every part of the scratch that must start
  // from zero (dQ accumulator, scheduler counter), so the previous call's
  // contents do not matter.
  return launch_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal != 0, scratch,
                    grad_dtype, info->sms, info->status, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
