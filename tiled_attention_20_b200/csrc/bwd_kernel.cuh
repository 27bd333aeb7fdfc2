// bwd_kernel.cuh -- attention backward on sm_100a (placeholder until the
// tensor-core backward lands).
#pragma once
#include "sm100.cuh"

namespace fa {

inline int bwd_units(int B, int H, int N) { return B * H * ((N + 127) / 128); }

inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const size_t rows = static_cast<size_t>(B) * H * N;
  return round256(rows * d * 4) + round256(rows * 4);
}

typedef CUresult (*EncodeTiledFnT)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline int launch_bwd(const void*, const void*, const void*, const void*, const void*, const float*,
                      void*, void*, void*, int, int, int, int, float, bool, void*, int, int, int*,
                      cudaStream_t, EncodeTiledFnT) {
  return -6;
}

}  // namespace fa
