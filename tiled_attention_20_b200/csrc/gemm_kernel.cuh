// gemm_kernel.cuh -- C = A B in bf16 with fp32 accumulation, the matrix
// multiply whose throughput-versus-size curve opens "CS336 Lecture 5 · GPUs,
// TPUs" (notes: the opening goal and the "矩阵谜题" section; transcript
// [01:06:15]-[01:08:35]): throughput climbs with arithmetic intensity
// (roofline), sizes divisible only by 1 or 2 fall off (the tile loads lose
// their alignment), and the curve steps down whenever the count of output
// tiles crosses a multiple of the SM count (wave quantization).
//
// B200 design: one persistent CTA per SM walks the 256 x BN output tiles in
// a static round-robin order, so the number of tiles over 148 SMs sets the
// number of rounds.  BN = 128 is the tile shape of that example; BN = 256
// halves the operand traffic per FLOP (A is reused for twice the columns)
// and is used whenever it still gives every SM a tile.  Per CTA:
//   warp 0      TMA producer: per 64-wide K block, A as two 128 x 64 boxes
//               (K-major) and B as BN/64 boxes of 64 x 64 (row-major B is
//               MN-major for the tensor core), 128-byte swizzle;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               M = 128, N = BN, K = 16 per instruction, two M halves;
//   warps 4-7   epilogue: TMEM -> registers -> bf16 -> global memory.
// With BN = 128 TMEM holds two 256-column accumulators, so the epilogue of
// one tile overlaps the main loop of the next; with BN = 256 the one
// accumulator fills all 512 columns and the epilogue runs between tiles.
// Ragged M, N, K edges read zeros from the TMA out-of-bounds fill; the
// epilogue checks rows and columns.  TMA needs 16-byte aligned row strides:
// the host packs an operand whose leading dimension is not a multiple of 8
// elements into an aligned copy first, which is where the ÷1 and ÷2 sizes
// lose throughput on this machine.
#pragma once
#include "sm100.cuh"

namespace fa {

constexpr int kGemmBM = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmMaxStages = 4;

template <int BN>
struct GemmLayout {
  static constexpr int kStages = BN == 128 ? 4 : 3;
  static constexpr int kAccBufs = BN == 128 ? 2 : 1;       // accumulators in 512 TMEM columns
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;   // two 128 x 64 boxes, 16 KB each
  static constexpr int kBBytes = kGemmBK * BN * 2;        // BN/64 boxes of 64 x 64, 8 KB each
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBar + 256 + 1024;  // + manual 1024-byte alignment
};

struct GemmParams {
  uint16_t* c;  // bf16 [M, ldc]
  int M, N, K, ldc;
  int tiles_n, n_tiles, k_blocks;
  int* status;
};

struct GemmBarriers {
  uint64_t full[kGemmMaxStages], empty[kGemmMaxStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool gemm_wait1(uint64_t* bar, uint32_t parity, GemmBarriers* b,
                                           int* status) {
  if (*(volatile int*)&b->abort_flag) return false;
  if (mbar_wait(bar, parity, status)) return true;
  *(volatile int*)&b->abort_flag = 1;
  return false;
}

__device__ __forceinline__ bool gemm_wait_warp(uint64_t* bar, uint32_t parity, GemmBarriers* b,
                                               int* status) {
  bool ok = !*(volatile int*)&b->abort_flag;
  if (ok) ok = mbar_wait(bar, parity, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *(volatile int*)&b->abort_flag = 1;
  return ok;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

template <int BN>
__global__ void __launch_bounds__(256, 1)
    fa_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const GemmParams p) {
  using L = GemmLayout<BN>;
  constexpr int S = L::kStages;
  constexpr int NB = L::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  GemmBarriers* b = reinterpret_cast<GemmBarriers*>(smem + L::kBar);
  const int warp = threadIdx.x >> 5;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&b->full[i], 1);
      mbar_init(&b->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->acc_full[i], 1);
      mbar_init(&b->acc_empty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&b->mma_done, 1);
    b->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane_id() == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane_id() == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += G) {
        const int m0 = (tile / p.tiles_n) * kGemmBM, n0 = (tile % p.tiles_n) * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % S;
          if (it >= S && !gemm_wait1(&b->empty[st], ((it / S) - 1) & 1, b, p.status)) goto drain;
          mbar_arrive_expect_tx(&b->full[st], L::kStageBytes);
          uint8_t* sa = smem + st * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          const int k0 = kb * kGemmBK;
          tma_load_2d(sa, &tm_a, &b->full[st], k0, m0);
          tma_load_2d(sa + 16384, &tm_a, &b->full[st], k0, m0 + 128);
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sb + 8192 * j, &tm_b, &b->full[st], n0 + 64 * j, k0);
        }
      }
    drain:
      // Every copy this thread armed has landed before the CTA may exit.
      for (int st = 0; st < S; ++st) {
        const int n = it / S + (st < it % S ? 1 : 0);
        if (n > 0) mbar_wait(&b->full[st], (n - 1) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane_id() == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, true);
      const uint32_t sbase = smem_u32(smem);
      int it = 0, tc = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += G, ++tc) {
        const int buf = tc % NB, use = tc / NB;
        if (use >= 1 && !gemm_wait1(&b->acc_empty[buf], (use - 1) & 1, b, p.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * 2 * BN;
        bool ok = true;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int st = it % S;
          if (!gemm_wait1(&b->full[st], (it / S) & 1, b, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + st * L::kStageBytes;
          const uint32_t sb = sa + L::kABytes;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(acc + h * BN, sdesc_sw128(sa + h * 16384 + kk * 32, 16, 1024),
                     sdesc_sw128(sb + kk * 2048, 8192, 1024), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&b->empty[st]);
        }
        if (!ok) break;
        mma_commit(&b->acc_full[buf]);
      }
      mma_commit(&b->mma_done);
      mbar_wait(&b->mma_done, 0, p.status);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int t = threadIdx.x - 128;  // TMEM lane = row within an M half
    const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
    const bool vec_ok = (p.ldc % 8) == 0 && (reinterpret_cast<uintptr_t>(p.c) & 15) == 0;
    int tc = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += G, ++tc) {
      const int buf = tc % NB;
      if (!gemm_wait_warp(&b->acc_full[buf], (tc / NB) & 1, b, p.status)) break;
      tc_fence_after();
      const int m0 = (tile / p.tiles_n) * kGemmBM, n0 = (tile % p.tiles_n) * BN;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int row = m0 + 128 * h + t;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld_x32(tmem + lane_base + buf * 2 * BN + h * BN + c0, r);
          uint16_t* dst = p.c + static_cast<size_t>(row) * p.ldc + n0 + c0;
          const int ncols = row < p.M ? min(32, p.N - (n0 + c0)) : 0;
          if (vec_ok && ncols == 32) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(dst)[v] = make_uint4(
                  pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1])),
                  pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                  pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                  pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < ncols) dst[c] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[c])));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&b->acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Row-by-row copy of a bf16 matrix into a buffer with an aligned leading
// dimension (the padding columns are never read: the TMA box stops at the
// logical width and fills zeros beyond it).
__global__ void fa_gemm_pack(const uint16_t* __restrict__ src, int ld_src, uint16_t* __restrict__ dst,
                             int ld_dst, int rows, int cols) {
  const long long total = static_cast<long long>(rows) * cols;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / cols, c = i - r * cols;
    dst[r * ld_dst + c] = src[r * ld_src + c];
  }
}

}  // namespace fa
