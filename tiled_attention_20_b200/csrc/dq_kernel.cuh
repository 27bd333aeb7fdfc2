// dq_kernel.cuh -- dQ pass of the deterministic attention backward (sm_100a).
//
// The atomic backward (fa_bwd_kernel with DQ = true) adds every K/V block's
// contribution to dQ into an fp32 accumulator, in an order that varies from
// run to run.  This kernel instead owns one 128-row Q block per work unit and
// walks the K/V blocks in a fixed order, recomputing the probabilities from
// the saved lse (the recomputation the pages describe: "CS336 Lecture 5 ·
// GPUs, TPUs" notes, section "FlashAttention 解析", item ②) and keeping dQ in
// TMEM until the block is done:
//     S  = Q K_j^T,  P = exp(scale S - lse),  dP = dO V_j^T,
//     dS = P (dP - D),  dQ += dS K_j,   dQ_out = scale * dQ.
// Every dQ element is written once, so results are bit-identical between runs.
//
// Per CTA (persistent, 12 warps): warp 0 TMA producer (Q and dO once per
// unit, K in a 3-slot ring, V in a 2-slot ring), warp 1 TMEM allocator and
// single-thread MMA issuer, warps 4-7 and 8-11 two compute warpgroups that
// split the 128 key columns of S and dP (thread = query row, so lse and D are
// per-thread registers).  TMEM: S in two slots [0,128) [128,256), dP
// [256,384), dQ [384, 384+D).  dS (bf16 pairs) overwrites, for each
// warpgroup, the first half of the S columns that warpgroup read, and is the
// A operand of dQ += dS K straight from TMEM.
#pragma once
#include "sm100.cuh"

namespace fa {

struct DqParams {
  void* dq;           // output [BH][N][D], bf16 or fp32
  const float* lse2;  // lse * log2(e), [BH][Npad] (+inf on padding rows)
  const float* dvec;  // D = rowsum(dO * O), [BH][Npad]
  int BH;
  int N;
  int Npad;
  int nqt;      // ceil(N / 128) Q tiles per head
  int n_units;  // BH * nqt
  float scale_log2;
  float scale;
  int grad_f32;
  int* status;
};

template <int D>
struct DqLayout {
  static constexpr int kTile = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kTile;
  static constexpr int kK = 2 * kTile;
  static constexpr int kV = kK + kKStages * kTile;
  static constexpr int kBar = kV + kVStages * kTile;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kBar + kBarBytes + 1024;
  static constexpr uint32_t kTS = 0;    // + 128 * slot
  static constexpr uint32_t kTdP = 256;
  static constexpr uint32_t kTdQ = 384;
};

// Registers: launched with 168 per thread (384 threads); warpgroup 0 gives
// registers to the two compute warpgroups.
constexpr int kDqLaunchRegs = 168;
constexpr int kDqCtlRegs = 72;
constexpr int kDqComputeRegs = 216;
static_assert(128 * kDqCtlRegs + 256 * kDqComputeRegs <= 384 * kDqLaunchRegs,
              "register split exceeds the launch allocation");

struct DqBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], dp_full, dp_free, ds_ready[2];
  uint64_t dq_full, dq_empty;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct DqUnit {
  int bh, q0, nk;  // head, first query row, key tiles visited
};

// Work unit w -> (head, Q tile), ordered as the forward's units: longest
// first across heads when causal, heads in groups of kDqHeadGroup (shared K
// and V in L2) otherwise.
constexpr int kDqHeadGroup = 8;

template <bool CAUSAL>
__device__ __forceinline__ DqUnit dq_decode(const DqParams& p, int w) {
  DqUnit u;
  int idx;
  if (CAUSAL) {
    idx = w / p.BH;
    u.bh = w - idx * p.BH;
  } else {
    const int g = w / (kDqHeadGroup * p.nqt), g0 = g * kDqHeadGroup;
    const int gs = min(kDqHeadGroup, p.BH - g0);
    const int r = w - g * kDqHeadGroup * p.nqt;
    idx = r / gs;
    u.bh = g0 + (r - idx * gs);
  }
  const int qt = CAUSAL ? (p.nqt - 1 - idx) : idx;  // causal: longest first
  u.q0 = qt * 128;
  const int nkv = (p.N + 127) / 128;
  u.nk = CAUSAL ? min(qt + 1, nkv) : nkv;
  return u;
}

__device__ __forceinline__ int dq_snake_unit(int r, int n_units) {
  const int G = gridDim.x, c = blockIdx.x;
  const int w = r * G + ((r & 1) ? (G - 1 - c) : c);
  return w < n_units ? w : -1;
}

__device__ __forceinline__ bool dwait1(uint64_t* bar, uint32_t parity, DqBarriers* b, int* status) {
  if (*(volatile int*)&b->abort_flag) return false;
  if (mbar_wait(bar, parity, status)) return true;
  *(volatile int*)&b->abort_flag = 1;
  return false;
}

__device__ __forceinline__ bool dwait_warp(uint64_t* bar, uint32_t parity, DqBarriers* b,
                                           int* status) {
  bool ok = !*(volatile int*)&b->abort_flag;
  if (ok) ok = mbar_wait(bar, parity, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *(volatile int*)&b->abort_flag = 1;
  return ok;
}

// ---------------------------------------------------------------- producer
template <int D, bool CAUSAL>
__device__ void dq_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                            const CUtensorMap* tm_v, const CUtensorMap* tm_do, const DqParams& p,
                            uint8_t* smem, DqBarriers* b, int& units, int& kc, int& vc) {
  using L = DqLayout<D>;
  const int rounds = (p.n_units + gridDim.x - 1) / gridDim.x;
  for (int r = 0; r < rounds; ++r) {
    const int w = dq_snake_unit(r, p.n_units);
    if (w < 0) continue;
    const DqUnit u = dq_decode<CAUSAL>(p, w);
    if (units > 0 && !dwait1(&b->q_empty, (units - 1) & 1, b, p.status)) return;
    mbar_arrive_expect_tx(&b->q_full, 2 * L::kTile);
    ++units;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(smem + L::kQ + c * 16384, tm_q, &b->q_full, c * 64, u.q0, u.bh);
      tma_load_3d(smem + L::kDO + c * 16384, tm_do, &b->q_full, c * 64, u.q0, u.bh);
    }
    for (int j = 0; j < u.nk; ++j) {
      {
        const int st = kc % L::kKStages;
        if (kc >= L::kKStages &&
            !dwait1(&b->k_empty[st], ((kc / L::kKStages) - 1) & 1, b, p.status))
          return;
        mbar_arrive_expect_tx(&b->k_full[st], L::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kK + st * L::kTile + c * 16384, tm_k, &b->k_full[st], c * 64,
                      j * 128, u.bh);
        ++kc;
      }
      {
        const int st = vc % L::kVStages;
        if (vc >= L::kVStages &&
            !dwait1(&b->v_empty[st], ((vc / L::kVStages) - 1) & 1, b, p.status))
          return;
        mbar_arrive_expect_tx(&b->v_full[st], L::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kV + st * L::kTile + c * 16384, tm_v, &b->v_full[st], c * 64,
                      j * 128, u.bh);
        ++vc;
      }
    }
  }
}

// ---------------------------------------------------------------- MMA issuer
template <int D>
__device__ __forceinline__ void dq_issue_qk(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
  // 128x128 tile over K = D: both operands K-major 128-byte-swizzled tiles.
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    mma_ss(d_tmem, sdesc_sw128(a_smem + off, 16, 1024), sdesc_sw128(b_smem + off, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// dQ (+)= dS K: M=128 queries, N=D, K=128 keys.  A = dS from TMEM (keys
// 0-63 in columns [0,32) of the S slot, keys 64-127 in [64,96)); B = K tile,
// MN-major view.
template <int D>
__device__ __forceinline__ void dq_issue_dsk(uint32_t d_tmem, uint32_t s_slot, uint32_t k_smem,
                                             bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t a = s_slot + 64 * (kk >> 2) + (kk & 3) * 8;
    mma_ts(d_tmem, a, sdesc_sw128(k_smem + kk * 2048, 16384, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Issue order per unit, for key tiles j = 0 .. nk-1 (g = running tile count
// across units, S slot = g & 1):  S_j, [dP_{j-1} read] dP_j, [dS_{j-1} ready]
// dQ += dS_{j-1} K_{j-1};  then dQ += dS_{nk-1} K_{nk-1} after the loop.
// S_j lands in the slot whose dS was consumed by the dQ MMA of tile j-2,
// issued earlier, so the in-order tensor pipe never overwrites a live operand.
template <int D, bool CAUSAL>
__device__ void dq_mma(const DqParams& p, uint8_t* smem, DqBarriers* b, uint32_t tmem) {
  using L = DqLayout<D>;
  const uint32_t sb = smem_u32(smem);
  int qc = 0, kc = 0, vc = 0, g = 0, uc = 0;
  const int rounds = (p.n_units + gridDim.x - 1) / gridDim.x;
  for (int r = 0; r < rounds; ++r) {
    const int w = dq_snake_unit(r, p.n_units);
    if (w < 0) continue;
    const DqUnit u = dq_decode<CAUSAL>(p, w);
    if (!dwait1(&b->q_full, qc & 1, b, p.status)) return;
    ++qc;
    tc_fence_after();
    int prev_ks = 0;
    for (int j = 0; j <= u.nk; ++j) {
      int ks = 0;
      if (j < u.nk) {  // S_j and dP_j
        ks = kc % L::kKStages;
        const int vs = vc % L::kVStages;
        if (!dwait1(&b->k_full[ks], (kc / L::kKStages) & 1, b, p.status)) return;
        if (!dwait1(&b->v_full[vs], (vc / L::kVStages) & 1, b, p.status)) return;
        tc_fence_after();
        const int slot = g & 1;
        dq_issue_qk<D>(tmem + L::kTS + 128 * slot, sb + L::kQ, sb + L::kK + ks * L::kTile);
        mma_commit(&b->s_full[slot]);
        if (g >= 1) {  // the compute warps have read dP of the previous tile
          if (!dwait1(&b->dp_free, (g - 1) & 1, b, p.status)) return;
          tc_fence_after();
        }
        dq_issue_qk<D>(tmem + L::kTdP, sb + L::kDO, sb + L::kV + vs * L::kTile);
        mma_commit(&b->dp_full);
        mma_commit(&b->v_empty[vs]);
        ++vc;
      } else {
        mma_commit(&b->q_empty);  // Q and dO of this unit are no longer read
      }
      if (j >= 1) {  // dQ += dS_{j-1} K_{j-1}; tile j-1 has running count g-1
        const int gp = g - 1;
        const int slot = gp & 1;
        if (j == 1 && uc > 0) {  // the previous unit's dQ has been read out
          if (!dwait1(&b->dq_empty, (uc - 1) & 1, b, p.status)) return;
          tc_fence_after();
        }
        if (!dwait1(&b->ds_ready[slot], (gp >> 1) & 1, b, p.status)) return;
        tc_fence_after();
        dq_issue_dsk<D>(tmem + L::kTdQ, tmem + L::kTS + 128 * slot,
                        sb + L::kK + prev_ks * L::kTile, j > 1);
        mma_commit(&b->k_empty[prev_ks]);
      }
      if (j < u.nk) {
        prev_ks = ks;
        ++kc;
        ++g;
      }
    }
    mma_commit(&b->dq_full);
    ++uc;
  }
}

// ---------------------------------------------------------------- compute warpgroups
template <int D, bool CAUSAL>
__device__ void dq_compute(const DqParams& p, DqBarriers* b, uint32_t tmem, int h) {
  using L = DqLayout<D>;
  const int t = (threadIdx.x - 128) & 127;  // query row within the tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const float sl2 = p.scale_log2;
  int gj = 0, uc = 0;
  const int rounds = (p.n_units + gridDim.x - 1) / gridDim.x;
  for (int r = 0; r < rounds; ++r) {
    const int w = dq_snake_unit(r, p.n_units);
    if (w < 0) continue;
    const DqUnit u = dq_decode<CAUSAL>(p, w);
    const int row = u.q0 + t;
    const size_t srow = static_cast<size_t>(u.bh) * p.Npad + row;  // row < Npad
    const float lse2 = p.lse2[srow];
    const float drow = p.dvec[srow];
    const float2 sl2v = make_float2(sl2, sl2);
    const float2 nlse = make_float2(-lse2, -lse2);
    const float2 nd = make_float2(-drow, -drow);
    for (int j = 0; j < u.nk; ++j, ++gj) {
      const int slot = gj & 1;
      if (!dwait_warp(&b->s_full[slot], (gj >> 1) & 1, b, p.status)) return;
      if (!dwait_warp(&b->dp_full, gj & 1, b, p.status)) return;
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + L::kTS + 128 * slot + 64 * h;
      uint32_t rs[64], rp[64];
      tmem_ld_x64_pair(tS, tmem + lane_base + L::kTdP + 64 * h, rs, rp);
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&b->dp_free);  // dP may be overwritten
      const int key0 = j * 128 + 64 * h;
      const bool diag = CAUSAL && key0 + 63 > u.q0;  // some key here is after some row
      uint32_t pk[32];
#pragma unroll
      for (int c2 = 0; c2 < 32; ++c2) {
        const float2 x = fma2(make_float2(__uint_as_float(rs[2 * c2]), __uint_as_float(rs[2 * c2 + 1])),
                              sl2v, nlse);
        float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
        if (diag) {
          p0 = (key0 + 2 * c2 <= row) ? p0 : 0.f;
          p1 = (key0 + 2 * c2 + 1 <= row) ? p1 : 0.f;
        }
        const float2 dp = add2(make_float2(__uint_as_float(rp[2 * c2]), __uint_as_float(rp[2 * c2 + 1])), nd);
        const float2 ds = mul2(make_float2(p0, p1), dp);
        pk[c2] = pack_bf16x2(ds.x, ds.y);
      }
      tmem_st_x32(tS, pk);  // dS over this warpgroup's 64 keys, into its own columns
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&b->ds_ready[slot]);
    }
    // Epilogue: this warpgroup's half of the dQ row, times scale.
    if (!dwait_warp(&b->dq_full, uc & 1, b, p.status)) return;
    tc_fence_after();
    uint32_t o[D / 2];
    if (D == 128)
      tmem_ld_x64(tmem + lane_base + L::kTdQ + (D / 2) * h, o);
    else
      tmem_ld_x32(tmem + lane_base + L::kTdQ + (D / 2) * h, o);
    tc_fence_before();
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(&b->dq_empty);
    if (row < p.N) {
      const size_t off = (static_cast<size_t>(u.bh) * p.N + row) * D + (D / 2) * h;
      const float sc = p.scale;
      if (p.grad_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.dq) + off);
#pragma unroll
        for (int v = 0; v < D / 8; ++v)
          dst[v] = make_float4(__uint_as_float(o[4 * v]) * sc, __uint_as_float(o[4 * v + 1]) * sc,
                               __uint_as_float(o[4 * v + 2]) * sc, __uint_as_float(o[4 * v + 3]) * sc);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dq) + off);
#pragma unroll
        for (int v = 0; v < D / 16; ++v)
          dst[v] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * v]) * sc, __uint_as_float(o[8 * v + 1]) * sc),
                              pack_bf16x2(__uint_as_float(o[8 * v + 2]) * sc, __uint_as_float(o[8 * v + 3]) * sc),
                              pack_bf16x2(__uint_as_float(o[8 * v + 4]) * sc, __uint_as_float(o[8 * v + 5]) * sc),
                              pack_bf16x2(__uint_as_float(o[8 * v + 6]) * sc, __uint_as_float(o[8 * v + 7]) * sc));
      }
    }
    ++uc;
  }
}

// ---------------------------------------------------------------- kernel
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fa_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const DqParams p) {
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  DqBarriers* b = reinterpret_cast<DqBarriers*>(smem + L::kBar);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&b->q_full, 1);
    mbar_init(&b->q_empty, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&b->k_full[i], 1);
      mbar_init(&b->k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->v_full[i], 1);
      mbar_init(&b->v_empty[i], 1);
      mbar_init(&b->s_full[i], 1);
      mbar_init(&b->ds_ready[i], 8);  // one arrival per compute warp
    }
    mbar_init(&b->dp_full, 1);
    mbar_init(&b->dp_free, 8);
    mbar_init(&b->dq_full, 1);
    mbar_init(&b->dq_empty, 8);
    mbar_init(&b->mma_done, 1);
    b->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane_id() == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;
  if (warp >= 4) {
    regs_increase<kDqComputeRegs>();
    dq_compute<D, CAUSAL>(p, b, tmem, (warp - 4) >> 2);
  } else {
    regs_decrease<kDqCtlRegs>();
    if (warp == 0) {
      if (lane_id() == 0) {
        int units = 0, kc = 0, vc = 0;
        dq_producer<D, CAUSAL>(&tm_q, &tm_k, &tm_v, &tm_do, p, smem, b, units, kc, vc);
        // No copy may be in flight when the CTA exits.
        if (units > 0) mbar_wait(&b->q_full, (units - 1) & 1, p.status);
        for (int st = 0; st < L::kKStages; ++st) {
          const int n = kc / L::kKStages + (st < kc % L::kKStages ? 1 : 0);
          if (n > 0) mbar_wait(&b->k_full[st], (n - 1) & 1, p.status);
        }
        for (int st = 0; st < L::kVStages; ++st) {
          const int n = vc / L::kVStages + (st < vc % L::kVStages ? 1 : 0);
          if (n > 0) mbar_wait(&b->v_full[st], (n - 1) & 1, p.status);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane_id() == 0) {
        dq_mma<D, CAUSAL>(p, smem, b, tmem);
        mma_commit(&b->mma_done);
        mbar_wait(&b->mma_done, 0, p.status);
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace fa
