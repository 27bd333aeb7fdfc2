// bwd_kernel.cuh -- attention backward on sm_100a.
//
// The pages only say that the backward throws away the N x N probabilities
// and recomputes them tile by tile ("CS336 Lecture 5 · GPUs, TPUs" notes,
// section "FlashAttention 解析", item ②; "GPU 架构与大模型高效计算", §7.2
// item 3).  What is recomputed and how the gradient flows is the exact
// gradient of sum(O * dO):
//     P_ij  = exp(scale q_i.k_j - lse_i)
//     D_i   = sum_c dO_ic O_ic
//     dV_j += P_ij dO_i                dP_ij = dO_i.v_j
//     dS_ij = P_ij (dP_ij - D_i)
//     dK_j += scale dS_ij q_i          dQ_i += scale dS_ij k_j
//
// Three kernels run back to back on the caller's stream:
//   1. fa_bwd_prep: D_i = rowsum(dO * O), lse_i * log2(e) (and +inf / 0 on
//      the padding rows of the last Q block), zero the fp32 dQ accumulator.
//   2. fa_bwd_kernel (persistent, tensor cores): one work unit is one
//      128-key K/V block of one head; it loops over 64-row Q blocks (from the
//      diagonal when causal) and keeps dK, dV accumulating in TMEM.
//   3. fa_bwd_dq_convert: dQ = scale * accumulator, to the output dtype.
//
// Main kernel, 16 warps:
//   warp 0      scheduler and TMA producer: takes the next work unit from a
//               global atomic counter and publishes it to the other roles
//               through a 4-entry ring in shared memory; loads K_j, V_j once
//               per unit and Q_i, dO_i, lse_i, D_i per Q block (3-slot ring).
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 4-7   compute warpgroup 0, warps 8-11 compute warpgroup 1: both
//               work on every Q block, 32 of its 64 queries each, one thread
//               per key row: P^T from S^T and lse, dS^T = P^T (dP^T - D).
//               P^T goes back to TMEM (A of dV += P^T dO), dS^T to shared
//               memory (A of dK += dS^T Q and, read transposed, B of
//               dQ^T = K^T dS^T).  At the end of a unit warpgroup 0 writes
//               dV and warpgroup 1 writes dK.
//   warps 12-15 dQ drain: one thread per head-dimension column; moves dQ^T
//               from TMEM through shared memory into the fp32 accumulator in
//               global memory with bulk reduce-add copies.
// Work units are ordered in groups of a few heads (so the dQ accumulator,
// Q and dO of the heads in flight stay in L2; bwd_group_heads), longest
// first (ascending K/V block) within a group, and handed out dynamically.
// TMEM columns: dV [0,D) dK [D,2D) S^T_s [2D+64s, +64) dP^T_s [2D+128+64s, +64)
// for the two pipeline slots s; dQ^T of slot s overwrites dP^T_s once the
// compute warps have read it, P^T_s (bf16 pairs) overwrites S^T_s.
#pragma once
#include <cfloat>

#include "sm100.cuh"

namespace fa {

inline int bwd_units(int B, int H, int N) { return B * H * ((N + 127) / 128); }

inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: dQ accumulator [BH][N][d] fp32, then lse*log2e and D, each
// [BH][Npad] fp32 with Npad = N rounded up to 128 (whole 64-row and 128-row
// query blocks read padding, never the next head), then the scheduler's
// work-unit counter.
inline size_t bwd_npad(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }
inline size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  return round256(bh * N * d * 4) + 2 * round256(bh * bwd_npad(N) * 4) + 256;
}

// Heads per scheduling group: the heads in flight keep their K, V, Q, dO and
// dQ accumulator in L2 (126 MB on B200).  The largest power of two up to 16
// whose group needs at most 112 MB of it: per head N*d*12 bytes (four bf16
// tensors and the fp32 accumulator).  More heads per group let the dynamic
// scheduler balance the causal units' unequal lengths over more of them;
// past the L2 budget the group's data no longer stays resident.
inline int bwd_group_heads(int N, int d) {
  const double per_head = static_cast<double>(N) * d * 12.0;
  int g = 16;
  while (g > 1 && g * per_head > 112.0 * (1 << 20)) g >>= 1;
  return g;
}

struct BwdParams {
  void* dk;
  void* dv;
  float* dq_acc;
  const float* lse2;  // [BH][Npad]
  const float* dvec;  // [BH][Npad]
  int* sched;         // work-unit counter, zero at launch
  int BH;
  int N;
  int Npad;
  int nq;       // ceil(N / 64) Q blocks
  int nkv;      // ceil(N / 128) K/V blocks
  int n_units;  // BH * nkv
  int group_heads;  // heads per scheduling group (bwd_group_heads)
  float scale_log2;
  float scale;
  int grad_f32;
  int* status;
};

template <int D>
struct BwdLayout {
  static constexpr int kKVBytes = 128 * D * 2;  // one 128-row K or V tile
  static constexpr int kQBytes = 64 * D * 2;    // one 64-row Q or dO tile
  static constexpr int kQStages = 3;
  static constexpr int kDsBytes = 128 * 64 * 2;  // dS^T tile [128 keys][64 q]
  static constexpr int kStageRows = 32;          // dQ rows per bulk reduce
  static constexpr int kStageBytes = kStageRows * D * 4;
  static constexpr int kK = 0;
  static constexpr int kV = kKVBytes;
  static constexpr int kQ = 2 * kKVBytes;
  static constexpr int kDO = kQ + kQStages * kQBytes;
  static constexpr int kDs = kDO + kQStages * kQBytes;
  static constexpr int kStage = kDs + 2 * kDsBytes;  // two dQ staging buffers
  static constexpr int kLse = kStage + 2 * kStageBytes;  // [3][64] fp32
  static constexpr int kDv = kLse + kQStages * 256;   // [3][64] fp32
  static constexpr int kBar = kDv + kQStages * 256;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kBar + kBarBytes + 1024;
  // TMEM columns
  static constexpr uint32_t kTdV = 0;
  static constexpr uint32_t kTdK = D;
  static constexpr uint32_t kTS = 2 * D;         // + 64 s
  static constexpr uint32_t kTdP = 2 * D + 128;  // + 64 s
};

// Registers per thread: launched with kBwdLaunchRegs (512 threads), then
// warpgroup 0 (producer, MMA issuer, two idle warps) and the drain
// warpgroup give registers to the two compute warpgroups.
constexpr int kBwdLaunchRegs = 128;
constexpr int kBwdCtlRegs = 72;
constexpr int kBwdComputeRegs = 168;
constexpr int kBwdDrainRegs = 88;
static_assert(128 * kBwdCtlRegs + 256 * kBwdComputeRegs + 128 * kBwdDrainRegs <=
                  512 * kBwdLaunchRegs,
              "register split exceeds the launch allocation");

constexpr int kUnitRing = 4;
// Consumers of the unit ring, counted in arrivals: the MMA thread, the 8
// compute warps and, when the kernel computes dQ, the 4 drain warps (one
// lane each).
constexpr int unit_consumers(bool dq) { return 1 + 8 + (dq ? 4 : 0); }

struct BwdBarriers {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[3], q_empty[3];
  uint64_t s_full[2], dp_full[2], p_ready[2], ds_ready[2], dq_full[2], dq_empty[2];
  uint64_t acc_full, acc_empty;
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t mma_done;
  int unit_id[kUnitRing];
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdUnit {
  int bh, j, i0, n;  // head, K/V block, first Q block, number of Q blocks
};

// Unit w -> (head, K/V block): groups of p.group_heads heads, K/V blocks in
// ascending order within a group (the longest causal units first), heads
// innermost.
template <bool CAUSAL>
__device__ __forceinline__ BwdUnit bwd_decode(const BwdParams& p, int w) {
  BwdUnit u;
  const int gh = p.group_heads;
  const int per_group = gh * p.nkv;
  const int g = w / per_group;
  const int r = w - g * per_group;
  const int heads = min(gh, p.BH - g * gh);
  u.j = r / heads;
  u.bh = g * gh + (r - u.j * heads);
  u.i0 = CAUSAL ? 2 * u.j : 0;
  u.n = p.nq - u.i0;
  return u;
}

__device__ __forceinline__ bool bwait1(uint64_t* bar, uint32_t parity, BwdBarriers* b,
                                       int* status) {
  if (*(volatile int*)&b->abort_flag) return false;
  if (mbar_wait(bar, parity, status)) return true;
  *(volatile int*)&b->abort_flag = 1;
  return false;
}

// The same from every lane of a warp, with a warp-uniform answer.
__device__ __forceinline__ bool bwait_warp(uint64_t* bar, uint32_t parity, BwdBarriers* b,
                                           int* status) {
  bool ok = !*(volatile int*)&b->abort_flag;
  if (ok) ok = mbar_wait(bar, parity, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *(volatile int*)&b->abort_flag = 1;
  return ok;
}

// Next unit from the ring for a consumer warp (all 32 lanes call; lane 0
// releases the entry).  Returns -1 when the schedule is exhausted, -2 on abort.
__device__ __forceinline__ int next_unit_warp(BwdBarriers* b, int& rc, int* status) {
  const int slot = rc % kUnitRing;
  if (!bwait_warp(&b->unit_full[slot], (rc / kUnitRing) & 1, b, status)) return -2;
  const int w = *(volatile int*)&b->unit_id[slot];
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(&b->unit_empty[slot]);
  ++rc;
  return w;
}

// The same for the single MMA thread.
__device__ __forceinline__ int next_unit_one(BwdBarriers* b, int& rc, int* status) {
  const int slot = rc % kUnitRing;
  if (!bwait1(&b->unit_full[slot], (rc / kUnitRing) & 1, b, status)) return -2;
  const int w = *(volatile int*)&b->unit_id[slot];
  mbar_arrive(&b->unit_empty[slot]);
  ++rc;
  return w;
}

__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile(
      "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
          reinterpret_cast<uint64_t>(dst)),
      "r"(smem_u32(src)), "r"(bytes)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------- producer
template <int D>
__device__ __forceinline__ void bwd_load_q(const CUtensorMap* tm_q, const CUtensorMap* tm_do,
                                           const BwdParams& p, uint8_t* smem, BwdBarriers* b,
                                           int qs, int bh, int i) {
  using L = BwdLayout<D>;
  mbar_arrive_expect_tx(&b->q_full[qs], 2 * L::kQBytes + 2 * 256);
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    tma_load_3d(smem + L::kQ + qs * L::kQBytes + c * 8192, tm_q, &b->q_full[qs], c * 64, i * 64, bh);
    tma_load_3d(smem + L::kDO + qs * L::kQBytes + c * 8192, tm_do, &b->q_full[qs], c * 64, i * 64,
                bh);
  }
  const size_t off = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * 64;
  bulk_load(smem + L::kLse + qs * 256, p.lse2 + off, 256, &b->q_full[qs]);
  bulk_load(smem + L::kDv + qs * 256, p.dvec + off, 256, &b->q_full[qs]);
}

template <int D, bool CAUSAL>
__device__ void bwd_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                             const CUtensorMap* tm_v, const CUtensorMap* tm_do,
                             const BwdParams& p, uint8_t* smem, BwdBarriers* b, int& qc,
                             int& kvc) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kQStages;
  for (int uc = 0;; ++uc) {
    // Take the next unit and publish it to the other roles.
    const int slot = uc % kUnitRing;
    if (uc >= kUnitRing && !bwait1(&b->unit_empty[slot], ((uc / kUnitRing) - 1) & 1, b, p.status))
      return;
    int w = atomicAdd(p.sched, 1);
    if (w >= p.n_units) w = -1;
    *(volatile int*)&b->unit_id[slot] = w;
    mbar_arrive(&b->unit_full[slot]);
    if (w < 0) return;
    const BwdUnit u = bwd_decode<CAUSAL>(p, w);
    // Prefetch the first Q blocks of this unit before waiting for the K/V
    // buffers, which the previous unit may still be using.
    const int pre = u.n < 2 ? u.n : 2;
    for (int it = 0; it < pre; ++it) {
      const int qs = qc % QS;
      if (qc >= QS && !bwait1(&b->q_empty[qs], ((qc / QS) - 1) & 1, b, p.status)) return;
      bwd_load_q<D>(tm_q, tm_do, p, smem, b, qs, u.bh, u.i0 + it);
      ++qc;
    }
    if (kvc > 0 && !bwait1(&b->kv_empty, (kvc - 1) & 1, b, p.status)) return;
    mbar_arrive_expect_tx(&b->kv_full, 2 * L::kKVBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(smem + L::kK + c * 16384, tm_k, &b->kv_full, c * 64, u.j * 128, u.bh);
      tma_load_3d(smem + L::kV + c * 16384, tm_v, &b->kv_full, c * 64, u.j * 128, u.bh);
    }
    ++kvc;
    for (int it = pre; it < u.n; ++it) {
      const int qs = qc % QS;
      if (qc >= QS && !bwait1(&b->q_empty[qs], ((qc / QS) - 1) & 1, b, p.status)) return;
      bwd_load_q<D>(tm_q, tm_do, p, smem, b, qs, u.bh, u.i0 + it);
      ++qc;
    }
  }
}

// ---------------------------------------------------------------- MMA issuer
template <int D>
struct BwdMma {
  // S^T = K Q^T and dP^T = V dO^T: M=128 keys, N=64 queries, K=D.
  static __device__ __forceinline__ void kq(uint32_t d_tmem, uint32_t a_kv, uint32_t b_q) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t oa = (kk >> 2) * 16384 + (kk & 3) * 32;
      const uint32_t ob = (kk >> 2) * 8192 + (kk & 3) * 32;
      mma_ss(d_tmem, sdesc_sw128(a_kv + oa, 16, 1024), sdesc_sw128(b_q + ob, 16, 1024), idesc,
             kk > 0 ? 1u : 0u);
    }
  }
  // dV += P^T dO (A = P^T from TMEM): M=128 keys, N=D, K=64 queries.  P^T of
  // queries 0-31 sits in columns [0,16) of the S^T slot, queries 32-63 in
  // [32,48) (each compute warpgroup writes inside the columns it read).
  static __device__ __forceinline__ void dv(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_do,
                                            bool acc) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(d_tmem, a_tmem + 32 * (kk >> 1) + (kk & 1) * 8,
             sdesc_sw128(b_do + kk * 2048, 8192, 1024), idesc, (acc || kk > 0) ? 1u : 0u);
  }
  // dK += dS^T Q (A = dS^T, K-major in smem): M=128 keys, N=D, K=64 queries.
  static __device__ __forceinline__ void dk(uint32_t d_tmem, uint32_t a_ds, uint32_t b_q,
                                            bool acc) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(d_tmem, sdesc_sw128(a_ds + kk * 32, 16, 1024), sdesc_sw128(b_q + kk * 2048, 8192, 1024),
             idesc, (acc || kk > 0) ? 1u : 0u);
  }
  // dQ^T = K^T dS^T: M=D (head dim), N=64 queries, K=128 keys; both
  // operands MN-major views of the K tile and of the dS^T tile.
  static __device__ __forceinline__ void dqt(uint32_t d_tmem, uint32_t a_k, uint32_t b_ds) {
    constexpr uint32_t idesc = idesc_bf16_f32(D, 64, true, true);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ss(d_tmem, sdesc_sw128(a_k + kk * 2048, 16384, 1024),
             sdesc_sw128(b_ds + kk * 2048, 16384, 1024), idesc, kk > 0 ? 1u : 0u);
  }
};

template <int D, bool CAUSAL, bool DQ>
__device__ void bwd_mma(const BwdParams& p, uint8_t* smem, BwdBarriers* b, uint32_t tmem) {
  using L = BwdLayout<D>;
  using M = BwdMma<D>;
  constexpr int QS = L::kQStages;
  const uint32_t sb = smem_u32(smem);
  int g = 0;      // global Q-block iteration counter (pipeline slot = g % 2)
  int qbase = 0;  // Q-ring uses before this unit
  int rc = 0;     // unit-ring reads
  for (int uc = 0;; ++uc) {
    const int w = next_unit_one(b, rc, p.status);
    if (w < 0) return;
    const BwdUnit u = bwd_decode<CAUSAL>(p, w);
    if (!bwait1(&b->kv_full, uc & 1, b, p.status)) return;
    tc_fence_after();
    auto sdp = [&](int it) -> bool {
      const int gg = g + it, s = gg & 1, qi = qbase + it, qs = qi % QS;
      if (!bwait1(&b->q_full[qs], (qi / QS) & 1, b, p.status)) return false;
      tc_fence_after();
      M::kq(tmem + L::kTS + 64 * s, sb + L::kK, sb + L::kQ + qs * L::kQBytes);
      mma_commit(&b->s_full[s]);
      if (DQ && gg >= 2) {
        if (!bwait1(&b->dq_empty[s], ((gg >> 1) - 1) & 1, b, p.status)) return false;
        tc_fence_after();
      }
      M::kq(tmem + L::kTdP + 64 * s, sb + L::kV, sb + L::kDO + qs * L::kQBytes);
      mma_commit(&b->dp_full[s]);
      return true;
    };
    auto grads = [&](int it) -> bool {
      const int gg = g + it, s = gg & 1, qi = qbase + it, qs = qi % QS;
      if (it == 0 && uc > 0) {  // the previous unit's dK, dV have been written out
        if (!bwait1(&b->acc_empty, (uc - 1) & 1, b, p.status)) return false;
        tc_fence_after();
      }
      if (!bwait1(&b->p_ready[s], (gg >> 1) & 1, b, p.status)) return false;
      tc_fence_after();
      M::dv(tmem + L::kTdV, tmem + L::kTS + 64 * s, sb + L::kDO + qs * L::kQBytes, it > 0);
      if (!bwait1(&b->ds_ready[s], (gg >> 1) & 1, b, p.status)) return false;
      tc_fence_after();
      M::dk(tmem + L::kTdK, sb + L::kDs + s * L::kDsBytes, sb + L::kQ + qs * L::kQBytes, it > 0);
      if (DQ) {
        M::dqt(tmem + L::kTdP + 64 * s, sb + L::kK, sb + L::kDs + s * L::kDsBytes);
        mma_commit(&b->dq_full[s]);
      }
      mma_commit(&b->q_empty[qs]);
      return true;
    };
    if (!sdp(0)) return;
    if (u.n > 1 && !sdp(1)) return;
    for (int it = 0; it < u.n; ++it) {
      if (!grads(it)) return;
      if (it + 2 < u.n && !sdp(it + 2)) return;
    }
    mma_commit(&b->acc_full);
    mma_commit(&b->kv_empty);
    g += u.n;
    qbase += u.n;
  }
}

// ---------------------------------------------------------------- compute warpgroups
// Both warpgroups work on every Q block: warpgroup h takes queries
// [32h, 32h+32) of the 64 (thread = key row), so one Q block's element-wise
// work finishes in half the time.
template <int D, bool CAUSAL>
__device__ void bwd_compute(const BwdParams& p, uint8_t* smem, BwdBarriers* b, uint32_t tmem,
                            int h) {
  using L = BwdLayout<D>;
  constexpr int QS = L::kQStages;
  const int t = (threadIdx.x - 128) & 127;  // key row within the K/V block == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const float sl2 = p.scale_log2;
  int g = 0, qbase = 0, rc = 0;
  for (int uc = 0;; ++uc) {
    const int w = next_unit_warp(b, rc, p.status);
    if (w < 0) return;
    const BwdUnit u = bwd_decode<CAUSAL>(p, w);
    const int key = u.j * 128 + t;
    for (int it = 0; it < u.n; ++it) {
      const int gg = g + it, s = gg & 1, qs = (qbase + it) % QS;
      const int q0 = (u.i0 + it) * 64 + 32 * h;  // first query of this warpgroup's half
      if (!bwait_warp(&b->s_full[s], (gg >> 1) & 1, b, p.status)) return;
      if (!bwait_warp(&b->dp_full[s], (gg >> 1) & 1, b, p.status)) return;
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + L::kTS + 64 * s + 32 * h;
      const uint32_t tdP = tmem + lane_base + L::kTdP + 64 * s + 32 * h;
      const float4* lse4 = reinterpret_cast<const float4*>(smem + L::kLse + qs * 256) + 8 * h;
      const float4* dv4 = reinterpret_cast<const float4*>(smem + L::kDv + qs * 256) + 8 * h;
      uint8_t* ds_row = smem + L::kDs + s * L::kDsBytes + t * 128;
      const bool diag = CAUSAL && q0 < u.j * 128 + 127;
      uint32_t rs[32], rp[32];
      tmem_ld_x32_pair(tS, tdP, rs, rp);
      const float2 sl2v = make_float2(sl2, sl2);
      // P^T = exp2(scale*log2e * S^T - lse*log2e) into TMEM as bf16 pairs (the
      // first 16 of the 32 columns this warpgroup read); rs[] keeps P in fp32.
      {
        uint32_t pk[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l4 = lse4[c4];
          const int c = 4 * c4;
          const float2 x0 = fma2(make_float2(__uint_as_float(rs[c]), __uint_as_float(rs[c + 1])),
                                 sl2v, make_float2(-l4.x, -l4.y));
          const float2 x1 = fma2(make_float2(__uint_as_float(rs[c + 2]), __uint_as_float(rs[c + 3])),
                                 sl2v, make_float2(-l4.z, -l4.w));
          float p0 = ex2_approx(x0.x), p1 = ex2_approx(x0.y), p2 = ex2_approx(x1.x),
                p3 = ex2_approx(x1.y);
          if (diag) {
            p0 = (key <= q0 + c) ? p0 : 0.f;
            p1 = (key <= q0 + c + 1) ? p1 : 0.f;
            p2 = (key <= q0 + c + 2) ? p2 : 0.f;
            p3 = (key <= q0 + c + 3) ? p3 : 0.f;
          }
          rs[c] = __float_as_uint(p0);
          rs[c + 1] = __float_as_uint(p1);
          rs[c + 2] = __float_as_uint(p2);
          rs[c + 3] = __float_as_uint(p3);
          pk[2 * c4] = pack_bf16x2(p0, p1);
          pk[2 * c4 + 1] = pack_bf16x2(p2, p3);
        }
        tmem_st_x16(tS, pk);
      }
      // dS^T = P^T (dP^T - D), to shared memory as bf16 in the 128-byte
      // swizzled layout the tensor core reads (this half: pieces 4h .. 4h+3).
#pragma unroll
      for (int piece = 0; piece < 4; ++piece) {  // 8 queries = 16 bytes per piece
        const float4 da = dv4[2 * piece], db = dv4[2 * piece + 1];
        const int c = 8 * piece;
        uint32_t w4[4];
        const float2 d2[4] = {make_float2(da.x, da.y), make_float2(da.z, da.w),
                              make_float2(db.x, db.y), make_float2(db.z, db.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 pp = make_float2(__uint_as_float(rs[c + 2 * e]), __uint_as_float(rs[c + 2 * e + 1]));
          const float2 dp = make_float2(__uint_as_float(rp[c + 2 * e]), __uint_as_float(rp[c + 2 * e + 1]));
          const float2 ds = mul2(pp, add2(dp, make_float2(-d2[e].x, -d2[e].y)));
          w4[e] = pack_bf16x2(ds.x, ds.y);
        }
        const int pc = 4 * h + piece;
        *reinterpret_cast<uint4*>(ds_row + ((pc ^ (t & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      // Each lane orders its own TMEM and shared-memory writes; after the
      // warp synchronises, one arrival per warp publishes the warp's work.
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane_id() == 0) {
        mbar_arrive(&b->p_ready[s]);
        mbar_arrive(&b->ds_ready[s]);
      }
    }
    // Unit epilogue: warpgroup 0 writes dV, warpgroup 1 writes scale * dK.
    if (!bwait_warp(&b->acc_full, uc & 1, b, p.status)) return;
    tc_fence_after();
    const bool valid = key < p.N;
    const size_t row = static_cast<size_t>(u.bh) * p.N + key;
    const uint32_t col = h ? L::kTdK : L::kTdV;
    const float mul = h ? p.scale : 1.f;
    void* out = h ? p.dk : p.dv;
    uint32_t r[D];
    if (D == 128)
      tmem_ld_x128(tmem + lane_base + col, r);
    else
      tmem_ld_x64(tmem + lane_base + col, r);
    tc_fence_before();
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(&b->acc_empty);  // TMEM read: dK, dV may be overwritten
    if (valid) {
      if (p.grad_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row * D);
#pragma unroll
        for (int v = 0; v < D / 4; ++v)
          dst[v] = make_float4(__uint_as_float(r[4 * v]) * mul, __uint_as_float(r[4 * v + 1]) * mul,
                               __uint_as_float(r[4 * v + 2]) * mul,
                               __uint_as_float(r[4 * v + 3]) * mul);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row * D);
#pragma unroll
        for (int v = 0; v < D / 8; ++v)
          dst[v] = make_uint4(
              pack_bf16x2(__uint_as_float(r[8 * v + 0]) * mul, __uint_as_float(r[8 * v + 1]) * mul),
              pack_bf16x2(__uint_as_float(r[8 * v + 2]) * mul, __uint_as_float(r[8 * v + 3]) * mul),
              pack_bf16x2(__uint_as_float(r[8 * v + 4]) * mul, __uint_as_float(r[8 * v + 5]) * mul),
              pack_bf16x2(__uint_as_float(r[8 * v + 6]) * mul, __uint_as_float(r[8 * v + 7]) * mul));
      }
    }
    g += u.n;
    qbase += u.n;
  }
}

// ---------------------------------------------------------------- dQ drain
// Moves dQ^T of each Q block from TMEM to registers, stages it row-major in
// shared memory (32 rows at a time, two buffers) and adds it into the fp32
// accumulator with bulk reduce-add copies, one in flight while the other
// buffer fills.
//
// The 128 drain threads meet at named barriers, so they must agree on every
// wait's outcome: each wait ends with a barrier reduction over the 128
// threads, and on an abort all four warps leave together (none is left
// waiting at a named barrier for a warp that has gone).

// True on every drain thread iff `ok` holds on all 128 (barrier 1).
__device__ __forceinline__ bool drain_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(ok))
      : "memory");
  return r != 0;
}

// A bounded mbarrier wait by every drain thread, with one answer for all.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, BwdBarriers* b,
                                           int* status) {
  bool ok = !*(volatile int*)&b->abort_flag;
  if (ok) ok = mbar_wait(bar, parity, status);
  ok = drain_all(ok);
  if (!ok) *(volatile int*)&b->abort_flag = 1;
  return ok;
}

template <int D, bool CAUSAL>
__device__ void bwd_drain(const BwdParams& p, uint8_t* smem, BwdBarriers* b, uint32_t tmem) {
  using L = BwdLayout<D>;
  const int t = threadIdx.x - 384;
  const int quarter = t >> 5, ln = t & 31;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  // M = D accumulator layout: D = 128 fills all 128 lanes (lane = column of
  // the head dimension); D = 64 uses lanes 0-15 of each 32-lane quarter.
  const bool valid = (D == 128) || (ln < 16);
  const int dcol = (D == 128) ? t : (quarter * 16 + ln);
  const bool issuer = (t == 0);
  int g = 0, rc = 0;
  for (;;) {
    // Next unit from the ring, with one answer for the four warps.
    const int slot = rc % kUnitRing;
    if (!drain_wait(&b->unit_full[slot], (rc / kUnitRing) & 1, b, p.status)) break;
    const int w = *(volatile int*)&b->unit_id[slot];
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(&b->unit_empty[slot]);
    ++rc;
    if (w < 0) break;
    const BwdUnit u = bwd_decode<CAUSAL>(p, w);
    bool ok = true;
    for (int it = 0; it < u.n; ++it, ++g) {
      const int s = g & 1;
      const int q0 = (u.i0 + it) * 64;
      // Each warp waits and reads its TMEM quarter on its own; the four
      // agree on the outcome at the barrier before the first staging write.
      // (After a failed wait the values read are dropped there.)
      ok = !*(volatile int*)&b->abort_flag && mbar_wait(&b->dq_full[s], (g >> 1) & 1, p.status);
      tc_fence_after();
      uint32_t r[64];
      tmem_ld_x64(tmem + lane_base + L::kTdP + 64 * s, r);
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&b->dq_empty[s]);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float* stage = reinterpret_cast<float*>(smem + L::kStage + half * L::kStageBytes);
        if (issuer) bulk_wait_read1();  // this buffer's previous reduce has read it
        if (half == 0) {
          ok = drain_all(ok);
          if (!ok) {
            *(volatile int*)&b->abort_flag = 1;
            break;
          }
        } else {
          named_bar_sync(1, 128);
        }
        if (valid) {
#pragma unroll
          for (int c = 0; c < L::kStageRows; ++c)
            stage[c * D + dcol] = __uint_as_float(r[half * L::kStageRows + c]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (issuer) {
          const int r0 = q0 + half * L::kStageRows;
          const int rows = min(L::kStageRows, p.N - r0);
          if (rows > 0)
            bulk_reduce_add_f32(p.dq_acc + (static_cast<size_t>(u.bh) * p.N + r0) * D, stage,
                                rows * D * 4);
          bulk_commit();  // an empty group keeps the two-buffer accounting exact
        }
      }
      if (!ok) break;
    }
    if (!ok) break;
  }
  if (issuer) bulk_wait0();  // no copy may read shared memory after the CTA exits
}

// ---------------------------------------------------------------- kernels
// DQ = false computes dK and dV only (the deterministic backward computes dQ
// in a separate pass, fa_dq_kernel).
template <int D, bool CAUSAL, bool DQ>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  BwdBarriers* b = reinterpret_cast<BwdBarriers*>(smem + L::kBar);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&b->kv_full, 1);
    mbar_init(&b->kv_empty, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&b->q_full[i], 1);
      mbar_init(&b->q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->s_full[i], 1);
      mbar_init(&b->dp_full[i], 1);
      mbar_init(&b->p_ready[i], 8);   // one arrival per compute warp (both warpgroups)
      mbar_init(&b->ds_ready[i], 8);
      mbar_init(&b->dq_full[i], 1);
      mbar_init(&b->dq_empty[i], 4);  // one arrival per drain warp
    }
    mbar_init(&b->acc_full, 1);
    mbar_init(&b->acc_empty, 8);  // one arrival per compute warp
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&b->unit_full[i], 1);
      mbar_init(&b->unit_empty[i], unit_consumers(DQ));
    }
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

  if (warp >= 4 && warp < 12) {
    regs_increase<kBwdComputeRegs>();
    bwd_compute<D, CAUSAL>(p, smem, b, tmem, (warp - 4) >> 2);
  } else if (warp >= 12) {
    regs_decrease<kBwdDrainRegs>();
    if (DQ) bwd_drain<D, CAUSAL>(p, smem, b, tmem);
  } else {
    regs_decrease<kBwdCtlRegs>();
    if (warp == 0) {
      if (lane_id() == 0) {
        int qc = 0, kvc = 0;
        bwd_producer<D, CAUSAL>(&tm_q, &tm_k, &tm_v, &tm_do, p, smem, b, qc, kvc);
        // No copy may be in flight when the CTA exits.
        constexpr int QS = L::kQStages;
        if (kvc > 0) mbar_wait(&b->kv_full, (kvc - 1) & 1, p.status);
        for (int st = 0; st < QS; ++st) {
          const int n = qc / QS + (st < qc % QS ? 1 : 0);
          if (n > 0) mbar_wait(&b->q_full[st], (n - 1) & 1, p.status);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane_id() == 0) {
        bwd_mma<D, CAUSAL, DQ>(p, smem, b, tmem);
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

// D_i = rowsum(dO * O); lse2 = lse * log2(e) (+inf and D = 0 on rows N..Npad);
// zero the dQ accumulator and the work-unit counter; latch the assert bit if
// an lse is not finite.  One thread per 8 consecutive elements of a row.
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_prep(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dvec,
                float* __restrict__ dq_acc, int* __restrict__ sched, int BH, int N, int Npad,
                int zero_acc, int* __restrict__ status) {
  constexpr int TPR = D / 8;  // threads per row
  if (blockIdx.x == 0 && threadIdx.x == 0) *sched = 0;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gid / TPR;  // over BH * Npad
  const int part = static_cast<int>(gid % TPR);
  const bool in_range = row < static_cast<long long>(BH) * Npad;
  const int bh = in_range ? static_cast<int>(row / Npad) : 0;
  const int q = in_range ? static_cast<int>(row % Npad) : 0;
  const bool real = in_range && q < N;
  float acc = 0.f;
  if (real) {
    const size_t off = (static_cast<size_t>(bh) * N + q) * D + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 c = *reinterpret_cast<const uint4*>(dO + off);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(a2[e]);
      const float2 y = __bfloat1622float2(c2[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
    if (zero_acc) {
      float4* z = reinterpret_cast<float4*>(dq_acc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int m = TPR / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m, TPR);
  if (in_range && part == 0) {
    const size_t i = static_cast<size_t>(bh) * Npad + q;
    const float l = real ? lse[static_cast<size_t>(bh) * N + q] : 0.f;
    // Consistency check: a forward's lse is finite on every row.
    if (real && !(fabsf(l) <= FLT_MAX)) atomicOr(status, kDevAssert);
    dvec[i] = real ? acc : 0.f;
    lse2[i] = real ? l * 1.4426950408889634f : INFINITY;
  }
}

// dQ = scale * accumulator, to bf16 or fp32; 8 elements per thread.
__global__ void __launch_bounds__(256)
    fa_bwd_dq_convert(const float* __restrict__ acc, void* __restrict__ dq, long long n8,
                      float scale, int to_f32) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  if (to_f32) {
    float4* d = reinterpret_cast<float4*>(dq);
    d[2 * i] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
    d[2 * i + 1] = make_float4(c.x * scale, c.y * scale, c.z * scale, c.w * scale);
  } else {
    reinterpret_cast<uint4*>(dq)[i] =
        make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                   pack_bf16x2(c.x * scale, c.y * scale), pack_bf16x2(c.z * scale, c.w * scale));
  }
}

}  // namespace fa
