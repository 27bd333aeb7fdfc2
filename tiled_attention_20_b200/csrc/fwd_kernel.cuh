// fwd_kernel.cuh -- attention forward on sm_100a.
//
// Computes O = softmax(scale Q K^T [+ causal]) V and lse per row, tile by tile
// with the online softmax of "第17讲 Tensor Core、HBM、SRAM 与
// FlashAttention" §8.3 (running max m, running sum l, rescale of the output
// accumulator by e^{m - m'}, O = o / l at the end), following the tiled flow
// of §8.2 of the same page: a Q tile is loaded once, K/V tiles are streamed
// through shared memory, and scores and probabilities live only on chip.
//
// B200 mapping (one persistent CTA per SM, 12 warps):
//   warp 0      TMA producer: Q tile pair once per work unit, then a K ring
//               and a V ring of kStages slots each.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 4-7   softmax warpgroup 0: owns Q tile 0 (rows q0 .. q0+127).
//   warps 8-11  softmax warpgroup 1: owns Q tile 1 (rows q0+128 .. q0+255).
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// P_i (bf16, packed in pairs) overwrites the first 64 columns of S_i and is
// the A operand of O_i += P_i V straight from TMEM.  One thread owns one row,
// so row max and row sum need no shuffles.
//
// A work unit is (b*H+h, pair of 128-row Q tiles).  Scheduling items of one
// or two units are dealt to a persistent grid of min(items, SMs) CTAs in a
// snake order, so no partial last wave of whole CTAs is left (wave
// quantization, "CS336 Lecture 5 · GPUs, TPUs" notes, section "波次量化").
// Causal items pair complementary tile pairs of one head (fwd_item).
//
// Causal masking is by tile skipping: Q tile i only visits key tiles up to
// its diagonal, and only the diagonal tile (and a ragged last key tile) pays
// for an element mask, which is a select to -inf (no divergent branches).
//
// The output rescale is lazy: the running max used for the exponentials is
// only raised when a tile's maximum exceeds it by more than 2^8 (in the
// exp2 domain), so most tiles skip the O read-modify-write.  The result is
// unchanged because O and l are always scaled by the same reference.
//
// FP8 variant (FP8 = true, d = 128): Q, K and V arrive as E4M3 with one fp32
// descale factor per head each (the low-precision operands of "第17讲" §4.4 /
// "CS336 Lecture 5" on FP8).  S = Q K^T and O += P V run as kind::f8f6f4
// MMAs (K = 32 per instruction, twice the bf16 rate); the score scale absorbs
// descale_q * descale_k, P is stored to TMEM as E4M3 (4 per column) and the
// output is O = descale_v * sum_j p~_j v_j / sum_j p~_j, where p~ is the E4M3
// value of p actually used by the MMA, so O stays a convex combination of V
// rows; lse uses the unrounded p.
#pragma once
#include <cfloat>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace fa {

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  const float* descale_q;  // FP8 only: per-head [B*H] dequantisation factors
  const float* descale_k;
  const float* descale_v;
  int BH;
  int N;
  int n_qt2;       // ceil(N / 256): Q tile pairs per head
  int n_units;     // scheduling items (fwd_item): BH * n_qt2 when h1 == 0
  int h1;          // causal: heads whose tile pairs are dealt two at a time
  int item_div;    // causal: n_qt2 / 2 if h1 > 0, else BH
  int tail_shift;  // causal: the single-pair heads number item_div << tail_shift
  float scale_log2;  // scale * log2(e)
  int* status;
};

template <int D, bool FP8 = false>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * (FP8 ? 1 : 2);
  static constexpr int kStages = (FP8 || D == 64) ? 4 : 2;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kBar + kBarBytes + 1024;  // + manual 1024-B alignment
};

// Registers per thread: the kernel is launched with kFwdLaunchRegs; then
// warpgroup 0 (producer, MMA issuer, two idle warps) gives registers up to
// the two softmax warpgroups, which hold a 128-score row per thread.
// 128 * kFwdCtlRegs + 256 * kFwdSoftmaxRegs == 384 * kFwdLaunchRegs.
constexpr int kFwdLaunchRegs = 168;
constexpr int kFwdCtlRegs = 72;
constexpr int kFwdSoftmaxRegs = 216;
static_assert(128 * kFwdCtlRegs + 256 * kFwdSoftmaxRegs <= 384 * kFwdLaunchRegs,
              "register split exceeds the launch allocation");

struct FwdBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t p_half[2];  // bf16: the first 64 keys of P are in TMEM
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int unit_nk[2][2];  // key tiles of the two Q tiles of the n-th unit, slot n & 1
};
static_assert(sizeof(FwdBarriers) <= FwdLayout<64>::kBarBytes, "barrier block overflows its slot");

struct FwdUnit {
  int bh, q0, nk0, nk1;
};

// One Q tile pair of one head: its first row and the key tiles each of its
// two Q tiles reads (all of them, or up to the diagonal when causal).  A
// second tile that lies wholly past the last row (N mod 256 in [1, 128])
// reads none: it holds no query.
__device__ __forceinline__ FwdUnit fwd_pair(const FwdParams& p, int bh, int qt2, bool causal) {
  FwdUnit u;
  u.bh = bh;
  u.q0 = qt2 * 256;
  const int nkv = (p.N + 127) / 128;
  u.nk0 = causal ? min(2 * qt2 + 1, nkv) : nkv;
  u.nk1 = (u.q0 + 128 >= p.N) ? 0 : (causal ? min(2 * qt2 + 2, nkv) : nkv);
  return u;
}

// Non-causal items (all equal): one tile pair each, heads in groups of
// kUnitHeadGroup, tile pair major within a group, so the CTAs running at
// one time share a few heads' K and V in L2 instead of streaming every
// head's.
constexpr int kUnitHeadGroup = 8;

// Causal scheduling items.  Tile pair t of a head costs about 4t + 3 key
// tiles, so pairs t and n_qt2 - 1 - t together cost the same for every t.
// The first h1 heads are dealt as such merged items, head-major: every item
// costs the same, and the CTAs running at one time share a few heads' K and
// V in L2 instead of streaming every head's.  The other R heads follow as
// single pairs, longest first across heads, so the snake's last rounds even
// out the per-CTA totals.  With merging (n_qt2 even), R = (n_qt2 / 2) <<
// tail_shift, so one division by item_div decodes both kinds of item; h1 = 0
// (item_div = BH, tail_shift = 0) is the plain longest-first order.  Item w
// holds one or two pairs; sets u to pair `sub` and returns true if it exists.
template <bool CAUSAL>
__device__ __forceinline__ bool fwd_item(const FwdParams& p, int w, int sub, FwdUnit& u) {
  if (w < 0) return false;
  if (!CAUSAL) {
    if (sub) return false;
    const int g = w / (kUnitHeadGroup * p.n_qt2), g0 = g * kUnitHeadGroup;
    const int gs = min(kUnitHeadGroup, p.BH - g0);
    const int r = w - g * kUnitHeadGroup * p.n_qt2;  // every earlier group is full
    const int idx = r / gs;
    u = fwd_pair(p, g0 + (r - idx * gs), idx, false);
    return true;
  }
  const int d = p.item_div, n1 = p.h1 * d, P = p.n_qt2;
  const bool merged = w < n1;
  if (sub && !merged) return false;
  const int w2 = merged ? w : w - n1;
  const int q = w2 / d;
  if (merged) {
    const int k = w2 - q * d;
    u = fwd_pair(p, q, sub ? k : P - 1 - k, true);
  } else {
    const int idx = q >> p.tail_shift;  // = w2 / R
    u = fwd_pair(p, p.h1 + w2 - ((idx * d) << p.tail_shift), P - 1 - idx, true);
  }
  return true;
}

// Whether item w has a pair `sub` (fwd_item without the decode).
template <bool CAUSAL>
__device__ __forceinline__ bool fwd_item_exists(const FwdParams& p, int w, int sub) {
  return w >= 0 && (!sub || (CAUSAL && w < p.h1 * p.item_div));
}

// Static "snake" assignment of work units to persistent CTAs: in round r,
// CTA c takes unit r*G + c when r is even and r*G + (G-1-c) when r is odd
// (G = gridDim.x).  With units sorted longest first this keeps every CTA's
// total close to the mean.  Returns -1 past the end; `r` is the round.
__device__ __forceinline__ int snake_unit(int r, int n_units) {
  const int G = gridDim.x, c = blockIdx.x;
  const int w = r * G + ((r & 1) ? (G - 1 - c) : c);
  return w < n_units ? w : -1;
}
__device__ __forceinline__ int snake_rounds(int n_units) {
  return (n_units + gridDim.x - 1) / gridDim.x;
}

// Wait on an mbarrier from one thread; false (and the CTA's abort flag set)
// if the wait timed out or another role already aborted.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, FwdBarriers* b,
                                      int* status) {
  if (*(volatile int*)&b->abort_flag) return false;
  if (mbar_wait(bar, parity, status)) return true;
  *(volatile int*)&b->abort_flag = 1;
  return false;
}

// The same from every lane of a warp, with a warp-uniform answer.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, FwdBarriers* b,
                                          int* status) {
  bool ok = !*(volatile int*)&b->abort_flag;
  if (ok) ok = mbar_wait(bar, parity, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *(volatile int*)&b->abort_flag = 1;
  return ok;
}

// ---------------------------------------------------------------- producer
template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                             const CUtensorMap* tm_v, const FwdParams& p, uint8_t* smem,
                             FwdBarriers* b, int& kc, int& vc, int& units) {
  using L = FwdLayout<D, FP8>;
  constexpr int S = L::kStages;
  // A tile is D/64 boxes of 64 bf16 columns, or one box of 128 E4M3 columns;
  // either way a box row is 128 bytes.
  constexpr int NB = FP8 ? 1 : D / 64;
  for (int it = 0, ni = 2 * snake_rounds(p.n_units); it < ni; ++it) {
    FwdUnit u;
    if (!fwd_item<CAUSAL>(p, snake_unit(it >> 1, p.n_units), it & 1, u)) continue;
    if (units > 0 && !wait1(&b->q_empty, (units - 1) & 1, b, p.status)) return;
    // The MMA issuer reads the unit's key-tile counts after its q_full wait
    // (the arrival below releases these stores); slot units & 1 was last read
    // two units ago, before that unit's Q tiles were released.
    *(volatile int*)&b->unit_nk[units & 1][0] = u.nk0;
    *(volatile int*)&b->unit_nk[units & 1][1] = u.nk1;
    mbar_arrive_expect_tx(&b->q_full, 2 * L::kTileBytes);
    ++units;  // number of times q_full has been armed
#pragma unroll
    for (int c = 0; c < NB; ++c) {
      tma_load_3d(smem + L::kQ0 + c * 16384, tm_q, &b->q_full, c * 64, u.q0, u.bh);
      tma_load_3d(smem + L::kQ1 + c * 16384, tm_q, &b->q_full, c * 64, u.q0 + 128, u.bh);
    }
    const int nk = max(u.nk0, u.nk1);
    for (int j = 0; j < nk; ++j) {
      {
        const int st = kc % S;
        if (kc >= S && !wait1(&b->k_empty[st], ((kc / S) - 1) & 1, b, p.status)) return;
        mbar_arrive_expect_tx(&b->k_full[st], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem + L::kK + st * L::kTileBytes + c * 16384, tm_k, &b->k_full[st],
                      c * 64, j * 128, u.bh);
        ++kc;
      }
      {
        const int st = vc % S;
        if (vc >= S && !wait1(&b->v_empty[st], ((vc / S) - 1) & 1, b, p.status)) return;
        mbar_arrive_expect_tx(&b->v_full[st], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < NB; ++c)
          tma_load_3d(smem + L::kV + st * L::kTileBytes + c * 16384, tm_v, &b->v_full[st],
                      c * 64, j * 128, u.bh);
        ++vc;
      }
    }
  }
}

// ---------------------------------------------------------------- MMA issuer
// S = Q K^T: K-major operands; each K-step reads the next 32 bytes of every
// row (16 bf16 or 32 E4M3 elements), and a bf16 row of D > 64 continues in
// the next 64-column box.
template <int D, bool FP8>
__device__ __forceinline__ void issue_s(uint32_t tmem_s, uint32_t q_smem, uint32_t k_smem) {
  if constexpr (FP8) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, 128, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk)
      mma_ss_f8(tmem_s, sdesc_sw128(q_smem + kk * 32, 16, 1024),
                sdesc_sw128(k_smem + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  } else {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
      mma_ss(tmem_s, sdesc_sw128(q_smem + off, 16, 1024), sdesc_sw128(k_smem + off, 16, 1024),
             idesc, kk > 0 ? 1u : 0u);
    }
  }
}

// O += P V: A = P from TMEM (8 columns per K-step in both types: 16 bf16 or
// 32 E4M3 keys), B = V MN-major (a K-step covers 16 or 32 key rows of 128
// bytes; bf16 rows of D = 128 span two 64-column boxes 16 KB apart).
// HALF = 0 / 1 issues only the K-steps of keys 0-63 / 64-127 (bf16).
template <int D, bool FP8, int HALF = -1>
__device__ __forceinline__ void issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_smem,
                                         bool accumulate) {
  if constexpr (FP8) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, D, false, true);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts_f8(tmem_o, tmem_p + kk * 8, sdesc_sw128(v_smem + kk * 4096, 16384, 1024), idesc,
                (accumulate || kk > 0) ? 1u : 0u);
  } else {
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
    for (int kk = (HALF == 1 ? 4 : 0); kk < (HALF == 0 ? 4 : 8); ++kk)
      mma_ts(tmem_o, tmem_p + kk * 8, sdesc_sw128(v_smem + kk * 2048, 16384, 1024), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_mma(const FwdParams& p, uint8_t* smem, FwdBarriers* b, uint32_t tmem) {
  using L = FwdLayout<D, FP8>;
  // O_i += P_i V for Q tile i.  bf16: the keys 0-63 half is issued as soon
  // as the softmax has stored it, the rest when the whole P is in TMEM.
  auto pv = [&](int i, int& pcount, uint32_t to, uint32_t ts, uint32_t v_smem, bool acc) -> bool {
    if constexpr (!FP8) {
      if (!wait1(&b->p_half[i], pcount & 1, b, p.status)) return false;
      tc_fence_after();
      issue_pv<D, FP8, 0>(to, ts, v_smem, acc);
    }
    if (!wait1(&b->p_full[i], pcount & 1, b, p.status)) return false;
    ++pcount;
    tc_fence_after();
    if constexpr (!FP8)
      issue_pv<D, FP8, 1>(to, ts, v_smem, true);
    else
      issue_pv<D, FP8>(to, ts, v_smem, acc);
    return true;
  };
  constexpr int S = L::kStages;
  const uint32_t sb = smem_u32(smem);
  const uint32_t tS[2] = {tmem + 0, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
  const uint32_t qs[2] = {sb + L::kQ0, sb + L::kQ1};
  int qc = 0, kc = 0, vc = 0;
  int pc[2] = {0, 0};
  for (int it = 0, ni = 2 * snake_rounds(p.n_units); it < ni; ++it) {
    if (!fwd_item_exists<CAUSAL>(p, snake_unit(it >> 1, p.n_units), it & 1)) continue;
    if (!wait1(&b->q_full, qc & 1, b, p.status)) return;
    const int nk0 = *(volatile int*)&b->unit_nk[qc & 1][0];
    const int nk1 = *(volatile int*)&b->unit_nk[qc & 1][1], nk = max(nk0, nk1);
    ++qc;
    tc_fence_after();
    for (int j = 0; j < nk; ++j) {
      const int ks = kc % S;
      if (!wait1(&b->k_full[ks], (kc / S) & 1, b, p.status)) return;
      tc_fence_after();
      const uint32_t k_smem = sb + L::kK + ks * L::kTileBytes;
      const int vs = vc % S;
      const uint32_t v_smem = sb + L::kV + vs * L::kTileBytes;
      if (j >= 1) {
        if (!wait1(&b->v_full[vs], (vc / S) & 1, b, p.status)) return;
        tc_fence_after();
      }
      if (j >= 1 && j - 1 < nk0) {
        if (!pv(0, pc[0], tO[0], tS[0], v_smem, j - 1 > 0)) return;
        if (j - 1 == nk0 - 1) mma_commit(&b->o_full[0]);
      }
      if (j < nk0) {
        issue_s<D, FP8>(tS[0], qs[0], k_smem);
        mma_commit(&b->s_full[0]);
      }
      if (j >= 1 && j - 1 < nk1) {
        if (!pv(1, pc[1], tO[1], tS[1], v_smem, j - 1 > 0)) return;
        if (j - 1 == nk1 - 1) mma_commit(&b->o_full[1]);
      }
      if (j >= 1) {
        mma_commit(&b->v_empty[vs]);
        ++vc;
      }
      if (j < nk1) {
        issue_s<D, FP8>(tS[1], qs[1], k_smem);
        mma_commit(&b->s_full[1]);
      }
      mma_commit(&b->k_empty[ks]);
      ++kc;
    }
    mma_commit(&b->q_empty);
    // P V for the last key tile.
    const int vs = vc % S;
    const uint32_t v_smem = sb + L::kV + vs * L::kTileBytes;
    if (!wait1(&b->v_full[vs], (vc / S) & 1, b, p.status)) return;
    tc_fence_after();
    if (nk - 1 < nk0) {
      if (!pv(0, pc[0], tO[0], tS[0], v_smem, nk - 1 > 0)) return;
      mma_commit(&b->o_full[0]);
    }
    if (nk - 1 < nk1) {
      if (!pv(1, pc[1], tO[1], tS[1], v_smem, nk - 1 > 0)) return;
      mma_commit(&b->o_full[1]);
    }
    mma_commit(&b->v_empty[vs]);
    ++vc;
  }
}

// ---------------------------------------------------------------- softmax
// Two probabilities as E4M3 (x.x in the low byte), and that pair back as f16.
__device__ __forceinline__ uint32_t pack_e4m3x2(float2 x) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint32_t v) {
  return __half2(__nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3));
}

// Which exponential pairs of an unmasked tile take the polynomial exp2 on the
// FMA pipe instead of MUFU.  The balance between the two pipes, and where
// in the unrolled loop the polynomial pairs sit, were measured per case
// (forward alone, causal and non-causal B=2 H=32 N=4096 d=128, A/B on one
// box): bf16 is fastest with pair 4 of every 8 (246 against 253 µs causal
// with pairs 0-2, and 458 against 481-512 µs non-causal); FP8 with pair 0 of
// every 8 when causal (228 against 241 µs) and pairs 0-2 otherwise (412 µs;
// one pair in eight: 441).
__device__ __forceinline__ bool bf16_poly_pair(int q2) { return (q2 & 7) == 4; }
template <bool CAUSAL>
__device__ __forceinline__ bool fp8_poly_pair(int q2) {
  return CAUSAL ? (q2 & 7) == 0 : (q2 & 7) < 3;
}

// FP8: P of one 128-key tile as E4M3, four keys per TMEM column (16 columns
// per half of 64 keys).  Adds the unrounded p to rs (for lse) and returns the
// sum of the rounded p (O's normaliser), accumulated in f16 pairs over 8
// pairs and then in fp32.  Masked tiles use the MUFU exp2 throughout so that
// masked probabilities are exactly 0; others take the polynomial on some
// pairs (FP8_POLY_PAIR below).
template <bool MASKED, bool CAUSAL>
__device__ __forceinline__ float fp8_p_tile(const float* s, float2 sl2v, float2 nmb, float2* rs,
                                            uint32_t tS) {
  float lq = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[16];
    __half2 hq[4] = {__float2half2_rn(0.f), __float2half2_rn(0.f), __float2half2_rn(0.f),
                     __float2half2_rn(0.f)};
#pragma unroll
    for (int q4 = 0; q4 < 16; ++q4) {
      const int c = 64 * h + 4 * q4;
      const float2 xa = fma2(make_float2(s[c], s[c + 1]), sl2v, nmb);
      const float2 xb = fma2(make_float2(s[c + 2], s[c + 3]), sl2v, nmb);
      const int qa = 2 * q4, qb = 2 * q4 + 1;
      float2 pa, pb;
      if (!MASKED && fp8_poly_pair<CAUSAL>(qa))
        pa = exp2_poly2(xa);
      else
        pa = make_float2(ex2_approx(xa.x), ex2_approx(xa.y));
      if (!MASKED && fp8_poly_pair<CAUSAL>(qb))
        pb = exp2_poly2(xb);
      else
        pb = make_float2(ex2_approx(xb.x), ex2_approx(xb.y));
      rs[qa & 3] = add2(rs[qa & 3], pa);
      rs[qb & 3] = add2(rs[qb & 3], pb);
      const uint32_t ea = pack_e4m3x2(pa), eb = pack_e4m3x2(pb);
      pk[q4] = ea | (eb << 16);
      hq[q4 & 3] = __hadd2(hq[q4 & 3], __hadd2(e4m3x2_to_half2(ea), e4m3x2_to_half2(eb)));
    }
    tmem_st_x16(tS + 16 * h, pk);
    const float2 f = __half22float2(__hadd2(hq[0], hq[1]));
    const float2 g = __half22float2(__hadd2(hq[2], hq[3]));
    lq += (f.x + f.y) + (g.x + g.y);
  }
  return lq;
}

template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_softmax(const FwdParams& p, FwdBarriers* b, uint32_t tmem, int wg) {
  const int t = threadIdx.x - 128 * (wg + 1);  // row within the Q tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const uint32_t tS = tmem + lane_base + (wg ? 128u : 0u);
  const uint32_t tO = tmem + lane_base + 256u + wg * D;
  const int N = p.N;
  int sc = 0, oc = 0;
  for (int it = 0, ni = 2 * snake_rounds(p.n_units); it < ni; ++it) {
    FwdUnit u;
    if (!fwd_item<CAUSAL>(p, snake_unit(it >> 1, p.n_units), it & 1, u)) continue;
    const int nk = wg ? u.nk1 : u.nk0;
    const int tile_row0 = u.q0 + wg * 128;
    const int row = tile_row0 + t;
    // FP8: the scores of E4M3 Q and K carry the two per-head descale factors.
    const float sl2 = FP8 ? fmaxf(p.scale_log2 * __ldg(p.descale_q + u.bh) *
                                      __ldg(p.descale_k + u.bh), FLT_MIN)
                          : p.scale_log2;
    float m_used = -INFINITY;  // reference max (exp2 domain) of O and l
    float l = 0.f;
    float lq = 0.f;  // FP8: sum of the E4M3-rounded p (O's normaliser)
    for (int j = 0; j < nk; ++j) {
      if (!wait_warp(&b->s_full[wg], sc & 1, b, p.status)) return;
      ++sc;
      tc_fence_after();
      uint32_t r[128];
      tmem_ld_x128(tS, r);
      float* s = reinterpret_cast<float*>(r);
      const int key0 = j * 128;
      const bool need_mask = (key0 + 128 > N) || (CAUSAL && key0 + 127 > tile_row0);
      if (need_mask) {
        const int lim = CAUSAL ? min(row + 1, N) : N;  // keys < lim are visible
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (key0 + c < lim) ? s[c] : -INFINITY;
      }
      // Row maximum: four independent chains of three-input max.
      float mx[4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        mx[k4] = fmaxf(s[32 * k4], s[32 * k4 + 1]);
#pragma unroll
        for (int c = 32 * k4 + 2; c < 32 * k4 + 32; c += 2) mx[k4] = max3(mx[k4], s[c], s[c + 1]);
      }
      float m_tile = max3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      m_tile *= sl2;
      const bool need = m_tile > m_used + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = fmaxf(m_used, m_tile);
        const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_used - m_new);
        l *= alpha;
        lq *= alpha;
        if (j > 0) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t o[16];
            tmem_ld_x16(tO + c0, o);
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x16(tO + c0, o);
          }
        }
        m_used = m_new;
      }
      const float mb = (m_used == -INFINITY) ? 0.f : m_used;
      const float2 sl2v = make_float2(sl2, sl2);
      const float2 nmb = make_float2(-mb, -mb);
      float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      // P in two halves of 64 keys; each half is stored as soon as it is
      // packed (S is already in registers, so overwriting it is safe), and
      // for bf16 the first half is published at once, so the P V MMA of
      // keys 0-63 overlaps the exponentials of keys 64-127.  On
      // unmasked tiles some pairs (bf16_poly_pair, fp8_poly_pair) take the
      // polynomial exp2 on the FMA pipe and the rest the MUFU unit; masked
      // tiles (which hold -inf) use the MUFU unit throughout so masked
      // probabilities are exactly 0.
      if constexpr (FP8) {
        if (need_mask)
          lq += fp8_p_tile<true, CAUSAL>(s, sl2v, nmb, rs, tS);
        else
          lq += fp8_p_tile<false, CAUSAL>(s, sl2v, nmb, rs, tS);
      } else if (need_mask) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) {
            const int c = 64 * h + 2 * q2;
            const float2 x = fma2(make_float2(s[c], s[c + 1]), sl2v, nmb);
            const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            rs[q2 & 3] = add2(rs[q2 & 3], pp);
            pk[q2] = pack_bf16x2(pp.x, pp.y);
          }
          tmem_st_x32(tS + 32 * h, pk);
          if (h == 0) {  // keys 0-63 of P are ready: the MMA may start on them
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&b->p_half[wg]);
          }
        }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) {
            const int c = 64 * h + 2 * q2;
            const float2 x = fma2(make_float2(s[c], s[c + 1]), sl2v, nmb);
            const float2 pp = bf16_poly_pair(q2) ? exp2_poly2(x)
                                             : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            rs[q2 & 3] = add2(rs[q2 & 3], pp);
            pk[q2] = pack_bf16x2(pp.x, pp.y);
          }
          tmem_st_x32(tS + 32 * h, pk);
          if (h == 0) {  // keys 0-63 of P are ready: the MMA may start on them
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&b->p_half[wg]);
          }
        }
      }
      const float2 rsum = add2(add2(rs[0], rs[1]), add2(rs[2], rs[3]));
      l += rsum.x + rsum.y;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(&b->p_full[wg]);  // one arrival per warp
    }
    if (nk == 0) continue;  // a tile wholly past the last row: nothing to write
    // Epilogue: O = o / l, lse = (m + log2 l) ln 2.
    if (!wait_warp(&b->o_full[wg], oc & 1, b, p.status)) return;
    ++oc;
    tc_fence_after();
    // FP8: O = descale_v * (sum p~ v) / (sum p~).
    const float inv_l = FP8 ? __ldg(p.descale_v + u.bh) / lq : 1.f / l;
    const bool valid = row < N;
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(u.bh) * N + row) * D;
    uint32_t o[D];
    if (D == 128)
      tmem_ld_x128(tO, o);
    else
      tmem_ld_x64(tO, o);
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
      for (int v = 0; v < D / 8; ++v)
        dst[v] = make_uint4(
            pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l),
            pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l),
            pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l),
            pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
    }
    if (valid) p.lse[static_cast<size_t>(u.bh) * N + row] = (m_used + __log2f(l)) * 0.69314718055994531f;
    // Consistency check: the reference maximum never exceeds the row's
    // maximum score, so that key alone adds 2^0 = 1 to the normaliser, up to
    // the rounding of the exponent and of the exponential (relative 2^-13 at
    // worst, also after E4M3 rounding of p); a normaliser below 1/2, or not
    // finite (which non-finite inputs also give), latches the assert bit.
    if (valid && !(((FP8 ? lq : l) >= 0.5f) && ((FP8 ? lq : l) <= FLT_MAX)))
      atomicOr(p.status, kDevAssert);
  }
}

// ---------------------------------------------------------------- kernel
template <int D, bool CAUSAL, bool FP8 = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  FwdBarriers* b = reinterpret_cast<FwdBarriers*>(smem + L::kBar);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&b->q_full, 1);
    mbar_init(&b->q_empty, 1);
    for (int i = 0; i < L::kStages; ++i) {
      mbar_init(&b->k_full[i], 1);
      mbar_init(&b->k_empty[i], 1);
      mbar_init(&b->v_full[i], 1);
      mbar_init(&b->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->s_full[i], 1);
      mbar_init(&b->p_full[i], 4);
      mbar_init(&b->p_half[i], 4);
      mbar_init(&b->o_full[i], 1);
    }
    mbar_init(&b->mma_done, 1);
    b->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane_id() == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
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
    // Softmax warpgroups: take the registers warpgroup 0 gives up.
    regs_increase<kFwdSoftmaxRegs>();
    fwd_softmax<D, CAUSAL, FP8>(p, b, tmem, (warp - 4) >> 2);
  } else {
    regs_decrease<kFwdCtlRegs>();
    if (warp == 0) {
      if (lane_id() == 0) {
        int kc = 0, vc = 0, units = 0;
        fwd_producer<D, CAUSAL, FP8>(&tm_q, &tm_k, &tm_v, p, smem, b, kc, vc, units);
        // Wait for every TMA load this thread armed (all long complete on the
        // normal path) so no copy is in flight when the CTA exits.
        constexpr int S = L::kStages;
        if (units > 0) mbar_wait(&b->q_full, (units - 1) & 1, p.status);
        for (int st = 0; st < S; ++st) {
          const int nk = kc / S + (st < kc % S ? 1 : 0);
          const int nv = vc / S + (st < vc % S ? 1 : 0);
          if (nk > 0) mbar_wait(&b->k_full[st], (nk - 1) & 1, p.status);
          if (nv > 0) mbar_wait(&b->v_full[st], (nv - 1) & 1, p.status);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane_id() == 0) {
        fwd_mma<D, CAUSAL, FP8>(p, smem, b, tmem);
        // Drain every MMA this thread issued before TMEM is released.
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
