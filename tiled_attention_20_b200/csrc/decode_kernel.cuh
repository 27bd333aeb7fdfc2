// decode_kernel.cuh -- attention of a few new queries against a key/value
// cache, split along the cached keys.
//
// "第17讲 Tensor Core、HBM、SRAM 与 FlashAttention" §9.2: a decode step handles
// one or a few new tokens, and low-batch decode tends to be limited by memory
// traffic; §9.3: the KV cache holds the keys and values of earlier tokens,
// which each step reads instead of recomputing.  With Nq <= 8 queries per head
// the work is a pass over the cached K and V rows, so the kernel is written
// for HBM bandwidth on the CUDA cores (no tensor-core tile would be more than
// 8/128 full) and the parallelism comes from splitting each head's cache.
//
// One CTA takes one (batch, head) and one contiguous chunk of cache rows.  A
// producer warp streams the chunk's K tiles, then its V tiles, through a ring
// of shared-memory stages with 1-D bulk copies (one head's rows are
// contiguous).  Eight compute warps then work in two passes, without any
// rescaling inside the chunk:
//   pass 1: s_j = scale*log2(e) * q . k_j for every key of the chunk, kept in
//           shared memory; the chunk's max m and p_j = 2^(s_j - m), l = sum p_j;
//   pass 2: o = sum_j p_j v_j.
// (m, l, o) of a chunk is a partial softmax state.  The CTA that finishes a
// head last merges the states with the rescaling of the online softmax (same
// page, §8.3): M = max m_s, L = sum l_s 2^(m_s - M), O = sum o_s 2^(m_s - M) / L.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fa {

constexpr int kDecTileKeys = 64;
constexpr int kDecComputeThreads = 256;  // 8 compute warps
constexpr int kDecThreads = 288;         // + 1 producer warp

// Queries per head are padded to NQP in {1, 2, 4, 8}.
constexpr int dec_nqp(int nq) { return nq <= 1 ? 1 : nq <= 2 ? 2 : nq <= 4 ? 4 : 8; }

template <int D, int NQP>
struct DecLayout {
  static constexpr int kStages = 4;
  static constexpr int kTileBytes = kDecTileKeys * D * 2;
  // Longest chunk of keys a CTA takes: its scores fill at most 16 KB.
  static constexpr int kMaxChunk = 4096 / NQP;
  static constexpr int kRing = 0;
  static constexpr int kS = kRing + kStages * kTileBytes;
  static constexpr int kRed = kS + kMaxChunk * NQP * 4;  // [8 warps][NQP] floats
  static constexpr int kStat = kRed + 8 * NQP * 4;       // m[NQP], l[NQP], last-CTA flag
  static constexpr int kBar = (kStat + 2 * NQP * 4 + 4 + 15) / 16 * 16;
  static constexpr int kSmemBytes = kBar + 2 * kStages * 8;
  // The cross-warp sum of o reuses the ring once every tile is consumed.
  static_assert(8 * NQP * D * 4 <= kStages * kTileBytes, "o reduction must fit in the ring");
};

struct DecodeParams {
  const uint16_t* q;  // [B, H, Nq, D] bf16
  const uint16_t* k;  // [B, H, ld, D] bf16
  const uint16_t* v;
  uint16_t* o;        // [B, H, Nq, D] bf16
  float* lse;         // [B, H, Nq]
  const int* lens;    // [B] valid cache rows, or null (all Nk)
  float* part_o;      // [B*H][splits][NQP][D] unnormalised partial outputs
  float* part_ml;     // [B*H][splits][NQP][2] partial (m, l), log2 domain
  int* counter;       // [B*H] CTAs finished per head; zero between calls
  int* status;
  int H, Nq, Nk, ld, splits, chunk;
  float scale_log2;   // scale * log2(e)
  int causal;
};

// bf16 pairs of a 32-bit word to fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// One step of a transposing sum over the 8 lanes of a key group: lanes whose
// bit m is set keep the upper half of the C partial sums and trade the lower
// half with their partner, so after the three steps (m = 4, 2, 1) each lane
// holds one query's complete dot product (NQP = 8) or a duplicate of it.
template <int C, int NQP>
__device__ __forceinline__ void dec_xr_step(float (&v)[NQP], int m, int lane, int& q) {
  const bool hi = (lane & m) != 0;
  if constexpr (C >= 2) {
    constexpr int h = C / 2;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = hi ? v[i] : v[h + i];
      const float keep = hi ? v[h + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
    if (hi) q += h;
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
  }
}

template <int NQP>
__device__ __forceinline__ float dec_reduce8(float (&v)[NQP], int lane, int& q) {
  q = 0;
  constexpr int C1 = NQP;
  constexpr int C2 = C1 >= 2 ? C1 / 2 : 1;
  constexpr int C3 = C2 >= 2 ? C2 / 2 : 1;
  dec_xr_step<C1>(v, 4, lane, q);
  dec_xr_step<C2>(v, 2, lane, q);
  dec_xr_step<C3>(v, 1, lane, q);
  return v[0];
}

// Sum (or max) over the 256 compute threads of a per-thread value that
// belongs to query (t % NQP); the result for query q lands in out[q].
template <int NQP, bool MAX>
__device__ __forceinline__ void dec_block_reduce(float x, float* red, float* out, int t) {
  const int lane = t & 31, warp = t >> 5;
#pragma unroll
  for (int m = NQP; m < 32; m <<= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, m);
    x = MAX ? fmaxf(x, y) : x + y;
  }
  if (lane < NQP) red[warp * NQP + lane] = x;
  asm volatile("bar.sync 1, 256;" ::: "memory");
  if (t < NQP) {
    float r = red[t];
#pragma unroll
    for (int w = 1; w < 8; ++w) r = MAX ? fmaxf(r, red[w * NQP + t]) : r + red[w * NQP + t];
    out[t] = r;
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <int D, int NQP>
__global__ void __launch_bounds__(kDecThreads) fa_decode_kernel(const DecodeParams p) {
  using L = DecLayout<D, NQP>;
  constexpr int S = L::kStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + S;
  float* sbuf = reinterpret_cast<float*>(smem + L::kS);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* stat_m = reinterpret_cast<float*>(smem + L::kStat);
  float* stat_l = stat_m + NQP;
  int* last_flag = reinterpret_cast<int*>(stat_l + NQP);

  const int t = threadIdx.x;
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.H;
  int len = p.Nk;
  if (p.lens != nullptr) {
    len = p.lens[b];
    len = len < 0 ? 0 : (len > p.Nk ? p.Nk : len);
  }
  const int k0 = split * p.chunk;
  const int nkeys = max(min(k0 + p.chunk, len) - k0, 0);
  const int T = (nkeys + kDecTileKeys - 1) / kDecTileKeys;

  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);  // one arrival per compute warp
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (t >= kDecComputeThreads) {
    // ------------------------------------------------------------ producer
    if (t == kDecComputeThreads) {
      const size_t head = static_cast<size_t>(bh) * p.ld + k0;
      int issued = 0;
      for (int i = 0; i < 2 * T; ++i) {
        const int s = i % S, n = i / S;
        if (n > 0 && !mbar_wait(&empty[s], (n - 1) & 1, p.status)) break;
        const int tile = i < T ? i : i - T;
        const int rows = min(kDecTileKeys, nkeys - tile * kDecTileKeys);
        const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
        const uint16_t* src = (i < T ? p.k : p.v) + (head + static_cast<size_t>(tile) * kDecTileKeys) * D;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(smem + L::kRing + s * L::kTileBytes, src, bytes, &full[s]);
        issued = i + 1;
      }
      // Before the CTA may exit, the last copy into each stage has landed
      // (already true unless a wait above gave up).
      for (int s = 0; s < S && s < issued; ++s) {
        const int n = (issued - 1 - s) / S;  // uses of stage s, minus one
        mbar_wait(&full[s], n & 1, p.status);
      }
    }
    __syncthreads();
    return;
  }

  // -------------------------------------------------------------- compute
  const int lane = t & 31, warp = t >> 5;
  const int part = t & 7, kr = t >> 3;  // 8 lanes per key, 32 keys per sweep
  constexpr int EPT = D / 8;            // elements of a key row per lane
  constexpr int CH = EPT / 8;           // 16-byte chunks per lane: part, part + 8
  bool ok = true;

  // q (scaled into the log2 domain) for this lane's columns, fp32 registers.
  float qr[NQP][EPT];
#pragma unroll
  for (int qi = 0; qi < NQP; ++qi) {
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (qi < p.Nq)
        w = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(bh) * p.Nq + qi) * D +
                                            (part + 8 * c) * 8);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qr[qi][8 * c + 2 * e] = bf16_lo(ww[e]) * p.scale_log2;
        qr[qi][8 * c + 2 * e + 1] = bf16_hi(ww[e]) * p.scale_log2;
      }
    }
  }

  // Pass 1: scores of every key of the chunk into sbuf[key][query].
  const int vis0 = len - p.Nq;  // causal: query qi sees keys <= vis0 + qi
  for (int i = 0; i < T && ok; ++i) {
    const int s = i % S;
    if (!mbar_wait(&full[s], (i / S) & 1, p.status)) {
      ok = false;
      break;
    }
    const uint8_t* tile = smem + L::kRing + s * L::kTileBytes;
    const int rows = min(kDecTileKeys, nkeys - i * kDecTileKeys);
#pragma unroll
    for (int sweep = 0; sweep < 2; ++sweep) {
      const int kk = kr + 32 * sweep;
      float acc[NQP];
#pragma unroll
      for (int qi = 0; qi < NQP; ++qi) acc[qi] = 0.f;
      if (kk < rows) {
        float x[EPT];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(tile + kk * D * 2 + (part + 8 * c) * 16);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[8 * c + 2 * e] = bf16_lo(ww[e]);
            x[8 * c + 2 * e + 1] = bf16_hi(ww[e]);
          }
        }
#pragma unroll
        for (int qi = 0; qi < NQP; ++qi) {
          float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < EPT; e += 2)
            a2 = fma2(make_float2(qr[qi][e], qr[qi][e + 1]), make_float2(x[e], x[e + 1]), a2);
          acc[qi] = a2.x + a2.y;
        }
      }
      int myq;
      const float sv = dec_reduce8<NQP>(acc, lane, myq);
      constexpr int kUnused = 7 >> (NQP == 8 ? 3 : NQP == 4 ? 2 : NQP == 2 ? 1 : 0);
      if (kk < rows && (lane & kUnused) == 0 && myq < p.Nq) {
        const int j = i * kDecTileKeys + kk;
        const bool masked = p.causal && (k0 + j > vis0 + myq);
        sbuf[j * NQP + myq] = masked ? -INFINITY : sv;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");

  // Softmax statistics of the chunk: m per query, then p = 2^(s - m) in place
  // and l = sum p.  Thread t only touches query t % NQP.
  const int tq = t % NQP;
  const bool real_q = tq < p.Nq;
  const int n_el = nkeys * NQP;
  float mx = -INFINITY;
  if (real_q)
    for (int e = t; e < n_el; e += kDecComputeThreads) mx = fmaxf(mx, sbuf[e]);
  dec_block_reduce<NQP, true>(mx, red, stat_m, t);
  const float mq = stat_m[tq];
  float sum = 0.f;
  if (real_q)
    for (int e = t; e < n_el; e += kDecComputeThreads) {
      const float pe = (mq == -INFINITY) ? 0.f : ex2_approx(sbuf[e] - mq);
      sbuf[e] = pe;
      sum += pe;
    }
  dec_block_reduce<NQP, false>(sum, red, stat_l, t);

  // Pass 2: o = sum_j p_j v_j.  Warp w takes keys w, w + 8, ... of a tile;
  // lane l holds columns [CPL*l, CPL*l + CPL).
  constexpr int CPL = D / 32;
  float2 o_acc[NQP][CPL / 2];
#pragma unroll
  for (int qi = 0; qi < NQP; ++qi)
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) o_acc[qi][c] = make_float2(0.f, 0.f);
  for (int i = 0; i < T && ok; ++i) {
    const int g = T + i, s = g % S;
    if (!mbar_wait(&full[s], (g / S) & 1, p.status)) {
      ok = false;
      break;
    }
    const uint8_t* tile = smem + L::kRing + s * L::kTileBytes;
    const int rows = min(kDecTileKeys, nkeys - i * kDecTileKeys);
    for (int kk = warp; kk < rows; kk += 8) {
      const float* pj = sbuf + (i * kDecTileKeys + kk) * NQP;
      float pv[NQP];
      if constexpr (NQP >= 4) {
#pragma unroll
        for (int q4 = 0; q4 < NQP / 4; ++q4) {
          const float4 t4 = reinterpret_cast<const float4*>(pj)[q4];
          pv[4 * q4] = t4.x;
          pv[4 * q4 + 1] = t4.y;
          pv[4 * q4 + 2] = t4.z;
          pv[4 * q4 + 3] = t4.w;
        }
      } else {
#pragma unroll
        for (int qi = 0; qi < NQP; ++qi) pv[qi] = pj[qi];
      }
      float vf[CPL];
      if constexpr (CPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(tile + kk * D * 2 + lane * 8);
        vf[0] = bf16_lo(w.x);
        vf[1] = bf16_hi(w.x);
        vf[2] = bf16_lo(w.y);
        vf[3] = bf16_hi(w.y);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + kk * D * 2 + lane * 4);
        vf[0] = bf16_lo(w);
        vf[1] = bf16_hi(w);
      }
#pragma unroll
      for (int qi = 0; qi < NQP; ++qi) {
        const float2 pp = make_float2(pv[qi], pv[qi]);
#pragma unroll
        for (int c = 0; c < CPL / 2; ++c)
          o_acc[qi][c] = fma2(pp, make_float2(vf[2 * c], vf[2 * c + 1]), o_acc[qi][c]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  // Every tile has been consumed: the ring holds the per-warp sums of o.
  asm volatile("bar.sync 1, 256;" ::: "memory");
  float* ored = reinterpret_cast<float*>(smem + L::kRing);  // [8][NQP][D]
#pragma unroll
  for (int qi = 0; qi < NQP; ++qi)
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) {
      ored[(warp * NQP + qi) * D + lane * CPL + 2 * c] = o_acc[qi][c].x;
      ored[(warp * NQP + qi) * D + lane * CPL + 2 * c + 1] = o_acc[qi][c].y;
    }
  asm volatile("bar.sync 1, 256;" ::: "memory");

  constexpr float kLn2 = 0.6931471805599453f;
  const int nq_out = min(p.Nq, NQP);
  if (p.splits == 1) {
    // The chunk is the whole cache: normalise and write.
    for (int e = t; e < nq_out * D; e += kDecComputeThreads) {
      const int qi = e / D, c = e % D;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) acc += ored[(w * NQP + qi) * D + c];
      const float l = stat_l[qi];
      const float val = l > 0.f ? acc / l : 0.f;
      p.o[(static_cast<size_t>(bh) * p.Nq + qi) * D + c] =
          __bfloat16_as_ushort(__float2bfloat16_rn(val));
    }
    if (t < nq_out) {
      const float l = stat_l[t];
      p.lse[static_cast<size_t>(bh) * p.Nq + t] = l > 0.f ? (stat_m[t] + log2f(l)) * kLn2 : -INFINITY;
    }
  } else {
    const size_t slot = static_cast<size_t>(bh) * p.splits + split;
    for (int e = t; e < NQP * D; e += kDecComputeThreads) {
      const int qi = e / D, c = e % D;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) acc += ored[(w * NQP + qi) * D + c];
      p.part_o[(slot * NQP + qi) * D + c] = acc;
    }
    if (t < NQP) {
      p.part_ml[(slot * NQP + t) * 2] = stat_m[t];
      p.part_ml[(slot * NQP + t) * 2 + 1] = stat_l[t];
    }
    __threadfence();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (t == 0) *last_flag = (atomicAdd(&p.counter[bh], 1) == p.splits - 1) ? 1 : 0;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (*last_flag) {
      // Every chunk of this head is in: merge the partial states.
      __threadfence();
      const size_t base = static_cast<size_t>(bh) * p.splits;
      for (int e = t; e < nq_out * D; e += kDecComputeThreads) {
        const int qi = e / D, c = e % D;
        float M = -INFINITY;
        for (int s = 0; s < p.splits; ++s) M = fmaxf(M, __ldcg(p.part_ml + ((base + s) * NQP + qi) * 2));
        float Lsum = 0.f, acc = 0.f;
        if (M != -INFINITY) {
          for (int s = 0; s < p.splits; ++s) {
            const float ms = __ldcg(p.part_ml + ((base + s) * NQP + qi) * 2);
            if (ms == -INFINITY) continue;
            const float w = exp2f(ms - M);
            Lsum += __ldcg(p.part_ml + ((base + s) * NQP + qi) * 2 + 1) * w;
            acc += __ldcg(p.part_o + ((base + s) * NQP + qi) * D + c) * w;
          }
        }
        const float val = Lsum > 0.f ? acc / Lsum : 0.f;
        p.o[(static_cast<size_t>(bh) * p.Nq + qi) * D + c] =
            __bfloat16_as_ushort(__float2bfloat16_rn(val));
        if (c == 0)
          p.lse[static_cast<size_t>(bh) * p.Nq + qi] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
      }
      if (t == 0) p.counter[bh] = 0;  // ready for the next call
    }
  }
  __syncthreads();
}

}  // namespace fa
