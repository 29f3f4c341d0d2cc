// Prefill forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), bf16 in,
// fp32 accumulate, bf16 O and fp32 LSE out.
//
// Method: exact attention computed tile by tile with an online softmax, never writing
// the score matrix to HBM (CSDN interview article «注意力变体深挖», section 6.2 tiling
// and online-softmax merge; gocoding blog section 4, kernel fusion).  The pages'
// SRAM-tiling description targets older GPUs; this kernel is organised around sm_100a:
//
//  * One CTA owns two 128-row query tiles ("slots") that read the same K/V tiles: two
//    query heads of one KV group at the same positions (GQA: one K/V tile load serves
//    both heads), or, when the group has an odd head left over, two consecutive query
//    tiles of that head.
//  * warp 0 (one thread) streams Q once and K/V tiles of 128 keys through a 2-stage
//    shared-memory ring with TMA (128-byte swizzle).
//  * warp 1 (one thread) issues tcgen05 MMAs: S_i = Q_i K^T (A, B from shared memory)
//    into TMEM, and O_i += P_i V with P_i read from TMEM (it overwrites S_i as bf16).
//  * warps 2-5 and 6-9 are the softmax warpgroups of slot 0 and 1.  TMEM lane r holds
//    query row r, so each thread owns one full row: its row max and row sum need no
//    cross-lane reduction.  Scores are scaled into the log2 domain with one FFMA and
//    exponentiated with ex2.  The output is rescaled only when the running max grows
//    by more than 2^8 (the final O / l uses the same stale reference, so this is exact).
//  * TMEM (512 columns): S_0 | S_1 | O_0 | O_1.
//  * While one slot runs its softmax the tensor pipe works on the other slot.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace attn {
namespace tc {

constexpr int BM = 128;  // query rows per tile (MMA M)
constexpr int BN = 128;  // keys per K/V tile
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Layout {
  static constexpr int kTile = BM * D * 2;  // bytes of one Q, K or V tile (BN == BM)
  static constexpr int kBox = BM * 128;     // bytes of one 64-column TMA box
  static constexpr int kQ = 0;              // Q[2]
  static constexpr int kK = 2 * kTile;      // K[2]
  static constexpr int kV = 4 * kTile;      // V[2]
  static constexpr int kBar = 6 * kTile;
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static constexpr uint32_t kColS0 = 0, kColS1 = BN, kColO0 = 2 * BN, kColO1 = 2 * BN + D;
  static constexpr uint32_t kTmemCols = 512;
};

// barrier indices
enum : int {
  kBarQ = 0,
  kBarKFull = 1,   // [2]
  kBarKEmpty = 3,  // [2]
  kBarVFull = 5,   // [2]
  kBarVEmpty = 7,  // [2]
  kBarSFull = 9,   // [2] per slot: S_i written
  kBarPFull = 11,  // [2] per slot: P_i written and O_i rescaled (128 arrivals)
  kBarODone = 13,  // [2] per slot: PV_i finished
  kBarDrain = 15,
};

struct Params {
  void* o;
  float* lse;
  int B, Hq, Hkv, Sq, Sk;
  float scale_log2;  // scale * log2(e)
  int causal;
  int nq;           // query tiles per head
  int pairs;        // head pairs per KV group (g / 2)
  int items_a;      // work items made of head pairs
  int npq;          // query-tile pairs of the leftover head when g is odd
};

struct Item {
  int b, kvh;
  int h[2], t[2], n[2];
};

__device__ __forceinline__ int kv_tiles(const Params& p, int t) {
  if (!p.causal) return (p.Sk + BN - 1) / BN;
  long long last = (long long)t * BM + BM - 1 + (long long)p.Sk - p.Sq;
  if (last > p.Sk - 1) last = p.Sk - 1;
  return last < 0 ? 0 : (int)(last / BN) + 1;
}

// Work items, longest first under a causal mask.  Items [0, items_a): two heads of one KV
// group, same query tile.  Items [items_a, ...): the leftover head of an odd group, query
// tiles 2t and 2t+1.
__device__ __forceinline__ Item decode_item(const Params& p, int idx) {
  Item it;
  const int g = p.Hq / p.Hkv;
  if (idx < p.items_a) {
    const int per_t = p.B * p.Hkv * p.pairs;
    const int tr = idx / per_t;
    int rem = idx - tr * per_t;
    const int t = p.causal ? p.nq - 1 - tr : tr;
    it.b = rem / (p.Hkv * p.pairs);
    rem -= it.b * p.Hkv * p.pairs;
    it.kvh = rem / p.pairs;
    const int pp = rem - it.kvh * p.pairs;
    it.h[0] = it.kvh * g + 2 * pp;
    it.h[1] = it.h[0] + 1;
    it.t[0] = it.t[1] = t;
  } else {
    idx -= p.items_a;
    const int per = p.B * p.Hkv;
    const int tr = idx / per;
    const int rem = idx - tr * per;
    const int tp = p.causal ? p.npq - 1 - tr : tr;
    it.b = rem / p.Hkv;
    it.kvh = rem - it.b * p.Hkv;
    it.h[0] = it.h[1] = it.kvh * g + g - 1;
    it.t[0] = 2 * tp;
    it.t[1] = 2 * tp + 1;
  }
  for (int i = 0; i < 2; ++i) it.n[i] = it.t[i] < p.nq ? kv_tiles(p, it.t[i]) : 0;
  return it;
}

// All lanes wait; the warp proceeds only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Item it = decode_item(p, blockIdx.x);
  const int N = max(it.n[0], it.n[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), 128);
      mbar_init(bar(kBarODone + s), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t sQ[2] = {sbase + L::kQ, sbase + L::kQ + L::kTile};
  const uint32_t sK[2] = {sbase + L::kK, sbase + L::kK + L::kTile};
  const uint32_t sV[2] = {sbase + L::kV, sbase + L::kV + L::kTile};
  const uint32_t colS[2] = {L::kColS0, L::kColS1};
  const uint32_t colO[2] = {L::kColO0, L::kColO1};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && N > 0) {
      int k_fill[2] = {-1, -1}, v_fill[2] = {-1, -1};
      uint32_t qbytes = 0;
      for (int i = 0; i < 2; ++i) qbytes += it.n[i] > 0 ? (uint32_t)L::kTile : 0u;
      mbar_arrive_expect_tx(bar(kBarQ), qbytes);
      for (int i = 0; i < 2; ++i) {
        if (it.n[i] == 0) continue;
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ[i] + c * L::kBox, &tmQ, bar(kBarQ), c * 64, it.t[i] * BM,
                      it.b * p.Hq + it.h[i]);
      }
      const int zkv = it.b * p.Hkv + it.kvh;
      for (int j = 0; j < N; ++j) {
        const int s = j & 1;
        const int f = j >> 1;
        if (f > 0 && !mbar_wait(bar(kBarKEmpty + s), (f - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(kBarKFull + s), L::kTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sK[s] + c * L::kBox, &tmK, bar(kBarKFull + s), c * 64, j * BN, zkv);
        k_fill[s] = f;
        if (f > 0 && !mbar_wait(bar(kBarVEmpty + s), (f - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(kBarVFull + s), L::kTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sV[s] + c * L::kBox, &tmV, bar(kBarVFull + s), c * 64, j * BN, zkv);
        v_fill[s] = f;
      }
      if (*abort_flag) {
        // Let copies already in flight land before the CTA's shared memory is released.
        int never = 0;
        mbar_wait(bar(kBarQ), 0, &never, 100000000ull);
        for (int s = 0; s < 2; ++s) {
          if (k_fill[s] >= 0) mbar_wait(bar(kBarKFull + s), k_fill[s] & 1, &never, 100000000ull);
          if (v_fill[s] >= 0) mbar_wait(bar(kBarVFull + s), v_fill[s] & 1, &never, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && N > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
      auto issue_s = [&](int i, int s) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * L::kBox + (uint32_t)(kk & 3) * 32u;
          const uint64_t a = smem_desc_sw128(sQ[i] + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(sK[s] + off, 16, 1024);
          mma_ss(tmem + colS[i], a, b, idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull + i));
      };
      auto issue_pv = [&](int i, int s, int j) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // V tile: 128 key rows of 128 bytes per 64-column box; MN-major B operand.
          const uint64_t b = smem_desc_sw128(sV[s] + (uint32_t)kk * 2048u, L::kBox, 1024);
          mma_ts(tmem + colO[i], tmem + colS[i] + (uint32_t)kk * 8u, b, idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(kBarODone + i));
      };

      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag) && mbar_wait(bar(kBarKFull), 0, abort_flag);
      if (ok) {
        for (int i = 0; i < 2; ++i)
          if (it.n[i] > 0) issue_s(i, 0);
        tc_commit(bar(kBarKEmpty));
      }
      for (int j = 0; ok && j < N; ++j) {
        const int s = j & 1;
        const int s1 = (j + 1) & 1;
        bool next_k = false;
        if (!(ok = mbar_wait(bar(kBarVFull + s), (j >> 1) & 1, abort_flag))) break;
        for (int i = 0; i < 2; ++i) {
          if (j < it.n[i]) {
            if (!(ok = mbar_wait(bar(kBarPFull + i), j & 1, abort_flag))) break;
            issue_pv(i, s, j);
          }
          if (j + 1 < it.n[i]) {
            if (!next_k) {
              if (!(ok = mbar_wait(bar(kBarKFull + s1), ((j + 1) >> 1) & 1, abort_flag))) break;
              next_k = true;
            }
            // S_i is overwritten only after PV_i(j) has read P_i from the same columns.
            if (!(ok = mbar_wait(bar(kBarODone + i), j & 1, abort_flag))) break;
            issue_s(i, s1);
          }
        }
        if (!ok) break;
        tc_commit(bar(kBarVEmpty + s));
        if (j + 1 < N) tc_commit(bar(kBarKEmpty + s1));
      }
      if (!ok) {
        int never = 0;
        tc_commit(bar(kBarDrain));
        mbar_wait(bar(kBarDrain), 0, &never, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int i = (warp - 2) >> 2;  // slot
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int n = it.n[i];
    const int t = it.t[i];
    if (t < p.nq) {
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      const uint32_t tS = tmem + lane_off + colS[i];
      const uint32_t tO = tmem + lane_off + colO[i];
      const int qrow = t * BM + row;
      const long long key_limit = p.causal ? (long long)qrow + p.Sk - p.Sq : (long long)p.Sk - 1;
      const long long tile_limit = p.causal ? (long long)t * BM + p.Sk - p.Sq : (long long)p.Sk - 1;
      const float c = p.scale_log2;
      // l: fp32 row sum (for the LSE); lr: row sum of the bf16-rounded P that the tensor
      // core multiplies, so that O / lr uses exactly normalised weights.
      float m = -INFINITY, l = 0.f, lr = 0.f;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        if (!(ok = warp_wait(bar(kBarSFull + i), j & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t r[4][32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + 32u * q4, r[q4]);
        tmem_wait_ld();
        const int kv0 = j * BN;
        // Mask only tiles that reach past the last key or the causal diagonal.
        if ((long long)kv0 + BN - 1 > tile_limit || kv0 + BN > p.Sk) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int key = kv0 + q4 * 32 + e;
              if ((long long)key > key_limit || key >= p.Sk) r[q4][e] = __float_as_uint(-INFINITY);
            }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(r[q4][e]));
        const float m_new = fmaxf(m, mx * c);
        float alpha = 1.f;
        if (m_new > m + kRescaleThreshold) {  // also taken on the first finite max
          alpha = fast_exp2(m - m_new);
          m = m_new;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        float sum = 0.f, sum_r = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(r[q4][2 * e]), c, -mu));
            const float p1 = fast_exp2(fmaf(__uint_as_float(r[q4][2 * e + 1]), c, -mu));
            sum += p0 + p1;
            const uint32_t w = pack_bf16x2(p0, p1);
            sum_r += bf16lo(w) + bf16hi(w);
            r[q4 >> 1][(q4 & 1) * 16 + e] = w;
          }
        }
        l = l * alpha + sum;
        lr = lr * alpha + sum_r;
        // P (bf16 pairs) overwrites the first 64 columns of S_i.
        tmem_st32(tS, r[0]);
        tmem_st32(tS + 32u, r[1]);
        tmem_wait_st();
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!(ok = warp_wait(bar(kBarODone + i), (j - 1) & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            tmem_ld32(tO + 32u * c4, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + 32u * c4, ov);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + i));
      }
      // ---------------------------------------------------------- epilogue
      if (ok && n > 0) ok = warp_wait(bar(kBarODone + i), (n - 1) & 1, abort_flag);
      if (ok) {
        tc_fence_after();
        const int bh = it.b * p.Hq + it.h[i];
        const bool in_range = qrow < p.Sq;
        const float inv_l = lr > 0.f ? 1.f / lr : 0.f;
        __nv_bfloat16* orow =
            reinterpret_cast<__nv_bfloat16*>(p.o) + ((size_t)bh * p.Sq + (in_range ? qrow : 0)) * D;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t ov[32];
          if (n > 0) {
            tmem_ld32(tO + 32u * c4, ov);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        if (p.lse != nullptr && in_range)
          p.lse[(size_t)bh * p.Sq + qrow] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace tc
}  // namespace attn
