// Backward pass of exact attention with recomputation (CSDN «注意力变体深挖» §6.2, technique 2,
// and 追问2/追问3: the backward does not keep the attention matrix, it recomputes it from
// Q, K, V, so memory stays O(n)).  The gradients are the derivative of the definition:
//
//   P = exp(scale * Q K^T - LSE)   (recomputed from the forward's LSE, masked)
//   dV = P^T dO,  dP = dO V^T,  Delta_i = dO_i . O_i,  dS = P * (dP - Delta)
//   dQ = scale * dS K,  dK = scale * dS^T Q   (dK, dV summed over a GQA group's heads)
//
// Three kernels, no atomics: Delta per query row; dK and dV per 64-key tile of a KV head
// (looping over the group's query heads and the query tiles that see the keys); dQ per
// 64-row query tile (looping over the key tiles it sees).  The products are warp-level
// bf16 tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation): each warp owns 16 rows of
// the CTA's 64-row tile, P and dS are rounded to bf16 as MMA operands, everything else
// stays fp32 until dQ, dK, dV are rounded to bf16 at the end.  The tiles a kernel streams
// (query tiles for dK/dV, key tiles for dQ) are double-buffered with cp.async groups.
#pragma once

#include "common.cuh"

namespace attn {
namespace bwd {

constexpr int kRows = 64;     // rows of every tile (queries or keys)
constexpr int kThreads = 128; // 4 warps x 16 rows

struct Params {
  const __nv_bfloat16* q;   // [B, Hq, Sq, D]
  const __nv_bfloat16* k;   // [B, Hkv, Sk, D]
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;   // forward output
  const float* lse;         // [B, Hq, Sq] forward LSE (natural log)
  const __nv_bfloat16* dout;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* delta;             // [B, Hq, Sq] workspace
  int B, Hq, Hkv, Sq, Sk;
  float scale, scale_log2;
  int causal, window;
};

// ---------------------------------------------------------------------- helpers

// A [64][D] bf16 tile in shared memory: 16-byte chunk c of row r sits at chunk c ^ (r & 7),
// so the 8 rows read by one ldmatrix phase hit 8 different bank groups.
template <int D>
__device__ __forceinline__ uint32_t toff(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0: zero-fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N committed groups of this thread are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// One 4-byte element; zero-filled when !valid (the source address must still be mapped).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

// Rows [row0, row0 + 64) of a [rows][D] bf16 matrix into a swizzled tile; rows past `rows`
// are zero-filled (their source address stays inside the matrix).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t tile, const __nv_bfloat16* src, int row0, int rows) {
  constexpr int kChunks = D / 8;
  for (int idx = threadIdx.x; idx < kRows * kChunks; idx += kThreads) {
    const int r = idx / kChunks, c = idx - r * kChunks;
    const bool ok = row0 + r < rows;
    const __nv_bfloat16* g = src + (size_t)(ok ? row0 + r : 0) * D + c * 8;
    cp_async16(tile + toff<D>(r, c), g, ok);
  }
}

// A fragment of rows [m0, m0 + 16), columns [k0, k0 + 16) of a row-major tile.
template <int D>
__device__ __forceinline__ void ld_a(uint32_t tile, int m0, int k0, uint32_t (&a)[4]) {
  const int t = threadIdx.x & 31, mi = t >> 3;
  const int r = m0 + (t & 7) + (mi & 1) * 8, c = (k0 >> 3) + (mi >> 1);
  ldsm_x4(tile + toff<D>(r, c), a[0], a[1], a[2], a[3]);
}

// B fragments of two n-tiles [n0, n0 + 16) for k in [k0, k0 + 16) from a tile stored [n][k]:
// (b[0], b[1]) for n0 .. n0+7 and (b[2], b[3]) for n0+8 .. n0+15.
template <int D>
__device__ __forceinline__ void ld_b_nk(uint32_t tile, int n0, int k0, uint32_t (&b)[4]) {
  const int t = threadIdx.x & 31, mi = t >> 3;
  const int r = n0 + (t & 7) + (mi >> 1) * 8, c = (k0 >> 3) + (mi & 1);
  ldsm_x4(tile + toff<D>(r, c), b[0], b[1], b[2], b[3]);
}

// The same from a tile stored [k][n] (transposed read).
template <int D>
__device__ __forceinline__ void ld_b_kn(uint32_t tile, int n0, int k0, uint32_t (&b)[4]) {
  const int t = threadIdx.x & 31, mi = t >> 3;
  const int r = k0 + (t & 7) + (mi & 1) * 8, c = (n0 >> 3) + (mi >> 1);
  ldsm_x4_t(tile + toff<D>(r, c), b[0], b[1], b[2], b[3]);
}

__device__ __forceinline__ uint32_t pack_rn(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Is key j visible to query row i?  (causal bottom-right aligned, optional window)
__device__ __forceinline__ bool visible(const Params& p, int i, int j) {
  if (j >= p.Sk || i >= p.Sq) return false;
  if (!p.causal) return true;
  const long long pos = (long long)i + p.Sk - p.Sq;
  if ((long long)j > pos) return false;
  return p.window <= 0 || (long long)j > pos - p.window;
}


// Delta_i = dO_i . O_i (fp32), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const Params p) {
  const long long rows = (long long)p.B * p.Hq * p.Sq;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* a = p.o + row * D;
  const __nv_bfloat16* b = p.dout + row * D;
  float s = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) s = fmaf(__bfloat162float(a[d]), __bfloat162float(b[d]), s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) p.delta[row] = s;
}

// dQ of one 64-row query tile of one query head.
template <int D>
__global__ void __launch_bounds__(kThreads) dq_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kTileBytes = kRows * D * 2;
  // Q, dO, then two buffers of (K, V): the next key tile loads while this one is used.
  const uint32_t sQ = smem_u32(smem), sO = sQ + kTileBytes, sKV = sO + kTileBytes;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  const int kvh = h / (p.Hq / p.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int q0 = qt * kRows;
  const __nv_bfloat16* qb = p.q + (size_t)bh * p.Sq * D;
  const __nv_bfloat16* ob = p.dout + (size_t)bh * p.Sq * D;
  const __nv_bfloat16* kb = p.k + ((size_t)b * p.Hkv + kvh) * p.Sk * D;
  const __nv_bfloat16* vb = p.v + ((size_t)b * p.Hkv + kvh) * p.Sk * D;

  load_tile<D>(sQ, qb, q0, p.Sq);
  load_tile<D>(sO, ob, q0, p.Sq);
  cp_async_wait_all();
  __syncthreads();
  // This warp's rows: r0 + g and r0 + g + 8.
  const int r0 = warp * 16;
  uint32_t qa[D / 16][4], da[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    ld_a<D>(sQ, r0, kk * 16, qa[kk]);
    ld_a<D>(sO, r0, kk * 16, da[kk]);
  }
  float lse2[2], dl[2];
  int rowi[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    rowi[hf] = q0 + r0 + g + 8 * hf;
    const bool in = rowi[hf] < p.Sq;
    const float l = in ? p.lse[(size_t)bh * p.Sq + rowi[hf]] : -INFINITY;
    lse2[hf] = l * kLog2e;  // -inf: a row with no visible key, P = 0
    dl[hf] = in ? p.delta[(size_t)bh * p.Sq + rowi[hf]] : 0.f;
  }
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  // Key tiles this query tile sees.
  int kt_lo = 0, kt_hi = (p.Sk + kRows - 1) / kRows;
  if (p.causal) {
    long long last = (long long)q0 + kRows - 1 + p.Sk - p.Sq;
    if (last > p.Sk - 1) last = p.Sk - 1;
    kt_hi = last < 0 ? 0 : (int)(last / kRows) + 1;
    if (p.window > 0) {
      const long long first = (long long)q0 + p.Sk - p.Sq - p.window + 1;
      kt_lo = first <= 0 ? 0 : (int)(first / kRows);
    }
  }
  auto load_kv = [&](int kt, int bf) {
    const uint32_t dst = sKV + (uint32_t)bf * 2u * kTileBytes;
    load_tile<D>(dst, kb, kt * kRows, p.Sk);
    load_tile<D>(dst + kTileBytes, vb, kt * kRows, p.Sk);
    cp_async_commit();
  };
  if (kt_lo < kt_hi) load_kv(kt_lo, 0);
  int bf = 0;
  for (int kt = kt_lo; kt < kt_hi; ++kt, bf ^= 1) {
    const int k0 = kt * kRows;
    if (kt + 1 < kt_hi) {
      load_kv(kt + 1, bf ^ 1);
      cp_async_wait_group<1>();  // this tile's group has landed; the next one may still be in flight
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    const uint32_t sK = sKV + (uint32_t)bf * 2u * kTileBytes, sV = sK + kTileBytes;
    float s[8][4], dp[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {  // pairs of 8-key n-tiles
        uint32_t bk[4], bv[4];
        ld_b_nk<D>(sK, n2 * 16, kk * 16, bk);
        ld_b_nk<D>(sV, n2 * 16, kk * 16, bv);
        mma16816(s[2 * n2], qa[kk], bk[0], bk[1]);
        mma16816(s[2 * n2 + 1], qa[kk], bk[2], bk[3]);
        mma16816(dp[2 * n2], da[kk], bv[0], bv[1]);
        mma16816(dp[2 * n2 + 1], da[kk], bv[2], bv[3]);
      }
    // dS = P * (dP - Delta), P recomputed from the forward's LSE; as bf16 A fragments (k = keys).
    uint32_t dsa[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hf = e >> 1;
        const int j = k0 + n * 8 + 2 * t4 + (e & 1);
        float pr = 0.f;
        if (lse2[hf] != -INFINITY && visible(p, rowi[hf], j)) pr = fast_exp2(s[n][e] * p.scale_log2 - lse2[hf]);
        ds[e] = pr * (dp[n][e] - dl[hf]);
      }
      dsa[n >> 1][(n & 1) * 2 + 0] = pack_rn(ds[0], ds[1]);
      dsa[n >> 1][(n & 1) * 2 + 1] = pack_rn(ds[2], ds[3]);
    }
    // A fragment order: (row g, k 0-7), (row g+8, k 0-7), (row g, k 8-15), (row g+8, k 8-15).
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a[4] = {dsa[kk][0], dsa[kk][1], dsa[kk][2], dsa[kk][3]};
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t bk[4];
        ld_b_kn<D>(sK, n2 * 16, kk * 16, bk);
        mma16816(acc[2 * n2], a, bk[0], bk[1]);
        mma16816(acc[2 * n2 + 1], a, bk[2], bk[3]);
      }
    }
    __syncthreads();  // this buffer is no longer read: the prefetch two tiles on reuses it
  }
  // dQ = scale * dS K, rounded to bf16.
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (rowi[hf] >= p.Sq) continue;
    __nv_bfloat16* dst = p.dq + ((size_t)bh * p.Sq + rowi[hf]) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * t4) =
          pack_rn(acc[n][2 * hf] * p.scale, acc[n][2 * hf + 1] * p.scale);
  }
}

// dK and dV of one 64-key tile of one KV head, summed over the group's query heads.
template <int D>
__global__ void __launch_bounds__(kThreads) dkdv_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kTileBytes = kRows * D * 2;
  // K, V, then two buffers of (Q, dO) and of the rows' LSE and Delta: the next query tile loads
  // while this one is used.
  const uint32_t sK = smem_u32(smem), sV = sK + kTileBytes, sQO = sV + kTileBytes;
  float* s_lse = reinterpret_cast<float*>(smem + 6 * kTileBytes);  // [2][64] LSE (natural log)
  float* s_dl = s_lse + 2 * kRows;                                 // [2][64] Delta
  const int kt = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int grp = p.Hq / p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int k0 = kt * kRows;
  const int r0 = warp * 16;  // this warp's keys: k0 + r0 + g (+ 8)
  const size_t kvoff = ((size_t)b * p.Hkv + kvh) * p.Sk * D;
  load_tile<D>(sK, p.k + kvoff, k0, p.Sk);  // committed with the first query tile below
  load_tile<D>(sV, p.v + kvoff, k0, p.Sk);

  // Query tiles whose rows see some key of this tile.
  const int nq = (p.Sq + kRows - 1) / kRows;
  int qt_lo = 0, qt_hi = nq;
  if (p.causal) {
    const long long lo = (long long)k0 - ((long long)p.Sk - p.Sq);
    qt_lo = lo <= 0 ? 0 : (int)min((long long)nq, lo / kRows);
    if (p.window > 0) {
      const long long hi = (long long)k0 + kRows - 2 - ((long long)p.Sk - p.Sq) + p.window;
      qt_hi = hi < 0 ? 0 : (int)min((long long)nq, hi / kRows + 1);
    }
  }
  float acck[D / 8][4], accv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acck[n][e] = accv[n][e] = 0.f;

  // Work list: the group's query heads times the query tiles, flattened.
  const int nqt = qt_hi > qt_lo ? qt_hi - qt_lo : 0;
  const int n_it = grp * nqt;
  auto issue = [&](int it2, int bf2) {
    const int hh = it2 / nqt, qt = qt_lo + (it2 - hh * nqt);
    const int bh = b * p.Hq + kvh * grp + hh;
    const int q0 = qt * kRows;
    const uint32_t dst = sQO + (uint32_t)bf2 * 2u * kTileBytes;
    load_tile<D>(dst, p.q + (size_t)bh * p.Sq * D, q0, p.Sq);
    load_tile<D>(dst + kTileBytes, p.dout + (size_t)bh * p.Sq * D, q0, p.Sq);
    if (threadIdx.x < kRows) {
      // Rows past Sq read as 0; visible() gives them P = 0.
      const int i = q0 + threadIdx.x;
      const bool in = i < p.Sq;
      const size_t at = (size_t)bh * p.Sq + (in ? i : 0);
      cp_async4(smem_u32(s_lse + bf2 * kRows + threadIdx.x), p.lse + at, in);
      cp_async4(smem_u32(s_dl + bf2 * kRows + threadIdx.x), p.delta + at, in);
    }
    cp_async_commit();
  };
  if (n_it > 0) issue(0, 0);
  int bf = 0;
  for (int it2 = 0; it2 < n_it; ++it2, bf ^= 1) {
    {
      const int hh = it2 / nqt, qt = qt_lo + (it2 - hh * nqt);
      const int q0 = qt * kRows;
      if (it2 + 1 < n_it) {
        issue(it2 + 1, bf ^ 1);
        cp_async_wait_group<1>();  // this tile's group (and K, V) has landed
      } else {
        cp_async_wait_group<0>();
      }
      __syncthreads();
      const uint32_t sQ = sQO + (uint32_t)bf * 2u * kTileBytes, sO = sQ + kTileBytes;
      const float* lse_b = s_lse + bf * kRows;
      const float* dl_b = s_dl + bf * kRows;
      // S^T (keys x queries) and dP^T = V dO^T for this warp's 16 keys.
      float st[8][4], dpt[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t ka[4], va[4];
        ld_a<D>(sK, r0, kk * 16, ka);
        ld_a<D>(sV, r0, kk * 16, va);
#pragma unroll
        for (int n2 = 0; n2 < 4; ++n2) {
          uint32_t bq[4], bo[4];
          ld_b_nk<D>(sQ, n2 * 16, kk * 16, bq);
          ld_b_nk<D>(sO, n2 * 16, kk * 16, bo);
          mma16816(st[2 * n2], ka, bq[0], bq[1]);
          mma16816(st[2 * n2 + 1], ka, bq[2], bq[3]);
          mma16816(dpt[2 * n2], va, bo[0], bo[1]);
          mma16816(dpt[2 * n2 + 1], va, bo[2], bo[3]);
        }
      }
      // P^T and dS^T as bf16 A fragments (k = queries).
      uint32_t pa[4][4], dsa[4][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        float pv[4], dv4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = k0 + r0 + g + 8 * (e >> 1);
          const int qc = n * 8 + 2 * t4 + (e & 1);
          const float l2 = lse_b[qc] * kLog2e;  // -inf: a row with no visible key
          float pr = 0.f;
          if (l2 != -INFINITY && visible(p, q0 + qc, j)) pr = fast_exp2(st[n][e] * p.scale_log2 - l2);
          pv[e] = pr;
          dv4[e] = pr * (dpt[n][e] - dl_b[qc]);
        }
        pa[n >> 1][(n & 1) * 2 + 0] = pack_rn(pv[0], pv[1]);
        pa[n >> 1][(n & 1) * 2 + 1] = pack_rn(pv[2], pv[3]);
        dsa[n >> 1][(n & 1) * 2 + 0] = pack_rn(dv4[0], dv4[1]);
        dsa[n >> 1][(n & 1) * 2 + 1] = pack_rn(dv4[2], dv4[3]);
      }
      // dV += P^T dO, dK += dS^T Q (scale applied at the end).
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {
          uint32_t bo[4], bq[4];
          ld_b_kn<D>(sO, n2 * 16, kk * 16, bo);
          ld_b_kn<D>(sQ, n2 * 16, kk * 16, bq);
          mma16816(accv[2 * n2], pa[kk], bo[0], bo[1]);
          mma16816(accv[2 * n2 + 1], pa[kk], bo[2], bo[3]);
          mma16816(acck[2 * n2], dsa[kk], bq[0], bq[1]);
          mma16816(acck[2 * n2 + 1], dsa[kk], bq[2], bq[3]);
        }
    }
    __syncthreads();  // this buffer is no longer read: the prefetch two tiles on reuses it
  }
  cp_async_wait_all();  // nothing may be in flight when the CTA exits (empty query ranges)
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int j = k0 + r0 + g + 8 * hf;
    if (j >= p.Sk) continue;
    __nv_bfloat16* dk = p.dk + kvoff + (size_t)j * D;
    __nv_bfloat16* dv = p.dv + kvoff + (size_t)j * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      *reinterpret_cast<uint32_t*>(dk + n * 8 + 2 * t4) = pack_rn(acck[n][2 * hf] * p.scale, acck[n][2 * hf + 1] * p.scale);
      *reinterpret_cast<uint32_t*>(dv + n * 8 + 2 * t4) = pack_rn(accv[n][2 * hf], accv[n][2 * hf + 1]);
    }
  }
}

}  // namespace bwd
}  // namespace attn
