// Prefill forward on CUDA cores in fp32: the accuracy path for float32 inputs.
//
// One warp owns one query row and walks the visible keys 32 at a time (one key per
// lane).  Per block of 32 keys it takes the block max and the block sum of the
// exponentials with warp shuffles and merges them into the running max / denominator
// exactly like the online softmax of CSDN «注意力变体深挖» section 6.2, rescaling the
// running output when the max grows.  Each lane owns D/32 output columns.  fp32
// arithmetic throughout, accurate exp2f.
#pragma once

#include "common.cuh"

namespace attn {
namespace simt {

constexpr int kRowsPerBlock = 4;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
    fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    T* __restrict__ o, float* __restrict__ lse, int Hq, int Hkv, int Sq, int Sk,
                    float scale_log2, int causal, int window) {
  __shared__ float qs[kRowsPerBlock][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRowsPerBlock + warp;
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh - b * Hq;
  const int kvh = h / (Hq / Hkv);
  if (row >= Sq) return;

  const T* qrow = q + ((size_t)bh * Sq + row) * D;
  for (int d = lane; d < D; d += 32) qs[warp][d] = to_f(qrow[d]);
  __syncwarp();

  const T* kb = k + ((size_t)b * Hkv + kvh) * (size_t)Sk * D;
  const T* vb = v + ((size_t)b * Hkv + kvh) * (size_t)Sk * D;
  long long last = causal ? (long long)row + Sk - Sq : (long long)Sk - 1;
  if (last > Sk - 1) last = Sk - 1;
  const int nkeys = last < 0 ? 0 : (int)last + 1;
  // Sliding window (causal only): keys last - window + 1 .. last.
  const int kfirst = (window > 0 && nkeys > window) ? nkeys - window : 0;

  float m = -INFINITY, l = 0.f;
  float acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;

  for (int k0 = kfirst; k0 < nkeys; k0 += 32) {
    const int key = k0 + lane;
    float x = -INFINITY;
    if (key < nkeys) {
      const T* kr = kb + (size_t)key * D;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) dot = fmaf(qs[warp][d], to_f(kr[d]), dot);
      x = dot * scale_log2;
    }
    const float m_new = fmaxf(m, warp_max(x));
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    const float pk = (key < nkeys) ? exp2f(x - m_new) : 0.f;
    l = l * alpha + warp_sum(pk);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] *= alpha;
    const int cnt = min(32, nkeys - k0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, pk, jj);
      const T* vr = vb + (size_t)(k0 + jj) * D;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(pj, to_f(vr[lane + 32 * e]), acc[e]);
    }
    m = m_new;
  }

  T* orow = o + ((size_t)bh * Sq + row) * D;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) orow[lane + 32 * e] = from_f<T>(acc[e] * inv);
  if (lse != nullptr && lane == 0)
    lse[(size_t)bh * Sq + row] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

}  // namespace simt
}  // namespace attn
