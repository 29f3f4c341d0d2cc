// Single-token decode over a contiguous or paged KV cache: split-KV partials plus an
// LSE-weighted combine pass.
//
// The KV cache is read once from HBM, which bounds the step (CSDN «注意力变体深挖» §一
// and §七: decoding is memory-bound on KV reads).  Design for sm_100a:
//
//  * grid (split, kv head x head-subgroup, batch).  A CTA reads the K/V of one KV head
//    for one chunk of tokens and serves the G query heads of its subgroup from that
//    single read (GQA: the group's heads share each K/V row).
//  * warp 4 streams the chunk through a 3-stage ring of 64-token stages with cp.async.bulk:
//    every run of tokens that is contiguous in the cache (one page of a paged pool, or
//    the whole stage in a dense cache) is one bulk copy.  The page ids come from the
//    block table (gocoding §5), prefetched 32 pages ahead into the producer's lanes.
//  * warps 0-3 compute.  Eight lanes cover one token row (D/8 elements each, as
//    interleaved 16-byte slices so that reads are conflict-free); per step
//    each lane forms the partial dot products of 8 (token, head) pairs with packed fp32
//    FMAs and a 3-level reduce-scatter across the 8 lanes leaves one complete score per
//    lane (fewer lanes per row means less shuffle work per score).  Online softmax per
//    head (log2 domain, ex2), then the value rows are accumulated as fp32 pairs.
//  * each split writes its normalised partial output and its LSE; the combine kernel
//    merges the splits of a (sequence, head) with weights exp(lse_s - LSE), the same
//    two-way merge as the pages' online softmax, applied across splits.
#pragma once

#include "common.cuh"

namespace attn {
namespace dec {

constexpr int kStageTokens = 64;
constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxSplits = 128;  // the plan never splits a sequence into more chunks

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const int* seqlens;
  const int* block_table;  // nullptr: contiguous cache
  int block_size, max_blocks, num_blocks, max_seqlen;
  int B, Hq, Hkv;
  int chunk, max_splits, nsub;
  float scale_log2;
  float* ws_o;    // [B, Hq, max_splits, D]
  float* ws_lse;  // [B, Hq, max_splits]
  unsigned int* ws_err;
  int* ws_cnt;    // [B, Hkv * nsub] splits finished; the last one merges and resets it
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
struct Layout {
  static constexpr int kRow = D * 2;
  static constexpr int kStageBytes = kStageTokens * kRow;  // K (or V) bytes of one stage
  static constexpr int kK = 0;
  static constexpr int kV = kStages * kStageBytes;
  static constexpr int kBar = 2 * kStages * kStageBytes;
  static constexpr int kMisc = kBar + 2 * kStages * 8;
  static constexpr int kBytes = kMisc + 16;
};

__device__ __forceinline__ void flag_error(const Params& p, unsigned int f) {
  atomicOr(p.ws_err, f);
  raise_status(f);
}

// Valid length of sequence b after the device-side bound checks.
__device__ __forceinline__ int checked_len(const Params& p, int b, bool report) {
  int len = p.seqlens[b];
  const long long cap = p.block_table ? (long long)p.max_blocks * p.block_size : (long long)p.block_size;
  long long lim = p.max_seqlen < cap ? p.max_seqlen : cap;
  if (len < 0 || len > lim) {
    if (report) flag_error(p, ATTN_DEV_BAD_SEQLEN);
    len = len < 0 ? 0 : (int)lim;
  }
  return len;
}

__device__ __forceinline__ void unpack8(uint4 w, float (&f)[8]) {
  f[0] = bf16lo(w.x);
  f[1] = bf16hi(w.x);
  f[2] = bf16lo(w.y);
  f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z);
  f[5] = bf16hi(w.z);
  f[6] = bf16lo(w.w);
  f[7] = bf16hi(w.w);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Recursive-halving reduce-scatter over the LPT lanes of a group: on return lane j of
// the group holds in vals[0] the group-wide sum of the original vals[j].
template <int LPT>
__device__ __forceinline__ float reduce_scatter(float (&vals)[LPT], int j) {
#pragma unroll
  for (int off = LPT / 2, cnt = LPT / 2; off > 0; off >>= 1, cnt >>= 1) {
    const bool upper = (j & off) != 0;
#pragma unroll
    for (int i = 0; i < cnt; ++i) {
      const float send = upper ? vals[i] : vals[i + cnt];
      const float keep = upper ? vals[i + cnt] : vals[i];
      vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return vals[0];
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(const Params p) {
  // Lanes per token row: 8, except D=128 with 8 heads per CTA, where 16 lanes halve the
  // per-lane query and accumulator registers.
  constexpr int LPT = (D == 128 && G == 8) ? 16 : 8;
  constexpr int EPL = D / LPT;     // elements of a row per lane (16 at D=128, 8 at D=64)
  constexpr int WPL = EPL / 2;     // 32-bit words (bf16 pairs) per lane per row
  constexpr int TOK = LPT / G;     // tokens per lane group per step
  constexpr int GPW = 32 / LPT;    // lane groups per warp
  constexpr int TPW = GPW * TOK;   // tokens per warp step (= 32 / G)
  constexpr int UNITS = kStageTokens / TPW;  // warp steps per stage (= G)
  static_assert(G <= LPT && TOK * G == LPT, "heads per CTA must divide the lanes per token");
  static_assert(EPL % 8 == 0, "each lane reads whole 16-byte slices");
  constexpr bool kJoint = true;
  using L = Layout<D>;

  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  auto full_bar = [&](int s) -> uint32_t { return sbase + L::kBar + 8u * s; };
  auto empty_bar = [&](int s) -> uint32_t { return sbase + L::kBar + 8u * (kStages + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);

  const int b = blockIdx.z;
  const int split = blockIdx.x;
  const int len = checked_len(p, b, split == 0 && blockIdx.y == 0 && threadIdx.x == 0);
  const int nsplit = (len + p.chunk - 1) / p.chunk;
  const int kvh0 = blockIdx.y / p.nsub;
  const int hbase = kvh0 * (p.Hq / p.Hkv) + (blockIdx.y - kvh0 * p.nsub) * G;
  if (nsplit == 0 && split == 0) {  // empty sequence: O = 0, LSE = -inf
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
      const int hh = idx / D, d = idx - hh * D;
      p.o[((size_t)b * p.Hq + hbase + hh) * D + d] = __float2bfloat16_rn(0.f);
      if (p.lse != nullptr && d == 0) p.lse[(size_t)b * p.Hq + hbase + hh] = -INFINITY;
    }
  }
  if (split >= nsplit) return;
  const int t0 = split * p.chunk;
  const int t1 = min(len, t0 + p.chunk);
  const int niters = (t1 - t0 + kStageTokens - 1) / kStageTokens;
  const int kvh = blockIdx.y / p.nsub;
  const int sub = blockIdx.y - kvh * p.nsub;
  const int g = p.Hq / p.Hkv;
  const int h0 = kvh * g + sub * G;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ bulk-copy producer
    const int bs = p.block_size;
    const bool paged = p.block_table != nullptr;
    const int* table = paged ? p.block_table + (size_t)b * p.max_blocks : nullptr;
    auto load_id = [&](int page) -> int {
      return (paged && page < p.max_blocks) ? __ldg(table + page) : -1;
    };
    int cur_first = t0 / bs;
    int nxt_first = cur_first + 32;
    int cur_id = load_id(cur_first + lane);
    int nxt_id = load_id(nxt_first + lane);
    int last_fill[kStages];
    for (int s = 0; s < kStages; ++s) last_fill[s] = -1;
    for (int it = 0; it < niters; ++it) {
      const int s = it % kStages;
      const int f = it / kStages;
      if (f > 0) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(empty_bar(s), (f - 1) & 1, abort_flag));
        if (!ok) break;
      }
      const int a = t0 + it * kStageTokens;
      const int e = min(t1, a + kStageTokens);
      const uint32_t dk = sbase + L::kK + s * L::kStageBytes;
      const uint32_t dv = sbase + L::kV + s * L::kStageBytes;
      for (int tok = a; tok < e;) {
        const int page = tok / bs;
        const int slot = tok - page * bs;
        const int run = min(bs - slot, e - tok);
        while (page >= cur_first + 32) {
          cur_id = nxt_id;
          cur_first = nxt_first;
          nxt_first += 32;
          nxt_id = load_id(nxt_first + lane);
        }
        const int blk = paged ? __shfl_sync(0xffffffffu, cur_id, page - cur_first) : b;
        if (lane == 0) {
          if (blk < 0 || blk >= p.num_blocks) {
            flag_error(p, ATTN_DEV_BAD_BLOCK);
          } else {
            const size_t off = (((size_t)blk * p.Hkv + kvh) * (size_t)bs + slot) * D;
            const uint32_t bytes = (uint32_t)run * L::kRow;
            const uint32_t dst = (uint32_t)(tok - a) * L::kRow;
            mbar_expect_tx(full_bar(s), 2u * bytes);
            bulk_load(dk + dst, p.kc + off, bytes, full_bar(s));
            bulk_load(dv + dst, p.vc + off, bytes, full_bar(s));
          }
        }
        tok += run;
      }
      if (lane == 0) mbar_arrive(full_bar(s));
      last_fill[s] = f;
    }
    if (*abort_flag && lane == 0) {
      // Consumers gave up: let copies already in flight land before the CTA exits.
      int never = 0;
      for (int s = 0; s < kStages; ++s)
        if (last_fill[s] >= 0) mbar_wait(full_bar(s), last_fill[s] & 1, &never, 100000000ull);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Lane j of lane group gi owns the 16-byte slices j, j + 8, ... (8 elements each) of every
  // token row, so the 8 lanes of a group read 128 contiguous bytes per access (no bank
  // conflicts); a group covers one row, so a score is complete after a 3-level
  // reduce-scatter.
  const int gi = lane / LPT;
  const int j = lane - gi * LPT;
  uint64_t q2[G][WPL];  // this lane's query elements per head, as fp32 pairs
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + h0 + hh) * D) + j;
#pragma unroll
    for (int v4 = 0; v4 < EPL / 8; ++v4) {
      const uint4 w = __ldg(src + LPT * v4);
      q2[hh][4 * v4 + 0] = f2pack(bf16lo(w.x), bf16hi(w.x));
      q2[hh][4 * v4 + 1] = f2pack(bf16lo(w.y), bf16hi(w.y));
      q2[hh][4 * v4 + 2] = f2pack(bf16lo(w.z), bf16hi(w.z));
      q2[hh][4 * v4 + 3] = f2pack(bf16lo(w.w), bf16hi(w.w));
    }
  }
  const float c = p.scale_log2;
  float m_own = -INFINITY, l_own = 0.f;
  uint64_t acc[G][WPL];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int e = 0; e < WPL; ++e) acc[hh][e] = 0ull;

  bool ok = true;
  for (int it = 0; it < niters; ++it) {
    const int s = it % kStages;
    ok = __all_sync(0xffffffffu, mbar_wait(full_bar(s), (it / kStages) & 1, abort_flag));
    if (!ok) break;
    const int nv = min(kStageTokens, t1 - (t0 + it * kStageTokens));
    const uint32_t sk = sbase + L::kK + s * L::kStageBytes;
    const uint32_t sv = sbase + L::kV + s * L::kStageBytes;
    // Each warp takes two units of the stage at a time (u and u + 4 warps): their dot
    // products and reductions are independent, which gives the warp twice the ILP; they
    // share one max update and one rescale.  A second unit past the stage is empty.
    for (int u = warp; u < UNITS; u += (kJoint ? 2 : 1) * kConsumerWarps) {
      const int u1 = u + kConsumerWarps;
      const bool has1 = kJoint && u1 < UNITS;
      const int tb0 = u * TPW + gi * TOK;                   // first token of this lane group
      const int tb1 = (has1 ? u1 : u) * TPW + gi * TOK;
      float vals0[LPT], vals1[LPT];
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          uint64_t k2[WPL];
#pragma unroll
          for (int v4 = 0; v4 < EPL / 8; ++v4) {
            const uint4 w = lds128(sk + (uint32_t)((x ? tb1 : tb0) + tt) * L::kRow + 16u * (j + LPT * v4));
            k2[4 * v4 + 0] = f2pack(bf16lo(w.x), bf16hi(w.x));
            k2[4 * v4 + 1] = f2pack(bf16lo(w.y), bf16hi(w.y));
            k2[4 * v4 + 2] = f2pack(bf16lo(w.z), bf16hi(w.z));
            k2[4 * v4 + 3] = f2pack(bf16lo(w.w), bf16hi(w.w));
          }
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            uint64_t d2 = fmul2(q2[hh][0], k2[0]);
#pragma unroll
            for (int e = 1; e < WPL; ++e) d2 = ffma2(q2[hh][e], k2[e], d2);
            float lo, hi;
            f2unpack(d2, lo, hi);
            if (x) vals1[tt * G + hh] = lo + hi;
            else vals0[tt * G + hh] = lo + hi;
          }
        }
      }
      const float score0 = reduce_scatter<LPT>(vals0, j);
      const float score1 = reduce_scatter<LPT>(vals1, j);
      const float x0 = (tb0 + j / G < nv) ? score0 * c : -INFINITY;
      const float x1 = (has1 && tb1 + j / G < nv) ? score1 * c : -INFINITY;
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int o = G; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_own, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_own - m_new);
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      const float pr0 = fast_exp2(x0 - mu), pr1 = fast_exp2(x1 - mu);
      l_own = l_own * alpha + (pr0 + pr1);
      m_own = m_new;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float ah = __shfl_sync(0xffffffffu, alpha, hh);
          const uint64_t a2 = f2pack(ah, ah);
#pragma unroll
          for (int e = 0; e < WPL; ++e) acc[hh][e] = fmul2(acc[hh][e], a2);
        }
      }
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          uint64_t v2[WPL];
          const int tok = (x ? tb1 : tb0) + tt;
#pragma unroll
          for (int v4 = 0; v4 < EPL / 8; ++v4) {
            const uint4 w = lds128(sv + (uint32_t)tok * L::kRow + 16u * (j + LPT * v4));
            v2[4 * v4 + 0] = f2pack(bf16lo(w.x), bf16hi(w.x));
            v2[4 * v4 + 1] = f2pack(bf16lo(w.y), bf16hi(w.y));
            v2[4 * v4 + 2] = f2pack(bf16lo(w.z), bf16hi(w.z));
            v2[4 * v4 + 3] = f2pack(bf16lo(w.w), bf16hi(w.w));
          }
          const bool tv = (x == 0 || has1) && tok < nv;
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float ph = __shfl_sync(0xffffffffu, x ? pr1 : pr0, gi * LPT + tt * G + hh);
            if (tv) {
              const uint64_t p2 = f2pack(ph, ph);
#pragma unroll
              for (int e = 0; e < WPL; ++e) acc[hh][e] = ffma2(p2, v2[e], acc[hh][e]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }

  // Merge lane groups of this warp: per head, acc summed over groups, l over all lanes.
  float accf[G][EPL];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int e = 0; e < WPL; ++e) f2unpack(acc[hh][e], accf[hh][2 * e], accf[hh][2 * e + 1]);
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1)
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < EPL; ++e) accf[hh][e] += __shfl_xor_sync(0xffffffffu, accf[hh][e], o);
  float l_sum = l_own;
#pragma unroll
  for (int o = G; o < 32; o <<= 1) l_sum += __shfl_xor_sync(0xffffffffu, l_sum, o);

  // Merge the consumer warps through shared memory (the ring is idle now).
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  float* m_s = reinterpret_cast<float*>(smem);                 // [warps][G]
  float* l_s = m_s + kConsumerWarps * G;                       // [warps][G]
  float* a_s = l_s + kConsumerWarps * G;                       // [warps][G][D]
  // Outside the ring: in-flight copies of an aborted call must not touch these.
  volatile int* ok_s = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* last_s = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  // Any consumer that gave up set *abort_flag; snapshot it between two barriers so that
  // every consumer warp takes the same branch below (named barriers never time out).
  if (threadIdx.x == 0) *ok_s = (*abort_flag == 0);
  if (ok) {
    if (lane < G) {
      m_s[warp * G + lane] = m_own;  // lane hh holds head hh
      l_s[warp * G + lane] = l_sum;
    }
    if (gi == 0) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < EPL; ++e) a_s[(warp * G + hh) * D + 8 * (j + LPT * (e >> 3)) + (e & 7)] = accf[hh][e];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  if (!*ok_s) return;
  const size_t bh0 = (size_t)b * p.Hq + h0;
  for (int idx = threadIdx.x; idx < G * D; idx += kConsumerWarps * 32) {
    const int hh = idx / D, d = idx - hh * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, m_s[w * G + hh]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float sc = fast_exp2(m_s[w * G + hh] - M);
        Lsum += l_s[w * G + hh] * sc;
        O += a_s[(w * G + hh) * D + d] * sc;
      }
    }
    const float o_val = Lsum > 0.f ? O / Lsum : 0.f;
    const float lse_val = Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
    if (nsplit == 1) {  // the only split: write the result directly
      p.o[(bh0 + hh) * D + d] = __float2bfloat16_rn(o_val);
      if (p.lse != nullptr && d == 0) p.lse[bh0 + hh] = lse_val;
    } else {
      const size_t slot = (bh0 + hh) * p.max_splits + split;
      p.ws_o[slot * D + d] = o_val;
      if (d == 0) p.ws_lse[slot] = lse_val;
    }
  }
  if (nsplit == 1) return;

  // The last split of this (sequence, head group) to finish merges all partials.
  __threadfence();
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  int* cnt = p.ws_cnt + (size_t)b * gridDim.y + blockIdx.y;
  if (threadIdx.x == 0) *last_s = (atomicAdd(cnt, 1) == nsplit - 1);
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  if (!*last_s) return;
  __threadfence();
  // Stage the partial LSEs in shared memory (one independent load per thread), turn them
  // into merge weights exp(lse_s - LSE), then combine the partial outputs.
  float* w_s = reinterpret_cast<float*>(smem);  // [G][max_splits]
  float* lse_f = w_s + G * kMaxSplits;          // [G]
  for (int idx = threadIdx.x; idx < G * nsplit; idx += kConsumerWarps * 32) {
    const int hh = idx / nsplit, sp = idx - hh * nsplit;
    w_s[hh * kMaxSplits + sp] = __ldcg(p.ws_lse + (bh0 + hh) * p.max_splits + sp);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  if (threadIdx.x < G) {
    float* w = w_s + threadIdx.x * kMaxSplits;
    float M = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, w[sp]);
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float Lsum = 0.f;
      for (int sp = 0; sp < nsplit; ++sp) Lsum += expf(w[sp] - M);
      lse = M + logf(Lsum);
    }
    for (int sp = 0; sp < nsplit; ++sp) w[sp] = lse == -INFINITY ? 0.f : expf(w[sp] - lse);
    lse_f[threadIdx.x] = lse;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32));
  for (int idx = threadIdx.x; idx < G * D; idx += kConsumerWarps * 32) {
    const int hh = idx / D, d = idx - hh * D;
    const float* w = w_s + hh * kMaxSplits;
    const float* o_s = p.ws_o + (bh0 + hh) * p.max_splits * D + d;
    float out0 = 0.f, out1 = 0.f, out2 = 0.f, out3 = 0.f;
    int sp = 0;
    for (; sp + 4 <= nsplit; sp += 4) {
      out0 = fmaf(w[sp], __ldcg(o_s + (size_t)sp * D), out0);
      out1 = fmaf(w[sp + 1], __ldcg(o_s + (size_t)(sp + 1) * D), out1);
      out2 = fmaf(w[sp + 2], __ldcg(o_s + (size_t)(sp + 2) * D), out2);
      out3 = fmaf(w[sp + 3], __ldcg(o_s + (size_t)(sp + 3) * D), out3);
    }
    for (; sp < nsplit; ++sp) out0 = fmaf(w[sp], __ldcg(o_s + (size_t)sp * D), out0);
    p.o[(bh0 + hh) * D + d] = __float2bfloat16_rn((out0 + out1) + (out2 + out3));
    if (p.lse != nullptr && d == 0) p.lse[bh0 + hh] = lse_f[hh];
  }
  if (threadIdx.x == 0) *cnt = 0;  // ready for the next call
}

}  // namespace dec
}  // namespace attn
