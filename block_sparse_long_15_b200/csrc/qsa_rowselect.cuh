// Per-row scoring and selection pieces: the fp32 score of one candidate block (the
// decode selection kernel and the few-row scoring kernel), and the exact per-row
// top-k by one warp (the tensor-core prefill scoring and the select-from-scores
// kernel), so that every path that shares them takes the same ids from the same keys.
// Definitions: Hugging Face Transformers model doc "Qwen4-Exp", intro paragraph on
// QSA (multiple query heads score compressed key blocks, the most relevant blocks
// are selected) and Qwen4ExpTextConfig indexer_budget.
#pragma once

#include <stdint.h>

namespace qsa {

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

constexpr int kScoreMaxHi = 8;  // indexer heads scored together per k̄ piece

// s_j = sum_h max(0, qi[h] . kbar_j) in fp32 for one candidate, computed by one thread:
// qi_s [Hi][di] (fp32, any memory), kr the candidate's k̄ row (16-byte aligned,
// di % 4 == 0). Dots run in dim order, four at a time from float4 pairs; heads are
// summed in head order.
__device__ __forceinline__ float block_score_fp32(const float *qi_s, int Hi, int di, const float4 *kr) {
  float s = 0.f;
  if (di <= 64) {
    // the candidate's k̄ row in registers; the query heads, up to kScoreMaxHi at a
    // time, reuse it
    float4 kv[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) kv[c] = (c < di / 4) ? kr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int h0 = 0; h0 < Hi; h0 += kScoreMaxHi) {
      float dot[kScoreMaxHi];
#pragma unroll
      for (int h = 0; h < kScoreMaxHi; ++h) dot[h] = 0.f;
#pragma unroll
      for (int h = 0; h < kScoreMaxHi; ++h) {
        if (h0 + h >= Hi) break;
        const float4 *qh = (const float4 *)(qi_s + (h0 + h) * di);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (c >= di / 4) break;
          const float4 a = qh[c];
          dot[h] = fmaf(a.x, kv[c].x, dot[h]);
          dot[h] = fmaf(a.y, kv[c].y, dot[h]);
          dot[h] = fmaf(a.z, kv[c].z, dot[h]);
          dot[h] = fmaf(a.w, kv[c].w, dot[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < kScoreMaxHi; ++h)
        if (h0 + h < Hi) s += dot[h] > 0.f ? dot[h] : 0.f;
    }
  } else {
    // wider rows in 64-float pieces whose 16 loads are all in flight together
    for (int h0 = 0; h0 < Hi; h0 += kScoreMaxHi) {
      float dot[kScoreMaxHi];
#pragma unroll
      for (int h = 0; h < kScoreMaxHi; ++h) dot[h] = 0.f;
      for (int c0 = 0; c0 < di / 4; c0 += 16) {
        float4 kv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) kv[c] = (c0 + c < di / 4) ? kr[c0 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int h = 0; h < kScoreMaxHi; ++h) {
          if (h0 + h >= Hi) break;
          const float4 *qh = (const float4 *)(qi_s + (h0 + h) * di) + c0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            if (c0 + c >= di / 4) break;
            const float4 a = qh[c];
            dot[h] = fmaf(a.x, kv[c].x, dot[h]);
            dot[h] = fmaf(a.y, kv[c].y, dot[h]);
            dot[h] = fmaf(a.z, kv[c].z, dot[h]);
            dot[h] = fmaf(a.w, kv[c].w, dot[h]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < kScoreMaxHi; ++h)
        if (h0 + h < Hi) s += dot[h] > 0.f ? dot[h] : 0.f;
    }
  }
  return s;
}

// Exact top-k of one row by a warp: writes out[0 .. k) with the ids of the k largest
// keys in ascending id order, ties to the lower id, -1 padded; n < 0 marks a padding
// row (all -1) and n <= k keeps every id. key(j) returns the 32-bit key of id j whose
// unsigned order is the score order (fp32 bit patterns of scores >= +0, or the
// order-preserving map of any finite fp32). wh: 256 ints of shared memory for the warp.
//
// The k-th largest key is found by 8-bit radix passes from the highest bit in which
// the row's keys differ (the bits above it are common to all keys, so no pass piles
// every key into one bin); once the keys still matching the prefix are at most 32,
// they are gathered one per lane and sorted across the warp (bitonic, descending),
// which settles the k-th key and how many ties of it to keep. Then keys above it,
// and the lowest-id keys equal to it, are written in id order.
template <typename KeyFn>
__device__ __forceinline__ void warp_select_row(KeyFn key_of, int n, int k, int32_t *out, int *wh) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  if (n <= k) {  // padding row (n = -1), or every complete block kept
    for (int i = lane; i < k; i += 32) out[i] = (i < n) ? i : -1;
    return;
  }
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j = lane; j < n; j += 32) {
    const uint32_t key = key_of(j);
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const uint32_t diff = kmin ^ kmax;
  const int top = diff ? 31 - __clz(diff) : -1;
  uint32_t pmask = top >= 31 ? 0u : (0xffffffffu << (top + 1));
  uint32_t prefix = kmax & pmask;
  int remaining = k;
  auto settle = [&]() {
    __syncwarp();
    int base = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < n ? key_of(j) : 0u;
      const bool cand = j < n && (key & pmask) == prefix;
      const unsigned m = __ballot_sync(0xffffffffu, cand);
      if (cand) wh[base + __popc(m & lt)] = (int)key;
      base += __popc(m);
    }
    __syncwarp();
    uint32_t v = lane < base ? (uint32_t)wh[lane] : 0u;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
        // descending runs where (lane & size) == 0, ascending otherwise; the last
        // merge (size 32) leaves the whole warp descending
        const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0 || size == 32);
        v = keep_max ? max(v, o) : min(v, o);
      }
    }
    const uint32_t val = __shfl_sync(0xffffffffu, v, remaining - 1);
    remaining -= __popc(__ballot_sync(0xffffffffu, lane < base && v > val));
    prefix = val;
    pmask = 0xffffffffu;
    __syncwarp();
  };
  if (top >= 0 && n <= 32) settle();
  for (int hi_bit = top; hi_bit >= 0 && pmask != 0xffffffffu; hi_bit -= 8) {
    const int shift = hi_bit >= 7 ? hi_bit - 7 : 0;
    const uint32_t dmask = (2u << (hi_bit - shift)) - 1u;
    for (int i = lane; i < 256; i += 32) wh[i] = 0;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t key = key_of(j);
      if ((key & pmask) == prefix) atomicAdd(&wh[(key >> shift) & dmask], 1);
    }
    __syncwarp();
    // lane L owns digits 255-8L .. 248-8L (descending)
    int c[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = wh[255 - 8 * lane - q];
      tot += c[q];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - tot;
    int digit = 0, above = 0, cnt = 0;
    const bool mine = excl < remaining && incl >= remaining;
    if (mine) {
      above = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (above + c[q] >= remaining) {
          digit = 255 - 8 * lane - q;
          cnt = c[q];
          break;
        }
        above += c[q];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    cnt = __shfl_sync(0xffffffffu, cnt, src);
    prefix |= (uint32_t)digit << shift;
    pmask |= dmask << shift;
    remaining -= above;
    __syncwarp();
    if (shift > 0 && cnt <= 32) settle();
  }
  int base_i = 0, tie_base = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < n ? key_of(j) : 0u;
    const bool gt = j < n && key > prefix;
    const bool eq = j < n && key == prefix;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && tie_base + __popc(eq_mask & lt) < remaining);
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) out[base_i + __popc(take_mask & lt)] = j;
    base_i += __popc(take_mask);
    tie_base += __popc(eq_mask);
  }
}

}  // namespace qsa
