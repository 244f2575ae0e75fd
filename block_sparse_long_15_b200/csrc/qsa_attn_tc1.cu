// Step 4 on 5th-generation tensor cores (tcgen05) for prefill, one query tile per
// CTA: exact attention over each query's selected blocks plus its trailing block
// (Hugging Face Transformers model doc "Qwen4-Exp", intro paragraph on QSA; GQA per
// Qwen4ExpTextConfig num_key_value_heads; head_dim per the same config, whose
// default is 256).
//
// Work unit: one KV head g of one sequence and T = 128 / G consecutive query
// tokens, held as one 128-row MMA tile whose rows are (token, query head of g)
// pairs. The unit walks the union of its tokens' key sets in ascending 64-key
// chunks (a chunk lies inside one block, so a row sees a chunk whole, up to its
// query position, or not at all):
//   warp 0      TMA producer: K and V chunks (128-byte swizzle) into two 2-deep
//               rings, K released after its QK MMA, V after its PV MMA;
//   warp 1      TMEM owner and MMA issuer (the warp runs the loop, one elected
//               lane issues). S is double-buffered in
//               TMEM: while the softmax works on chunk n, S of chunk n + 1 is
//               already there, and the PV of chunk n is followed by the QK of chunk
//               n + 2 into the buffer that PV has just read;
//   warps 2-9   softmax, 16 rows per warp, whole: warp w reads TMEM lanes
//               32 (w % 4) + 16 s .. + 15 (s one bit of w) with 16x32bx2 accesses,
//               so thread t < 16 holds its row's first 32 keys of the chunk and
//               thread t + 16 the last 32: tcgen05.ld of the 32 logits, the row max by
//               one shuffle, online softmax with a lazily rescaled reference max, P
//               (bf16) over the first 32 columns of the S buffer for the PV MMA (A
//               operand from TMEM); each thread rescales and writes out half of the
//               row's O; epilogue O / l rounded to bf16.
// TMEM: O in columns [0, 256), S buffers at 256 and 320 (512 allocated); shared
// memory about 200 KB, one CTA per SM. Served for head_dim 256 only: head_dim 128
// takes the two-tile kernel (qsa_attn_tc.cu).
// Every wait is bounded; on expiry the kernel records QSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <math.h>
#include <stdio.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // MMA M: (token, head) rows of the tile
constexpr int kCK = 64;      // keys per chunk (MMA N of S = Q K^T, K of O += P V)
constexpr int kNK = 2;       // K ring depth
constexpr int kNV = 2;       // V ring depth
constexpr int kThreads = 320;  // producer, MMA, 4 lane groups x 2 sixteen-row groups
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSelBytes = 8192;  // selection lists of the unit, if they fit

// barrier slots
constexpr int kBarQ = 0;
constexpr int kBarKFull = 1;
constexpr int kBarKEmpty = kBarKFull + kNK;
constexpr int kBarVFull = kBarKEmpty + kNK;
constexpr int kBarVEmpty = kBarVFull + kNV;
constexpr int kBarSFull = kBarVEmpty + kNV;  // [S buffer]
constexpr int kBarPFull = kBarSFull + 2;     // [S buffer], 8 arrivals (one per softmax warp)
constexpr int kBarPVDone = kBarPFull + 2;    // one phase per PV
constexpr int kBarODone = kBarPVDone + 1;    // once, after the last PV
constexpr int kNumBars = kBarODone + 1;

template <int D_>
struct Layout {
  static constexpr uint32_t kQBytes = kRows * D_ * 2;  // D_/64 groups of [128 rows][128 B]
  static constexpr uint32_t kKVBytes = kCK * D_ * 2;   // D_/64 groups of [64 rows][128 B]
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffV = kOffK + kNK * kKVBytes;
  static constexpr uint32_t kOffBar = kOffV + kNV * kKVBytes;
  static constexpr uint32_t kOffMisc = kOffBar + 256;
  static constexpr uint32_t kOffSel = kOffMisc + 64;
  static constexpr uint32_t kOffBitmap = kOffSel + kSelBytes;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(D_ == 256, "one-tile kernel is built for head_dim 256 only");
};

struct Tc1Params {
  Dims D;
  Seqs S;
  const int32_t *sel;
  __nv_bfloat16 *out;
  int *status;
  int T;             // tokens per tile
  int n_units;       // units per (sequence, KV head)
  int bitmap_words;  // capacity of the chunk bitmap
};

// Smallest set bit >= c of bm, or -1.
__device__ __forceinline__ int next_chunk(const uint32_t *bm, int nwords, int c) {
  int w = c >> 5;
  if (w >= nwords) return -1;
  uint32_t bits = bm[w] & (0xffffffffu << (c & 31));
  while (true) {
    if (bits) return (w << 5) + __ffs(bits) - 1;
    if (++w >= nwords) return -1;
    bits = bm[w];
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

// P for one 32-key quarter held in registers (fp32 bits), written back in place
// over sv[0 .. 15] as 16 packed bf16 pairs: p = 2^(s * sl2 - m) for keys below
// `lim`, 0 from there on. Returns the quarter's sum (packed fp32 pairs).
template <bool kAll>
__device__ __forceinline__ float p_quarter(uint32_t (&sv)[32], int lim, uint64_t scale2, uint64_t negm2) {
  uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
  for (int u = 0; u < 32; u += 2) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(sv[u], sv[u + 1]), scale2, negm2), x0, x1);
    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    if (!kAll) {
      p0 = (u < lim) ? p0 : 0.f;
      p1 = (u + 1 < lim) ? p1 : 0.f;
    }
    sv[u >> 1] = pack_bf16x2(p0, p1);
    if ((u >> 1) & 1) acc1 = f2_add(acc1, f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
    else acc0 = f2_add(acc0, f2_pack(__float_as_uint(p0), __float_as_uint(p1)));
  }
  float s0, s1;
  f2_unpack(f2_add(acc0, acc1), s0, s1);
  return s0 + s1;
}

// Max of the first `lim` of 32 fp32 values, in 4 independent chains.
template <bool kAll>
__device__ __forceinline__ float max_quarter(const uint32_t (&sv)[32], int lim) {
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int u = 0; u < 32; u += 8) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int a = u + 2 * e;
      const float xa = (kAll || a < lim) ? __uint_as_float(sv[a]) : -INFINITY;
      const float xb = (kAll || a + 1 < lim) ? __uint_as_float(sv[a + 1]) : -INFINITY;
      mx[e] = max3f(mx[e], xa, xb);
    }
  }
  return max3f(mx[0], mx[1], fmaxf(mx[2], mx[3]));
}

template <int D_>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc1(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, Tc1Params P) {
  typedef Layout<D_> L;
  constexpr int kGroups = D_ / 64;  // 128-byte column groups of a row
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(base + L::kOffBar);
  uint32_t *tmem_slot = (uint32_t *)(base + L::kOffMisc);
  volatile int *abort_flag = (volatile int *)(base + L::kOffMisc + 8);
  int32_t *sel_s = (int32_t *)(base + L::kOffSel);
  uint32_t *const bm = (uint32_t *)(base + L::kOffBitmap);

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HB = D.Hkv * S.batch;
  const int unit = P.n_units - 1 - (int)(blockIdx.x / HB);  // heavy (late) units first
  const int g = (blockIdx.x % HB) % D.Hkv;
  const int b = (blockIdx.x % HB) / D.Hkv;
  const int T = P.T, G = D.G, k = D.k, B = D.B;
  const int r0 = unit * T;

  const bool ok = seq_ok(S, b, threadIdx.x == 0 ? P.status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int start = ok ? seq_start(S, b) : 0;
  const int qf = seq_qfirst(S, b);
  const int r_end = min(r0 + T, S.n_q);
  const int t_lo = max(0, qf + r0);
  const int t_hi = min(len - 1, qf + r_end - 1);
  const bool has_work = ok && r0 < S.n_q && t_lo <= t_hi;
  const int n_chunks = has_work ? t_hi / kCK + 1 : 0;
  const int nwords = min((n_chunks + 31) >> 5, P.bitmap_words);
  const bool sel_cached = T * k * 4 <= (int)kSelBytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], (i == kBarPFull || i == kBarPFull + 1) ? 8u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // Q tile: rows (token, head) of KV head g, kGroups column groups of 64.
  if (has_work && warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(&bars[kBarQ], L::kQBytes);
    const int z = b * S.n_q + r0;
    for (int q = 0; q < kGroups; ++q)
      tma_load_3d(&tm_q, &bars[kBarQ], base + L::kOffQ + q * (kRows * 128), q * 64, g * G, z);
  }
  // The tile's chunk set (selected blocks and trailing ranges of its tokens) and a
  // shared-memory copy of its selection lists.
  if (warp >= 2 && has_work) {
    constexpr int kSoftThreads = kThreads - 64;
    const int ts = threadIdx.x - 64;
    for (int w = ts; w < nwords; w += kSoftThreads) bm[w] = 0;
    asm volatile("bar.sync 1, %0;" ::"n"(kSoftThreads) : "memory");
    for (int e = ts; e < T * k; e += kSoftThreads) {
      const int tok = e / k, i = e - tok * k, r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      const int j = P.sel[((size_t)b * S.n_q + r) * k + i];
      if (sel_cached) sel_s[e] = j;
      if (j < 0 || j >= (t + 1) / B) continue;
      for (int c = (j * B) / kCK; c <= (j * B + B - 1) / kCK; ++c) atomicOr(&bm[c >> 5], 1u << (c & 31));
    }
    for (int tok = ts; tok < T; tok += kSoftThreads) {
      const int r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      const int lo = ((t + 1) / B) * B;
      if (lo <= t)
        for (int c = lo / kCK; c <= t / kCK; ++c) atomicOr(&bm[c >> 5], 1u << (c & 31));
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && has_work) {
      int i = 0;
      for (int c = next_chunk(bm, nwords, 0); c >= 0; c = next_chunk(bm, nwords, c + 1), ++i) {
        const int y = start + c * kCK, z = b * D.Hkv + g;
        const int sk = i % kNK, sv = i % kNV;
        if (i >= kNK && !mbar_wait(&bars[kBarKEmpty + sk], ((i / kNK) & 1) ^ 1, kWaitNs)) {
          record_status(P.status, QSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uint8_t *ks = base + L::kOffK + sk * L::kKVBytes;
        mbar_arrive_expect_tx(&bars[kBarKFull + sk], L::kKVBytes);
        for (int q = 0; q < kGroups; ++q) tma_load_3d(&tm_k, &bars[kBarKFull + sk], ks + q * (kCK * 128), q * 64, y, z);
        if (i >= kNV && !mbar_wait(&bars[kBarVEmpty + sv], ((i / kNV) & 1) ^ 1, kWaitNs)) {
          record_status(P.status, QSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uint8_t *vs = base + L::kOffV + sv * L::kKVBytes;
        mbar_arrive_expect_tx(&bars[kBarVFull + sv], L::kKVBytes);
        for (int q = 0; q < kGroups; ++q) tma_load_3d(&tm_v, &bars[kBarVFull + sv], vs + q * (kCK * 128), q * 64, y, z);
        if (*abort_flag) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop on warp-uniform values; one elected lane issues.
    if (has_work) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kCK, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, D_, false, true);
      bool fail = !mbar_wait_warp(&bars[kBarQ], 0, kWaitNs);
      tc_fence_after();
      const uint64_t q_desc = sdesc_sw128(smem_u32(base + L::kOffQ), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(base + L::kOffK), 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(base + L::kOffV), kCK * 128, 1024);
      // S(n) = Q K_n^T into S buffer n % 2; K is K-major, 64 keys x D_.
      auto issue_qk = [&](int n) -> bool {
        if (!mbar_wait_warp(&bars[kBarKFull + n % kNK], (n / kNK) & 1, kWaitNs)) return false;
        tc_fence_after();
        const uint64_t kd = k_desc0 + (uint64_t)(((n % kNK) * L::kKVBytes) >> 4);
        const uint32_t d = tbase + (uint32_t)(D_ + (n & 1) * kCK);
#pragma unroll
        for (int kk = 0; kk < D_ / 16; ++kk) {
          const uint64_t off_q = (uint64_t)(((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4);
          const uint64_t off_k = (uint64_t)(((kk >> 2) * (kCK * 128) + (kk & 3) * 32) >> 4);
          mma_ss_w(d, q_desc + off_q, kd + off_k, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(&bars[kBarSFull + (n & 1)]);
        mma_commit_w(&bars[kBarKEmpty + n % kNK]);
        return true;
      };
      int n_total = 0;
      for (int w = 0; w < nwords; ++w) n_total += __popc(bm[w]);
      if (!fail && n_total > 0 && !issue_qk(0)) fail = true;
      if (!fail && n_total > 1 && !issue_qk(1)) fail = true;
      int c = next_chunk(bm, nwords, 0);
      for (int n = 0; n < n_total && !fail; ++n, c = next_chunk(bm, nwords, c + 1)) {
        if (!mbar_wait_warp(&bars[kBarPFull + (n & 1)], (n >> 1) & 1, kWaitNs)) { fail = true; break; }
        if (!mbar_wait_warp(&bars[kBarVFull + n % kNV], (n / kNV) & 1, kWaitNs)) { fail = true; break; }
        tc_fence_after();
        // V rows past the sequence end are zeroed: their P is zero but the buffer
        // may hold anything there, and 0 * NaN is NaN.
        const int valid_rows = len - c * kCK;
        if (valid_rows < kCK && start + len < S.kv_cap) {
          uint8_t *vs = base + L::kOffV + (n % kNV) * L::kKVBytes;
          for (int rr = max(valid_rows, 0) + lane; rr < kCK; rr += 32)
            for (int q = 0; q < kGroups; ++q) {
              uint4 *p4 = (uint4 *)(vs + q * (kCK * 128) + rr * 128);
#pragma unroll
              for (int e = 0; e < 8; ++e) p4[e] = make_uint4(0, 0, 0, 0);
            }
          fence_proxy_async_smem();
          __syncwarp();
        }
        const uint64_t vd = v_desc0 + (uint64_t)(((n % kNV) * L::kKVBytes) >> 4);
        const uint32_t pcol = tbase + (uint32_t)(D_ + (n & 1) * kCK);
#pragma unroll
        for (int kk = 0; kk < kCK / 16; ++kk)
          mma_ts_w(tbase, pcol + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv, (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(&bars[kBarVEmpty + n % kNV]);
        mma_commit_w(&bars[kBarPVDone]);
        // S(n + 2) goes into the buffer this PV has just read; MMAs run in issue order.
        if (n + 2 < n_total && !issue_qk(n + 2)) { fail = true; break; }
        if (__any_sync(0xffffffffu, *abort_flag != 0)) fail = true;
      }
      mma_commit_w(&bars[kBarODone]);
      if (fail && lane == 0) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    // Warp (lane group q, sub-group s) owns rows 32 q + 16 s .. + 15, whole: thread
    // t < 16 holds row 32 q + 16 s + t's first 32 keys of every chunk and the first
    // D_/2 columns of its O, thread t + 16 the same row's last 32 keys and last D_/2
    // columns (16x32bx2 TMEM accesses).
    const int sw = warp - 2;
    const int sub = sw >> 2;
    const int lg = warp & 3;
    const int hh = lane >> 4;
    const int row = 32 * lg + 16 * sub + (lane & 15);
    const int tok = row / G, h = row % G;
    const int r = r0 + tok, t = qf + r;
    const bool valid = has_work && r < S.n_q && t >= 0 && t < len;
    const int n_c = valid ? (t + 1) / B : 0;
    const int32_t *srow = sel_cached ? sel_s + tok * k : P.sel + ((size_t)b * S.n_q + (valid ? r : 0)) * k;
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * lg + 16 * sub) << 16);
    const float sl2 = D.scale * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;
    int ptr = 0, n = 0;
    bool fail = false;
    if (has_work) {
      for (int c = next_chunk(bm, nwords, 0); c >= 0; c = next_chunk(bm, nwords, c + 1), ++n) {
        // keys of this thread's 32 the row sees: a selected block's keys whole, the
        // trailing block's up to the query position, nothing otherwise
        int lim = 0;
        if (valid) {
          const int key0 = c * kCK + hh * 32;
          const int jb = key0 / B;
          if (jb < n_c) {
            while (ptr < k && srow[ptr] >= 0 && srow[ptr] < jb) ++ptr;
            lim = (ptr < k && srow[ptr] == jb) ? 32 : 0;
          } else {
            const int last = t - key0;
            lim = last >= 0 ? min(last + 1, 32) : 0;
          }
        }
        const bool z = __all_sync(0xffffffffu, lim == 0);
        // Masking per key is needed only where a thread sees part of its 32 keys (its
        // row's trailing block) or the chunk reaches past the sequence end (the cache
        // may hold NaN there). Otherwise each thread sees all its keys or none: one that
        // sees none takes +inf as its reference, so its p = 2^(s - inf) is 0.
        const bool part = __any_sync(0xffffffffu, lim > 0 && lim < 32) || c * kCK + kCK > len;
        const uint32_t s_col = lane_addr + (uint32_t)(D_ + (n & 1) * kCK);
        if (!warp_wait(&bars[kBarSFull + (n & 1)], (n >> 1) & 1)) { fail = true; break; }
        tc_fence_after();
        float psum = 0.f, alpha = 1.f;
        bool rescale = false;
        uint32_t sv[32];
        float hmax = -INFINITY;
        if (!z) {
          // this thread's 32 logits stay in registers: max, then P in place
          tmem_ld32_split<32>(s_col, sv);
          tmem_ld_wait();
          hmax = part ? max_quarter<false>(sv, lim) : (lim ? max_quarter<true>(sv, 32) : -INFINITY);
        }
        // the row max: the other 32 keys are in thread lane ^ 16
        const float cmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, 16)) * sl2;
        if (cmax > -INFINITY) {
          if (m_ref == -INFINITY) {
            m_ref = cmax;
          } else if (cmax > m_ref + 8.f) {
            rescale = true;
            alpha = ex2_approx(m_ref - cmax);
            m_ref = cmax;
          }
        }
        uint32_t pk[16];
        if (z) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        } else {
          const uint64_t scale2 = f2_splat(sl2);
          const uint64_t negm2 = f2_splat(part || lim ? -m_ref : -INFINITY);
          psum = part ? p_quarter<false>(sv, lim, scale2, negm2) : p_quarter<true>(sv, 32, scale2, negm2);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = sv[e];
        }
        // P of keys 32 hh .. 32 hh + 31 at columns 16 hh .. of the S buffer
        tmem_st16_split<16>(s_col, pk);
        if (__any_sync(0xffffffffu, rescale)) {
          // The reference max moved up: scale this thread's half of the row's O (and
          // its part of l) by alpha. O is stable once the previous chunk's PV has
          // completed, and this chunk's PV waits for this warp's arrival below. S of
          // this chunk being there proves the PV of chunk n - 2 complete, so one
          // parity wait suffices.
          if (n >= 1 && !warp_wait(&bars[kBarPVDone], (n - 1) & 1)) { fail = true; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < D_ / 64; ++cb) {
            uint32_t ov[32];
            tmem_ld32_split<D_ / 2>(lane_addr + cb * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
            tmem_st32_split<D_ / 2>(lane_addr + cb * 32, ov);
          }
          l *= alpha;
        }
        l += psum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPFull + (n & 1)]);
        if (*abort_flag) { fail = true; break; }
      }
    }
    // the row's sum over both key ranges
    const float l_other = __shfl_xor_sync(0xffffffffu, l, 16);
    if (fail) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // ---------------------------------------------------------------- epilogue
    // All n PVs must be complete. Having seen S of chunk n - 1 only proves that the
    // PV of chunk n - 3 is, and by the time this warp waits the PV barrier may be
    // anywhere from phase n - 2 to phase n, two of which share a parity; so the
    // epilogue waits on a barrier committed once, after the last PV.
    const bool have_o = has_work && n > 0 && !fail && warp_wait(&bars[kBarODone], 0);
    if (has_work && n > 0 && !fail && !have_o) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    const bool write = r < S.n_q && ok;
    __nv_bfloat16 *orow = P.out + (((size_t)b * S.n_q + (write ? r : 0)) * D.Hq + g * G + h) * D_ + hh * (D_ / 2);
    // A row that is not a query of the sequence (left padding) may hold NaN queries,
    // hence NaN in O: its output is written as zeros by selection, not by scaling.
    const float lt = l + l_other;
    const bool keep = valid && lt > 0.f;
    const float inv = keep ? 1.f / lt : 0.f;
    if (__all_sync(0xffffffffu, !have_o)) {
      if (write) {
        uint4 *o4 = (uint4 *)orow;
#pragma unroll 1
        for (int q = 0; q < D_ / 16; ++q) o4[q] = make_uint4(0, 0, 0, 0);
      }
    } else {
#pragma unroll 1
      for (int cb = 0; cb < D_ / 32; ++cb) {
        uint32_t ov[16];
        tmem_ld16_split<D_ / 2>(lane_addr + cb * 16, ov);
        tmem_ld_wait();
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          pk[q] = keep ? pack_bf16x2(__uint_as_float(ov[2 * q]) * inv, __uint_as_float(ov[2 * q + 1]) * inv) : 0u;
        if (write) {
          uint4 *o4 = (uint4 *)(orow + cb * 16);
          o4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          o4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, L::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// 3-D bf16 tensor map, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1_bytes,
              uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D_>
cudaError_t launch_d(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                     const int32_t *sel, void *out, int *status, cudaStream_t st) {
  typedef Layout<D_> L;
  CUtensorMap tq, tk, tv;
  const uint64_t rows_q = (uint64_t)S.batch * S.n_q;
  const int T = kRows / D.G;
  if (!encode_fn()) {
    note_error("cuTensorMapEncodeTiled entry point", cudaErrorNotSupported);
    return cudaErrorNotSupported;
  }
  if (!make_map(&tq, q, D_, D.Hq, rows_q, (uint64_t)D_ * 2, (uint64_t)D.Hq * D_ * 2, 64, D.G, T) ||
      !make_map(&tk, k, D_, S.kv_cap, (uint64_t)S.batch * D.Hkv, (uint64_t)D_ * 2, (uint64_t)S.kv_cap * D_ * 2,
                64, kCK, 1) ||
      !make_map(&tv, v, D_, S.kv_cap, (uint64_t)S.batch * D.Hkv, (uint64_t)D_ * 2, (uint64_t)S.kv_cap * D_ * 2,
                64, kCK, 1))
    return cudaErrorInvalidValue;
  Tc1Params P;
  P.D = D;
  P.S = S;
  P.sel = sel;
  P.out = (__nv_bfloat16 *)out;
  P.status = status;
  P.T = T;
  P.n_units = (S.n_q + T - 1) / T;
  const int max_chunks = (S.kv_cap + kCK - 1) / kCK;
  P.bitmap_words = (max_chunks + 31) / 32;
  const size_t smem = 1024 + L::kOffBitmap + (size_t)P.bitmap_words * 4;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  cudaError_t e = ensure_smem(k_attn_tc1<D_>, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)P.n_units * D.Hkv * S.batch;
  if (units > 0x7fffffffLL) return cudaErrorNotSupported;
  note_launch();
  k_attn_tc1<D_><<<(unsigned)units, kThreads, smem, st>>>(tq, tk, tv, P);
  e = cudaGetLastError();
  if (e != cudaSuccess) note_error("k_attn_tc1 launch", e);
  return e;
}

}  // namespace

bool attn_tc1_supported(const Dims &D) {
  return D.bf16 && D.d == 256 && D.G >= 1 && kRows % D.G == 0 && D.B % kCK == 0;
}

cudaError_t launch_attn_tc1(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                            const int32_t *sel, void *out, int *status, cudaStream_t st) {
  if (!attn_tc1_supported(D)) return cudaErrorNotSupported;
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  return launch_d<256>(D, S, q, k, v, sel, out, status, st);
}

}  // namespace qsa
