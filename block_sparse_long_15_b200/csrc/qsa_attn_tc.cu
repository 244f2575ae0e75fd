// Step 4 on 5th-generation tensor cores (tcgen05) for prefill: exact attention
// over each query's selected blocks plus its trailing block (Hugging Face
// Transformers model doc "Qwen4-Exp", intro paragraph on QSA; GQA per
// Qwen4ExpTextConfig num_key_value_heads).
//
// Work unit (one CTA per SM): one KV head g of one sequence and 2 T consecutive
// query rows, T = 128 / G, held as two 128-row MMA tiles A and B whose rows are
// (token, query head of g) pairs -- the G heads that share a token's selection
// share every K/V tile, and both tiles share every K/V chunk in shared memory.
// The unit walks the union of its tokens' key sets in ascending 64-key chunks
// (a chunk is one block or a part of one):
//   warp 0      TMA producer: K and V chunks (128-byte swizzle) into two 4-deep
//               rings, K released after its QK MMAs, V after its PV MMAs;
//   warp 1      TMEM owner and single-thread MMA issuer, per chunk
//               S_A = Q_A K^T, O_A += P_A V (previous chunk), S_B = Q_B K^T,
//               O_B += P_B V, skipping a tile for a chunk none of its rows sees;
//               MMAs run in issue order, which orders a QK after the PV that
//               last read the same S buffer;
//   warps 2-5   softmax of tile A, warps 6-9 tile B (warp w reads TMEM lanes
//               32 (w % 4) ..): tcgen05.ld of the S row, the row's mask (a chunk
//               of a selected block is visible whole, a trailing chunk up to the
//               query position, anything else not at all), online softmax with a
//               lazily rescaled reference max, P (bf16) written back into the S
//               columns with tcgen05.st for the PV MMA (A operand from TMEM);
//               epilogue O / l rounded to bf16.
// TMEM (512 columns): tile w has S buffers at 128 w + {0, 64} and O at 256 + 128 w.
// Every wait is bounded; on expiry the kernel records QSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <math.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kD = 128;      // head dim served
constexpr int kRows = 128;   // MMA M: (token, head) rows per tile
constexpr int kTiles = 2;    // tiles per CTA sharing the K/V chunks
constexpr int kChunk = 64;   // keys per chunk (MMA N of S = Q K^T)
constexpr int kNK = 4;       // K ring depth
constexpr int kNV = 4;       // V ring depth
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr uint32_t kQBytes = kRows * kD * 2;    // 32 KB per tile, two 64-column halves
constexpr uint32_t kKVBytes = kChunk * kD * 2;  // 16 KB per K (or V) chunk
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTiles * kQBytes;
constexpr uint32_t kOffV = kOffK + kNK * kKVBytes;
constexpr uint32_t kOffBar = kOffV + kNV * kKVBytes;
constexpr uint32_t kOffMisc = kOffBar + 512;
constexpr uint32_t kOffBitmap = kOffMisc + 64;

// barrier slots
constexpr int kBarQ = 0;
constexpr int kBarKFull = 1;
constexpr int kBarKEmpty = kBarKFull + kNK;
constexpr int kBarVFull = kBarKEmpty + kNK;
constexpr int kBarVEmpty = kBarVFull + kNV;
constexpr int kBarSFull = kBarVEmpty + kNV;   // [tile][2]
constexpr int kBarPFull = kBarSFull + 4;      // [tile][2], 4 arrivals (one per softmax warp)
constexpr int kBarPVDone = kBarPFull + 4;     // [tile]
constexpr int kNumBars = kBarPVDone + 2;
static_assert(kNumBars * 8 <= 512, "barrier area");

struct TcParams {
  Dims D;
  Seqs S;
  const int32_t *sel;
  __nv_bfloat16 *out;
  int *status;
  int T;             // tokens per tile
  int n_units;       // units per (sequence, KV head)
  int bitmap_words;  // capacity of each chunk bitmap
};

// Smallest set bit >= c in (bm0 | bm1), or -1.
__device__ __forceinline__ int next_chunk(const uint32_t *bm0, const uint32_t *bm1, int nwords, int c) {
  int w = c >> 5;
  if (w >= nwords) return -1;
  uint32_t bits = (bm0[w] | bm1[w]) & (0xffffffffu << (c & 31));
  while (true) {
    if (bits) return (w << 5) + __ffs(bits) - 1;
    if (++w >= nwords) return -1;
    bits = bm0[w] | bm1[w];
  }
}
__device__ __forceinline__ bool bit_of(const uint32_t *bm, int c) { return (bm[c >> 5] >> (c & 31)) & 1u; }

// A wait taken by a whole warp: the result is the same on every lane, so the
// warp never splits around the warp-collective tcgen05 loads that follow.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(base + kOffBar);
  uint32_t *tmem_slot = (uint32_t *)(base + kOffMisc);
  volatile int *abort_flag = (volatile int *)(base + kOffMisc + 8);
  uint32_t *bmap[2] = {(uint32_t *)(base + kOffBitmap),
                       (uint32_t *)(base + kOffBitmap) + P.bitmap_words};

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HB = D.Hkv * S.batch;
  const int unit = P.n_units - 1 - (int)(blockIdx.x / HB);  // heavy (late) units first
  const int g = (blockIdx.x % HB) % D.Hkv;
  const int b = (blockIdx.x % HB) / D.Hkv;
  const int T = P.T, G = D.G, k = D.k, B = D.B;
  const int r0 = unit * kTiles * T;

  const bool ok = seq_ok(S, b, threadIdx.x == 0 ? P.status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int start = ok ? seq_start(S, b) : 0;
  const int qf = seq_qfirst(S, b);
  const int r_end = min(r0 + kTiles * T, S.n_q);
  const int t_lo = max(0, qf + r0);
  const int t_hi = min(len - 1, qf + r_end - 1);
  const bool has_work = ok && r0 < S.n_q && t_lo <= t_hi;
  const int n_chunks = has_work ? t_hi / kChunk + 1 : 0;
  const int nwords = min((n_chunks + 31) >> 5, P.bitmap_words);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], (i >= kBarPFull && i < kBarPFull + 4) ? 4u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
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

  // Q tiles: rows (token, head) of KV head g; each tile two 64-column halves.
  if (has_work && warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(&bars[kBarQ], kTiles * kQBytes);
    for (int w = 0; w < kTiles; ++w) {
      const int z = b * S.n_q + r0 + w * T;
      uint8_t *dst = base + kOffQ + w * kQBytes;
      tma_load_3d(&tm_q, &bars[kBarQ], dst, 0, g * G, z);
      tma_load_3d(&tm_q, &bars[kBarQ], dst + kQBytes / 2, 64, g * G, z);
    }
  }
  // Per-tile chunk sets: selected blocks and trailing ranges of the tile's tokens.
  if (warp >= 2 && has_work) {
    const int ts = threadIdx.x - 64;
    for (int w = ts; w < 2 * nwords; w += 256) bmap[w / nwords][w % nwords] = 0;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const int cpb = B / kChunk;
    for (int e = ts; e < kTiles * T * k; e += 256) {
      const int tok = e / k, i = e - tok * k, r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      const int j = P.sel[((size_t)b * S.n_q + r) * k + i];
      if (j < 0 || j >= (t + 1) / B) continue;
      uint32_t *bm = bmap[tok / T];
      for (int cc = 0; cc < cpb; ++cc) {
        const int c = j * cpb + cc;
        atomicOr(&bm[c >> 5], 1u << (c & 31));
      }
    }
    for (int tok = ts; tok < kTiles * T; tok += 256) {
      const int r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      uint32_t *bm = bmap[tok / T];
      const int lo = ((t + 1) / B) * B;
      for (int c = lo / kChunk; lo <= t && c <= t / kChunk; ++c) atomicOr(&bm[c >> 5], 1u << (c & 31));
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && has_work) {
      int i = 0;
      for (int c = next_chunk(bmap[0], bmap[1], nwords, 0); c >= 0;
           c = next_chunk(bmap[0], bmap[1], nwords, c + 1), ++i) {
        const int y = start + c * kChunk, z = b * D.Hkv + g;
        const int sk = i % kNK, sv = i % kNV;
        if (i >= kNK && !mbar_wait(&bars[kBarKEmpty + sk], ((i / kNK) & 1) ^ 1, kWaitNs)) {
          record_status(P.status, QSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uint8_t *ks = base + kOffK + sk * kKVBytes;
        mbar_arrive_expect_tx(&bars[kBarKFull + sk], kKVBytes);
        tma_load_3d(&tm_k, &bars[kBarKFull + sk], ks, 0, y, z);
        tma_load_3d(&tm_k, &bars[kBarKFull + sk], ks + kKVBytes / 2, 64, y, z);
        if (i >= kNV && !mbar_wait(&bars[kBarVEmpty + sv], ((i / kNV) & 1) ^ 1, kWaitNs)) {
          record_status(P.status, QSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uint8_t *vs = base + kOffV + sv * kKVBytes;
        mbar_arrive_expect_tx(&bars[kBarVFull + sv], kKVBytes);
        tma_load_3d(&tm_v, &bars[kBarVFull + sv], vs, 0, y, z);
        tma_load_3d(&tm_v, &bars[kBarVFull + sv], vs + kKVBytes / 2, 64, y, z);
        if (*abort_flag) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && has_work) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kChunk, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, kD, false, true);
      bool fail = !mbar_wait(&bars[kBarQ], 0, kWaitNs);
      tc_fence_after();
      int n_act[2] = {0, 0};    // chunks issued per tile
      int pend[2] = {-1, -1};   // per-tile index of the chunk whose PV is pending
      int v_wait_done = -1;     // union index whose V arrival has been observed
      auto issue_qk = [&](int w, int i) {
        const int idx = n_act[w]++;
        const uint32_t q_addr = smem_u32(base + kOffQ + w * kQBytes);
        const uint32_t k_addr = smem_u32(base + kOffK + (i % kNK) * kKVBytes);
        const uint32_t d_col = tbase + (uint32_t)(w * 128 + (idx & 1) * kChunk);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32;
          mma_ss(d_col, sdesc_sw128(q_addr + qoff, 16, 1024), sdesc_sw128(k_addr + koff, 16, 1024), idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kBarSFull + w * 2 + (idx & 1)]);
        return idx;
      };
      // PV of tile w for the chunk at union index iu (per-tile index idx).
      auto issue_pv = [&](int w, int idx, int iu, int cu) -> bool {
        if (!mbar_wait(&bars[kBarPFull + w * 2 + (idx & 1)], (idx >> 1) & 1, kWaitNs)) return false;
        uint8_t *vs = base + kOffV + (iu % kNV) * kKVBytes;
        if (v_wait_done < iu) {
          if (!mbar_wait(&bars[kBarVFull + iu % kNV], (iu / kNV) & 1, kWaitNs)) return false;
          v_wait_done = iu;
          // Rows past the sequence end but inside the buffer hold whatever the cache
          // holds there; their P is zero, but 0 * NaN is NaN, so zero them first.
          const int valid_rows = len - cu * kChunk;
          if (valid_rows < kChunk && start + len < S.kv_cap) {
            for (int rr = max(valid_rows, 0); rr < kChunk; ++rr) {
              uint4 *p0 = (uint4 *)(vs + rr * 128);
              uint4 *p1 = (uint4 *)(vs + kKVBytes / 2 + rr * 128);
#pragma unroll
              for (int q = 0; q < 8; ++q) p0[q] = p1[q] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        tc_fence_after();
        const uint32_t v_addr = smem_u32(vs);
        const uint32_t p_col = tbase + (uint32_t)(w * 128 + (idx & 1) * kChunk);
        const uint32_t o_col = tbase + 256u + (uint32_t)(w * 128);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_ts(o_col, p_col + kk * 8, sdesc_sw128(v_addr + kk * 2048, 8192, 1024), idesc_pv,
                 (idx > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[kBarPVDone + w]);
        return true;
      };
      int i = 0, c_prev = -1;
      for (int c = next_chunk(bmap[0], bmap[1], nwords, 0); c >= 0 && !fail;
           c = next_chunk(bmap[0], bmap[1], nwords, c + 1), ++i) {
        const bool act[2] = {bit_of(bmap[0], c), bit_of(bmap[1], c)};
        if (!mbar_wait(&bars[kBarKFull + i % kNK], (i / kNK) & 1, kWaitNs)) { fail = true; break; }
        tc_fence_after();
        int idx[2] = {-1, -1};
        for (int w = 0; w < kTiles && !fail; ++w) {
          if (act[w]) idx[w] = issue_qk(w, i);
          if (pend[w] >= 0 && !issue_pv(w, pend[w], i - 1, c_prev)) fail = true;
        }
        if (fail) break;
        mma_commit(&bars[kBarKEmpty + i % kNK]);
        if (i >= 1) mma_commit(&bars[kBarVEmpty + (i - 1) % kNV]);
        pend[0] = idx[0];
        pend[1] = idx[1];
        c_prev = c;
        if (*abort_flag) fail = true;
      }
      if (!fail && i >= 1) {
        for (int w = 0; w < kTiles && !fail; ++w)
          if (pend[w] >= 0 && !issue_pv(w, pend[w], i - 1, c_prev)) fail = true;
        if (!fail) mma_commit(&bars[kBarVEmpty + (i - 1) % kNV]);
      }
      if (fail) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int w = (warp - 2) >> 2;  // tile
    const uint32_t *bm = bmap[w];
    const int row = 32 * (warp & 3) + lane;
    const int tok = w * T + row / G, h = row % G;
    const int r = r0 + tok, t = qf + r;
    const bool valid = has_work && r < S.n_q && t >= 0 && t < len;
    const int n_c = valid ? (t + 1) / B : 0;
    const int32_t *srow = P.sel + ((size_t)b * S.n_q + (valid ? r : 0)) * k;
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t s_col0 = lane_addr + (uint32_t)(w * 128);
    const uint32_t o_col = lane_addr + 256u + (uint32_t)(w * 128);
    uint64_t *s_full = &bars[kBarSFull + w * 2];
    uint64_t *p_full = &bars[kBarPFull + w * 2];
    uint64_t *pv_done = &bars[kBarPVDone + w];
    const float sl2 = D.scale * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;
    int ptr = 0, n = 0;
    bool fail = false;
    if (has_work) {
      for (int c = next_chunk(bmap[0], bmap[1], nwords, 0); c >= 0;
           c = next_chunk(bmap[0], bmap[1], nwords, c + 1)) {
        if (!bit_of(bm, c)) continue;
        const int sb = n & 1;
        int lim = 0;
        if (valid) {
          const int jb = (c * kChunk) / B;
          if (jb < n_c) {
            while (ptr < k && srow[ptr] >= 0 && srow[ptr] < jb) ++ptr;
            lim = (ptr < k && srow[ptr] == jb) ? kChunk : 0;
          } else {
            const int last = t - c * kChunk;
            lim = last >= 0 ? min(last + 1, kChunk) : 0;
          }
        }
        if (!warp_wait(&s_full[sb], (n >> 1) & 1)) { fail = true; break; }
        tc_fence_after();
        uint32_t pk[32];
        if (__all_sync(0xffffffffu, lim == 0)) {
#pragma unroll
          for (int q = 0; q < 32; ++q) pk[q] = 0u;
        } else {
          uint32_t sv[64];
          tmem_ld32(s_col0 + sb * kChunk, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(s_col0 + sb * kChunk + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld_wait();
          float cmax = -INFINITY;
#pragma unroll
          for (int u = 0; u < 64; ++u)
            if (u < lim) cmax = fmaxf(cmax, __uint_as_float(sv[u]));
          cmax *= sl2;
          bool rescale = false;
          float alpha = 1.f;
          if (lim > 0) {
            if (m_ref == -INFINITY) {
              m_ref = cmax;
            } else if (cmax > m_ref + 8.f) {
              rescale = true;
              alpha = ex2_approx(m_ref - cmax);
            }
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // O is stable once PV of this tile's previous chunk has completed.
            if (n >= 1 && !warp_wait(pv_done, (n - 1) & 1)) { fail = true; break; }
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < kD / 32; ++cb) {
              uint32_t ov[32];
              tmem_ld32(o_col + cb * 32, ov);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
              tmem_st32(o_col + cb * 32, ov);
            }
            tmem_st_wait();
            if (rescale) {
              l *= alpha;
              m_ref = cmax;
            }
          }
          float psum = 0.f;
          if (__all_sync(0xffffffffu, lim == kChunk)) {
#pragma unroll
            for (int u = 0; u < 64; u += 2) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(sv[u]), sl2, -m_ref));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sv[u + 1]), sl2, -m_ref));
              psum += p0 + p1;
              pk[u >> 1] = pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int u = 0; u < 64; u += 2) {
              const float p0 = (u < lim) ? ex2_approx(fmaf(__uint_as_float(sv[u]), sl2, -m_ref)) : 0.f;
              const float p1 = (u + 1 < lim) ? ex2_approx(fmaf(__uint_as_float(sv[u + 1]), sl2, -m_ref)) : 0.f;
              psum += p0 + p1;
              pk[u >> 1] = pack_bf16x2(p0, p1);
            }
          }
          l += psum;
        }
        tmem_st32(s_col0 + sb * kChunk, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
        ++n;
        if (*abort_flag) { fail = true; break; }
      }
    }
    if (fail) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // ---------------------------------------------------------------- epilogue
    const bool have_o = has_work && n > 0 && !fail && warp_wait(pv_done, (n - 1) & 1);
    if (has_work && n > 0 && !fail && !have_o) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    const bool write = r < S.n_q && ok;
    __nv_bfloat16 *orow = P.out + (((size_t)b * S.n_q + (write ? r : 0)) * D.Hq + g * G + h) * kD;
    const float inv = (valid && l > 0.f) ? 1.f / l : 0.f;
    if (__all_sync(0xffffffffu, !have_o)) {
      if (write) {
        uint4 *o4 = (uint4 *)orow;
#pragma unroll
        for (int q = 0; q < kD / 8; ++q) o4[q] = make_uint4(0, 0, 0, 0);
      }
    } else {
#pragma unroll 1
      for (int cb = 0; cb < kD / 32; ++cb) {
        uint32_t ov[32];
        tmem_ld32(o_col + cb * 32, ov);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pk[q] = pack_bf16x2(__uint_as_float(ov[2 * q]) * inv, __uint_as_float(ov[2 * q + 1]) * inv);
        if (write) {
          uint4 *o4 = (uint4 *)(orow + cb * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) o4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
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

}  // namespace

bool attn_tc_supported(const Dims &D) {
  return D.bf16 && D.d == kD && D.G >= 1 && kRows % D.G == 0 && D.B % kChunk == 0;
}

size_t attn_tc_workspace(const Dims &, const Seqs &) { return 0; }

cudaError_t launch_attn_tc(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                           const int32_t *sel, void *out, void *, size_t, int *status, cudaStream_t st) {
  if (!attn_tc_supported(D)) return cudaErrorNotSupported;
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const uint64_t rows_q = (uint64_t)S.batch * S.n_q;
  const int T = kRows / D.G;
  if (!make_map(&tq, q, kD, D.Hq, rows_q, (uint64_t)kD * 2, (uint64_t)D.Hq * kD * 2, 64, D.G, T) ||
      !make_map(&tk, k, kD, S.kv_cap, (uint64_t)S.batch * D.Hkv, (uint64_t)kD * 2, (uint64_t)S.kv_cap * kD * 2,
                64, kChunk, 1) ||
      !make_map(&tv, v, kD, S.kv_cap, (uint64_t)S.batch * D.Hkv, (uint64_t)kD * 2, (uint64_t)S.kv_cap * kD * 2,
                64, kChunk, 1))
    return cudaErrorInvalidValue;
  TcParams P;
  P.D = D;
  P.S = S;
  P.sel = sel;
  P.out = (__nv_bfloat16 *)out;
  P.status = status;
  P.T = T;
  P.n_units = (S.n_q + kTiles * T - 1) / (kTiles * T);
  const int max_chunks = (S.kv_cap + kChunk - 1) / kChunk;
  P.bitmap_words = (max_chunks + 31) / 32;
  const size_t smem = 1024 + kOffBitmap + (size_t)2 * P.bitmap_words * 4;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  cudaError_t e = ensure_smem(k_attn_tc, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)P.n_units * D.Hkv * S.batch;
  if (units > 0x7fffffffLL) return cudaErrorNotSupported;
  note_launch();
  k_attn_tc<<<(unsigned)units, kThreads, smem, st>>>(tq, tk, tv, P);
  return cudaGetLastError();
}

}  // namespace qsa
