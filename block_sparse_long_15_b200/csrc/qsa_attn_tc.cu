// Step 4 on 5th-generation tensor cores (tcgen05) for prefill: exact attention
// over each query's selected blocks plus its trailing block (Hugging Face
// Transformers model doc "Qwen4-Exp", intro paragraph on QSA; GQA per
// Qwen4ExpTextConfig num_key_value_heads).
//
// Work unit: one KV head g of one sequence and a tile of T = 128 / G consecutive
// query rows; the tile's M = 128 MMA rows are (token, query head of g) pairs, so
// the G heads that share a token's selection share every K/V tile. The unit walks
// the union of its tokens' key sets in ascending 64-key chunks (a chunk is one
// block, or a part of one): TMA stages K and V chunks (128-byte swizzle) through
// a two-stage ring; one thread issues S = Q K^T (M=128, N=64) into a double-
// buffered TMEM accumulator; four softmax warps read S rows with tcgen05.ld,
// apply each row's own mask (a chunk of a selected block is visible whole, a
// trailing chunk up to the query position, anything else not at all), keep an
// online softmax with a lazily rescaled reference max, and write P (bf16) back
// into the S columns; the MMA thread then issues O += P V (A from TMEM, B = V
// MN-major) into a TMEM fp32 accumulator. Epilogue: O / l rounded to bf16.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-5
// softmax/epilogue (warp w owns TMEM lanes 32 (w % 4) ..). Every wait is bounded;
// on expiry the kernel records QSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <math.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kD = 128;      // head dim served
constexpr int kRows = 128;   // MMA M: (token, head) rows per tile
constexpr int kChunk = 64;   // keys per chunk (MMA N of S = Q K^T)
constexpr int kStages = 2;   // K/V ring depth
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;  // S buffers at columns 0 and 64, O at 128
constexpr uint32_t kColO = 128;
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr uint32_t kQBytes = kRows * kD * 2;      // 32 KB, two 64-column halves
constexpr uint32_t kKVBytes = kChunk * kD * 2;    // 16 KB per K (or V) chunk
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKVBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kKVBytes;
constexpr uint32_t kOffMisc = kOffBar + 256;
constexpr uint32_t kOffBitmap = kOffMisc + 64;

// barrier slots
constexpr int kBarQ = 0;
constexpr int kBarKFull = 1;
constexpr int kBarVFull = kBarKFull + kStages;
constexpr int kBarKVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarKVEmpty + kStages;
constexpr int kBarPFull = kBarSFull + 2;
constexpr int kBarPVDone = kBarPFull + 2;
constexpr int kNumBars = kBarPVDone + 1;
static_assert(kNumBars * 8 <= 256, "barrier area");

struct TcParams {
  Dims D;
  Seqs S;
  const int32_t *sel;
  __nv_bfloat16 *out;
  int *status;
  int T;             // tokens per tile
  int n_tiles;       // tiles per sequence
  int bitmap_words;  // capacity of the chunk bitmap
};

// Smallest set bit >= c in the chunk bitmap, or -1.
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

// A wait taken by a whole warp: the result is the same on every lane, so the
// warp never splits around the warp-collective tcgen05 loads that follow.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 2)
k_attn_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(base + kOffBar);
  uint32_t *tmem_slot = (uint32_t *)(base + kOffMisc);
  volatile int *abort_flag = (volatile int *)(base + kOffMisc + 8);
  uint32_t *bitmap = (uint32_t *)(base + kOffBitmap);

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HB = D.Hkv * S.batch;
  const int unit = blockIdx.x;
  const int tile = P.n_tiles - 1 - unit / HB;  // heavy (late) tiles first
  const int g = (unit % HB) % D.Hkv;
  const int b = (unit % HB) / D.Hkv;
  const int T = P.T, G = D.G, k = D.k, B = D.B;
  const int r0 = tile * T;

  const bool ok = seq_ok(S, b, threadIdx.x == 0 ? P.status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int start = ok ? seq_start(S, b) : 0;
  const int qf = seq_qfirst(S, b);
  // valid query positions of the tile
  const int r_end = min(r0 + T, S.n_q);
  const int t_lo = max(0, qf + r0);
  const int t_hi = min(len - 1, qf + r_end - 1);
  const bool has_work = ok && r0 < S.n_q && t_lo <= t_hi;
  const int n_chunks = has_work ? t_hi / kChunk + 1 : 0;
  const int nwords = min((n_chunks + 31) >> 5, P.bitmap_words);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(&bars[i], (i == kBarPFull || i == kBarPFull + 1) ? 4u : 1u);
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

  // Q tile: rows (token, head) of KV head g, two 64-column halves.
  if (has_work && warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(&bars[kBarQ], kQBytes);
    const int z = b * S.n_q + r0;
    tma_load_3d(&tm_q, &bars[kBarQ], base + kOffQ, 0, g * G, z);
    tma_load_3d(&tm_q, &bars[kBarQ], base + kOffQ + kQBytes / 2, 64, g * G, z);
  }
  // Union of the tile's key chunks: selected blocks and trailing ranges.
  if (warp >= 2 && has_work) {
    const int ts = threadIdx.x - 64;
    for (int w = ts; w < nwords; w += 128) bitmap[w] = 0;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int cpb = B / kChunk;
    for (int e = ts; e < T * k; e += 128) {
      const int tok = e / k, i = e - tok * k, r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      const int j = P.sel[((size_t)b * S.n_q + r) * k + i];
      if (j < 0 || j >= (t + 1) / B) continue;
      for (int cc = 0; cc < cpb; ++cc) {
        const int c = j * cpb + cc;
        atomicOr(&bitmap[c >> 5], 1u << (c & 31));
      }
    }
    for (int tok = ts; tok < T; tok += 128) {
      const int r = r0 + tok, t = qf + r;
      if (r >= S.n_q || t < 0 || t >= len) continue;
      const int lo = ((t + 1) / B) * B;
      for (int c = lo / kChunk; lo <= t && c <= t / kChunk; ++c) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && has_work) {
      int i = 0;
      for (int c = next_chunk(bitmap, nwords, 0); c >= 0; c = next_chunk(bitmap, nwords, c + 1), ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&bars[kBarKVEmpty + s], ((i / kStages) & 1) ^ 1, kWaitNs)) {
          record_status(P.status, QSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int y = start + c * kChunk, z = b * D.Hkv + g;
        uint8_t *ks = base + kOffK + s * kKVBytes;
        uint8_t *vs = base + kOffV + s * kKVBytes;
        mbar_arrive_expect_tx(&bars[kBarKFull + s], kKVBytes);
        tma_load_3d(&tm_k, &bars[kBarKFull + s], ks, 0, y, z);
        tma_load_3d(&tm_k, &bars[kBarKFull + s], ks + kKVBytes / 2, 64, y, z);
        mbar_arrive_expect_tx(&bars[kBarVFull + s], kKVBytes);
        tma_load_3d(&tm_v, &bars[kBarVFull + s], vs, 0, y, z);
        tma_load_3d(&tm_v, &bars[kBarVFull + s], vs + kKVBytes / 2, 64, y, z);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && has_work) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kChunk, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, kD, false, true);
      const uint32_t q_addr = smem_u32(base + kOffQ);
      bool fail = !mbar_wait(&bars[kBarQ], 0, kWaitNs);
      tc_fence_after();
      // PV for chunk j (stage s), reading P from S buffer j % 2.
      auto issue_pv = [&](int j, int cj) -> bool {
        const int s = j % kStages;
        if (!mbar_wait(&bars[kBarPFull + (j & 1)], (j >> 1) & 1, kWaitNs)) return false;
        if (!mbar_wait(&bars[kBarVFull + s], (j / kStages) & 1, kWaitNs)) return false;
        tc_fence_after();
        uint8_t *vs = base + kOffV + s * kKVBytes;
        // Rows past the sequence end but inside the buffer hold whatever the cache
        // holds there; their P is zero, but 0 * NaN is NaN, so zero them first.
        const int valid_rows = len - cj * kChunk;
        if (valid_rows < kChunk && start + len < S.kv_cap) {
          for (int rr = max(valid_rows, 0); rr < kChunk; ++rr) {
            uint4 *p0 = (uint4 *)(vs + rr * 128);
            uint4 *p1 = (uint4 *)(vs + kKVBytes / 2 + rr * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) p0[q] = p1[q] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        const uint32_t v_addr = smem_u32(vs);
        const uint32_t p_col = tbase + (uint32_t)((j & 1) * kChunk);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, 8192, 1024);
          mma_ts(tbase + kColO, p_col + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kBarPVDone]);
        mma_commit(&bars[kBarKVEmpty + s]);
        return true;
      };
      int i = 0, c_prev = -1;
      for (int c = next_chunk(bitmap, nwords, 0); c >= 0 && !fail;
           c = next_chunk(bitmap, nwords, c + 1), ++i) {
        const int s = i % kStages;
        // S buffer i % 2 is free once PV of chunk i - 2 has completed.
        if (i >= 2 && !mbar_wait(&bars[kBarPVDone], i & 1, kWaitNs)) { fail = true; break; }
        if (!mbar_wait(&bars[kBarKFull + s], (i / kStages) & 1, kWaitNs)) { fail = true; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + kOffK + s * kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * (kQBytes / 2) + (kk & 3) * 32;
          mma_ss(tbase + (uint32_t)((i & 1) * kChunk), sdesc_sw128(q_addr + qoff, 16, 1024),
                 sdesc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kBarSFull + (i & 1)]);
        if (i >= 1 && !issue_pv(i - 1, c_prev)) { fail = true; break; }
        c_prev = c;
        if (*abort_flag) { fail = true; break; }
      }
      if (!fail && i >= 1 && !issue_pv(i - 1, c_prev)) fail = true;
      if (fail) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int row = 32 * (warp & 3) + lane;
    const int tok = row / G, h = row - tok * G;
    const int r = r0 + tok, t = qf + r;
    const bool valid = has_work && tok < T && r < S.n_q && t >= 0 && t < len;
    const int n_c = valid ? (t + 1) / B : 0;
    const int32_t *srow = P.sel + ((size_t)b * S.n_q + (valid ? r : 0)) * k;
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
    const float sl2 = D.scale * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;
    int ptr = 0, i = 0;
    bool fail = false;
    if (has_work) {
      for (int c = next_chunk(bitmap, nwords, 0); c >= 0; c = next_chunk(bitmap, nwords, c + 1), ++i) {
        const int sb = i & 1;
        if (!warp_wait(&bars[kBarSFull + sb], (i >> 1) & 1)) { fail = true; break; }
        tc_fence_after();
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
        uint32_t sv[64];
        tmem_ld32(lane_addr + sb * kChunk, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(lane_addr + sb * kChunk + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
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
          // O is stable once PV of chunk i - 1 has completed.
          if (i >= 1 && !warp_wait(&bars[kBarPVDone], (i - 1) & 1)) { fail = true; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < kD / 32; ++cb) {
            uint32_t ov[32];
            tmem_ld32(lane_addr + kColO + cb * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
            tmem_st32(lane_addr + kColO + cb * 32, ov);
          }
          tmem_st_wait();
          if (rescale) {
            l *= alpha;
            m_ref = cmax;
          }
        }
        float psum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 64; u += 2) {
          const float p0 = (u < lim) ? ex2_approx(__uint_as_float(sv[u]) * sl2 - m_ref) : 0.f;
          const float p1 = (u + 1 < lim) ? ex2_approx(__uint_as_float(sv[u + 1]) * sl2 - m_ref) : 0.f;
          psum += p0 + p1;
          pk[u >> 1] = pack_bf16x2(p0, p1);
        }
        l += psum;
        tmem_st32(lane_addr + sb * kChunk, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPFull + sb]);
        if (*abort_flag) { fail = true; break; }
      }
    }
    if (fail) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // ---------------------------------------------------------------- epilogue
    const bool have_o = has_work && i > 0 && !fail && warp_wait(&bars[kBarPVDone], (i - 1) & 1);
    if (has_work && i > 0 && !fail && !have_o) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    tc_fence_after();
    const bool write = tok < T && r < S.n_q && ok;
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
        tmem_ld32(lane_addr + kColO + cb * 32, ov);
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
  P.n_tiles = (S.n_q + T - 1) / T;
  const int max_chunks = (S.kv_cap + kChunk - 1) / kChunk;
  P.bitmap_words = (max_chunks + 31) / 32;
  const size_t smem = 1024 + kOffBitmap + (size_t)P.bitmap_words * 4;
  cudaError_t e = ensure_smem(k_attn_tc, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)P.n_tiles * D.Hkv * S.batch;
  if (units > 0x7fffffffLL) return cudaErrorNotSupported;
  note_launch();
  k_attn_tc<<<(unsigned)units, kThreads, smem, st>>>(tq, tk, tv, P);
  return cudaGetLastError();
}

}  // namespace qsa
