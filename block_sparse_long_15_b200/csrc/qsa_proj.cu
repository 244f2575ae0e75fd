// Input projections and rotary position embedding on tcgen05 tensor cores: the
// steps before the QSA path, which produce its q, k, v and indexer q / k from the
// layer's hidden states (Hugging Face Transformers model doc "Qwen4-Exp",
// Qwen4ExpTextConfig: hidden_size, attention_bias = False, rope_parameters with
// rope_theta, num_attention_heads / num_key_value_heads / head_dim,
// indexer_n_heads / indexer_head_dim with a single indexer key head).
//
// One GEMM, Y = X W^T, X [rows][D] (rows = batch x tokens), W [n_out][D] the
// stacked weight rows [W_q | W_k | W_v | W_qi | W_ki], fp32 accumulation. Its
// epilogue applies RoPE (rotate-half form: in each rotated head the pair of dims
// (i, i + r/2), i < r/2, turns by pos * theta^(-2i/r), the angle formed in fp32)
// to every q and k head and -- when enabled -- to the indexer query heads and the
// indexer key head, never to v, and writes bf16 straight into the layouts the
// path reads: q [b][r][Hq][d], k / v [b][Hkv][kv_cap][d] at row kv_row0 + r,
// qi [b][r][Hi][di], ki [b][kv_cap][di] at row kv_row0 + r.
//
// Persistent CTAs (one per SM) walk the 128 x 256 output tiles, row tiles outer so
// that the CTAs working at the same time share X tiles in L2 (W stays in L2):
//   warp 0      TMA producer: X and W k-slices (64 columns, 128-byte swizzle) into
//               a 4-stage ring;
//   warp 1      TMEM owner and single-thread MMA issuer (kind::f16, M 128, N 256,
//               K 16), two 256-column accumulators so that a tile's epilogue
//               overlaps the next tile's MMAs;
//   warps 2-9   epilogue: warp w reads TMEM lanes 32 (w % 4) .. (its 32 rows) and
//               one 128-column half of the tile.
// Every wait is bounded; on expiry the kernel records QSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <math.h>
#include <stdio.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kBM = 128;        // rows (tokens) per tile: MMA M
constexpr int kBN = 256;        // output columns per tile: MMA N
constexpr int kBK = 64;         // k columns per stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr uint32_t kABytes = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;  // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 2 * kBN;
constexpr uint64_t kWaitNs = 2000000000ull;

struct ProjParams {
  int rows, n_tok, D, n_out;
  int Hq, Hkv, d, Hi, di;
  int rd_attn, rd_idx;        // rotary dims of q/k heads and of indexer heads (0 = none)
  float rope_theta;
  const int32_t *pos0;        // [batch] position of token row 0
  __nv_bfloat16 *q, *k, *v, *qi, *ki;
  int kv_cap, kv_row0;
  int tiles_m, tiles_n;
  int *status;
};

// Where output column c of a row goes: segment (0 q, 1 k, 2 v, 3 qi, 4 ki), head
// and the head's width.
struct ColMap {
  int seg, head, hd, col0;  // col0: first column of that head
};
__device__ __forceinline__ ColMap col_map(const ProjParams &P, int c) {
  const int e_q = P.Hq * P.d, e_k = e_q + P.Hkv * P.d, e_v = e_k + P.Hkv * P.d, e_qi = e_v + P.Hi * P.di;
  ColMap m;
  if (c < e_q) { m.seg = 0; m.hd = P.d; m.head = c / P.d; m.col0 = m.head * P.d; }
  else if (c < e_k) { m.seg = 1; m.hd = P.d; m.head = (c - e_q) / P.d; m.col0 = e_q + m.head * P.d; }
  else if (c < e_v) { m.seg = 2; m.hd = P.d; m.head = (c - e_k) / P.d; m.col0 = e_k + m.head * P.d; }
  else if (c < e_qi) { m.seg = 3; m.hd = P.di; m.head = (c - e_v) / P.di; m.col0 = e_v + m.head * P.di; }
  else { m.seg = 4; m.hd = P.di; m.head = 0; m.col0 = e_qi; }
  return m;
}

// Destination of 16 consecutive dims [c, c + 16) of one head for token row (b, r).
__device__ __forceinline__ __nv_bfloat16 *dst_of(const ProjParams &P, const ColMap &m, int b, int r, int dim) {
  switch (m.seg) {
    case 0: return P.q + (((size_t)b * P.n_tok + r) * P.Hq + m.head) * P.d + dim;
    case 1: return P.k + (((size_t)b * P.Hkv + m.head) * P.kv_cap + P.kv_row0 + r) * P.d + dim;
    case 2: return P.v + (((size_t)b * P.Hkv + m.head) * P.kv_cap + P.kv_row0 + r) * P.d + dim;
    case 3: return P.qi + (((size_t)b * P.n_tok + r) * P.Hi + m.head) * P.di + dim;
    default: return P.ki + ((size_t)b * P.kv_cap + P.kv_row0 + r) * P.di + dim;
  }
}

__device__ __forceinline__ void store16(__nv_bfloat16 *dst, const float (&x)[16]) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
  uint4 *o = (uint4 *)dst;
  o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

__global__ void __launch_bounds__(kThreads, 1)
k_proj_rope(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, ProjParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(base + kStages * kStageBytes);
  uint64_t *full = bars, *empty = bars + kStages;
  uint64_t *acc_full = bars + 2 * kStages, *acc_empty = acc_full + 2;
  uint32_t *tmem_slot = (uint32_t *)(acc_empty + 2);
  volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
  float *inv_freq = (float *)(tmem_slot + 4);  // [128] attention heads, then [128] indexer heads

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = P.tiles_m * P.tiles_n;
  const int k_steps = P.D / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // rotation frequencies theta^(-2i/r), shared by every row of the CTA
  for (int i = threadIdx.x; i < 128; i += kThreads) {
    inv_freq[i] = (2 * i < P.rd_attn) ? powf(P.rope_theta, -2.f * (float)i / (float)P.rd_attn) : 0.f;
    inv_freq[128 + i] = (2 * i < P.rd_idx) ? powf(P.rope_theta, -2.f * (float)i / (float)P.rd_idx) : 0.f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x) {
        const int tm = tile / P.tiles_n, tn = tile % P.tiles_n;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int st = it % kStages;
          if (it >= kStages && !mbar_wait(&empty[st], ((it / kStages) & 1) ^ 1, kWaitNs)) {
            record_status(P.status, QSA_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          uint8_t *sa = base + st * kStageBytes, *sb = sa + kABytes;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          tma_load_2d(&tm_x, &full[st], sa, ks * kBK, tm * kBM);
          tma_load_2d(&tm_w, &full[st], sb, ks * kBK, tn * kBN);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop on warp-uniform values; one elected lane issues.
    {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, false);
      int it = 0, local = 0;
      bool fail = false;
      for (int tile = blockIdx.x; tile < n_tiles && !fail; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        // the epilogue has drained this accumulator (its use two tiles ago)
        if (local >= 2 && !mbar_wait_warp(&acc_empty[buf], ((local >> 1) & 1) ^ 1, kWaitNs)) { fail = true; break; }
        tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(buf * kBN);
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int st = it % kStages;
          if (!mbar_wait_warp(&full[st], (it / kStages) & 1, kWaitNs)) { fail = true; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + st * kStageBytes), sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss_w(d, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                     (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(&empty[st]);
        }
        if (fail) break;
        mma_commit_w(&acc_full[buf]);
        if (__any_sync(0xffffffffu, *abort_flag != 0)) fail = true;
      }
      if (fail && lane == 0) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int lg = warp & 3;                // TMEM lane group: rows 32 lg .. 32 lg + 31
    const int half = ew >> 2;               // columns [128 half, 128 half + 128) of the tile
    const int row_in_tile = 32 * lg + lane;
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * lg) << 16);
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      const int tm = tile / P.tiles_n, tn = tile % P.tiles_n;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (local >> 1) & 1, kWaitNs))) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int row = tm * kBM + row_in_tile;
      const bool row_ok = row < P.rows;
      const int b = row_ok ? row / P.n_tok : 0, r = row_ok ? row - b * P.n_tok : 0;
      const float pos = row_ok ? (float)(P.pos0[b] + r) : 0.f;
      const uint32_t acc = lane_addr + (uint32_t)(buf * kBN);
      // The tile's heads (they never straddle a tile), head by head. A head of at most
      // 128 columns belongs to the warps of the half that holds it; a wider one (256)
      // is split between the two halves by 16-dim chunk.
      const int t0 = tn * kBN;
      int c = t0;
      const int c_end = min(t0 + kBN, P.n_out);
      while (c < c_end) {
        const ColMap m = col_map(P, c);
        c = m.col0 + m.hd;
        const bool wide = m.hd > 128;
        if (!wide && ((m.col0 - t0) >> 7) != half) continue;
        const int rd = (m.seg == 0 || m.seg == 1) ? P.rd_attn : (m.seg >= 3 ? P.rd_idx : 0);
        const float *fr = inv_freq + (m.seg >= 3 ? 128 : 0);
        const int hh = rd / 2;
        const uint32_t hc = acc + (uint32_t)(m.col0 - t0);  // TMEM column of the head's dim 0
        // rotated pairs: 16-dim chunks [i0, i0 + 16) with their partners [i0 + hh, ...)
        for (int i0 = 0; i0 < hh; i0 += 16) {
          if (wide && ((i0 >> 4) & 1) != half) continue;
          uint32_t ra[16], rb[16];
          tmem_ld16(hc + (uint32_t)i0, ra);
          tmem_ld16(hc + (uint32_t)(i0 + hh), rb);
          tmem_ld_wait();
          float xa[16], xb[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float sn, cs;
            sincosf(pos * fr[i0 + e], &sn, &cs);
            const float a = __uint_as_float(ra[e]), bb = __uint_as_float(rb[e]);
            xa[e] = a * cs - bb * sn;
            xb[e] = bb * cs + a * sn;
          }
          if (row_ok) {
            store16(dst_of(P, m, b, r, i0), xa);
            store16(dst_of(P, m, b, r, i0 + hh), xb);
          }
        }
        // dims from rd on pass through
        for (int i0 = rd; i0 < m.hd; i0 += 16) {
          if (wide && ((i0 >> 4) & 1) != half) continue;
          uint32_t ra[16];
          tmem_ld16(hc + (uint32_t)i0, ra);
          tmem_ld_wait();
          float xa[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) xa[e] = __uint_as_float(ra[e]);
          if (row_ok) store16(dst_of(P, m, b, r, i0), xa);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (*abort_flag) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

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

// [rows][cols] bf16, 128-byte swizzle, boxes of 64 columns x box_rows, zero fill.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

// Shapes served: bf16, D a multiple of 64, d and di multiples of 64 up to 256 (so a
// head never straddles a 256-column tile), rotary dims multiples of 32 (0 for the
// indexer heads: not rotated).
bool proj_supported(const Dims &D, int hidden, int rd_attn, int rd_idx) {
  return D.bf16 && hidden > 0 && hidden % kBK == 0 && D.d % 64 == 0 && D.d <= 256 && D.di % 64 == 0 &&
         D.di <= 256 && ((D.Hq + 2 * D.Hkv) * D.d) % D.di == 0 && rd_attn >= 32 && rd_attn % 32 == 0 &&
         rd_attn <= D.d && rd_idx >= 0 && rd_idx % 32 == 0 && rd_idx <= D.di;
}

cudaError_t launch_proj_rope(const Dims &D, int hidden, float rope_theta, int rd_attn, int rd_idx, const void *x,
                             const void *w, const int32_t *pos0, int batch, int n_tok, void *q, void *qi, void *k,
                             void *v, void *ki, int kv_cap, int kv_row0, int *status, cudaStream_t st) {
  if (!proj_supported(D, hidden, rd_attn, rd_idx)) return cudaErrorNotSupported;
  const long long rows = (long long)batch * n_tok;
  if (rows == 0) return cudaSuccess;
  if (rows > 0x7fffffffLL) return cudaErrorNotSupported;
  ProjParams P;
  P.rows = (int)rows;
  P.n_tok = n_tok;
  P.D = hidden;
  P.Hq = D.Hq;
  P.Hkv = D.Hkv;
  P.d = D.d;
  P.Hi = D.Hi;
  P.di = D.di;
  P.n_out = D.Hq * D.d + 2 * D.Hkv * D.d + D.Hi * D.di + D.di;
  P.rd_attn = rd_attn;
  P.rd_idx = rd_idx;
  P.rope_theta = rope_theta;
  P.pos0 = pos0;
  P.q = (__nv_bfloat16 *)q;
  P.k = (__nv_bfloat16 *)k;
  P.v = (__nv_bfloat16 *)v;
  P.qi = (__nv_bfloat16 *)qi;
  P.ki = (__nv_bfloat16 *)ki;
  P.kv_cap = kv_cap;
  P.kv_row0 = kv_row0;
  P.tiles_m = (int)((rows + kBM - 1) / kBM);
  P.tiles_n = (P.n_out + kBN - 1) / kBN;
  P.status = status;
  CUtensorMap tx, tw;
  if (!encode_fn()) {
    note_error("cuTensorMapEncodeTiled entry point", cudaErrorNotSupported);
    return cudaErrorNotSupported;
  }
  if (!make_map(&tx, x, hidden, rows, kBM) || !make_map(&tw, w, hidden, P.n_out, kBN)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)kStages * kStageBytes + 256 + 2 * 128 * 4;
  cudaError_t e = ensure_smem(k_proj_rope, smem);
  if (e != cudaSuccess) return e;
  const int tiles = P.tiles_m * P.tiles_n;
  const int grid = min(tiles, sm_count());
  note_launch();
  k_proj_rope<<<grid, kThreads, smem, st>>>(tx, tw, P);
  return cudaGetLastError();
}

}  // namespace qsa
