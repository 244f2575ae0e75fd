// Steps 2+3 on tcgen05 tensor cores: indexer block scores and causal top-k for a
// tile of query tokens (Hugging Face Transformers model doc "Qwen4-Exp", intro
// paragraph on QSA: several query heads score compressed key blocks and the most
// relevant blocks are selected; Qwen4ExpTextConfig indexer_budget).
//
// s[t][j] = sum_h max(0, qi[t][h] . kbar[j]) for the 32 tokens of a tile and every
// block j < n_c of the tile, with the MMA operands swapped so that a thread owns
// one block: D[j][(t, h)] = kbar[j] . qi[t][h] (M = 128 blocks, N = 32 Hi (token,
// head) pairs, K = di), then the thread sums max(0, .) over h in its own registers.
// kbar is fp32; it enters the MMA as a bf16 pair hi = bf16(kbar), lo = bf16(kbar - hi)
// (two accumulating passes), so the scores carry about 2^-16 relative error of kbar
// instead of bf16's 2^-9. The tile's scores go to shared memory as fp32 bit patterns
// (scores are >= +0, so the bit order is the value order) and each warp selects the
// top k of a token with an exact 8-bit radix select; the ids are written ascending,
// ties to the lower block index.
//
// Warps: 0 TMA producer, 1 TMEM owner and MMA issuer, 2-5 epilogue (warp w reads TMEM
// lanes 32 (w % 4) ..), then all sixteen warps run the per-token selection.
#include <cuda.h>
#include <math.h>
#include <stdio.h>

#include "qsa_internal.h"
#include "qsa_rowselect.cuh"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kTok = 32;        // query tokens per CTA
constexpr int kCand = 128;      // blocks per candidate tile (MMA M)
constexpr int kThreads = 512;  // warps 0-5 run the MMA pipeline, all 16 the selection
constexpr int kMaxBlocks = 1024;  // blocks a token may score (shared-memory score rows)
constexpr uint64_t kWaitNs = 2000000000ull;

struct ScoreParams {
  Dims D;
  Seqs S;
  int32_t *sel;
  float *scores_out;  // if set: write the rows' scores [batch][n_q][nb_cap] here, select nothing
  int *status;
  int n_tiles;  // token tiles per sequence
  int N;        // kTok * Hi
  int stages;   // candidate-tile stages and accumulator buffers: 1 when every token has at most
                // kCand candidate blocks (one tile), else 2
};

// Split fp32 kbar into bf16 hi and lo planes [batch * nb_cap][di].
__global__ void k_kbar_split(const float *__restrict__ kbar, __nv_bfloat16 *__restrict__ hi,
                             __nv_bfloat16 *__restrict__ lo, size_t n) {
  pdl_trigger();
  pdl_wait();  // k̄ comes from the kernel before (qsa_forward's compression)
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float v = kbar[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// At most 64 registers a thread, so that two CTAs fit on an SM when the shared memory
// and TMEM of one candidate stage allow it.
template <int HI>
__global__ void __launch_bounds__(kThreads, 2)
k_score_topk_tc(const __grid_constant__ CUtensorMap tm_qi, const __grid_constant__ CUtensorMap tm_hi,
                const __grid_constant__ CUtensorMap tm_lo, ScoreParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Dims &D = P.D;
  const Seqs &S = P.S;
  constexpr int Hi = HI;
  const int di = D.di, N = P.N;
  const int halves = di / 64;                       // 128-byte column groups of a row
  const uint32_t qi_bytes = (uint32_t)N * di * 2;   // B operand: N rows (token, head)
  const uint32_t cand_bytes = (uint32_t)kCand * di * 2;
  uint8_t *qi_s = base;                             // [halves][N][128 B]
  uint8_t *kb_s = base + qi_bytes;                  // [stages][hi, lo][halves][128][128 B]
  uint64_t *bars = (uint64_t *)(kb_s + 2 * P.stages * cand_bytes);
  // bars: 0 q_full, 1..2 k_full[stage], 3..4 k_empty[stage], 5..6 d_full[buf], 7..8 d_empty[buf]
  uint32_t *tmem_slot = (uint32_t *)(bars + 16);
  int *ncs = (int *)(tmem_slot + 4);                // [kTok] candidates per token (-1: padding row)
  uint32_t *scores = (uint32_t *)(ncs + kTok);      // [kTok][row stride]
  int *hist = (int *)kb_s;                          // [16 warps][256], over the candidate tiles once they are dead

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, b = blockIdx.y;
  const int r0 = tile * kTok;
  pdl_trigger();
  const bool ok = seq_ok(S, b, threadIdx.x == 0 ? P.status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int qf = seq_qfirst(S, b);

  if (threadIdx.x < kTok) {
    const int r = r0 + threadIdx.x, t = qf + r;
    ncs[threadIdx.x] = (ok && r < S.n_q && t >= 0 && t < len) ? (t + 1) / D.B : -1;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(&bars[i], (i >= 7) ? 4u : 1u);
    fence_mbar_init();
  }
  // P.stages accumulator buffers of N columns (a power of two >= 32)
  const uint32_t tcols = (uint32_t)(P.stages * N < 32 ? 32 : P.stages * N);
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  int nc_max = 0;
  for (int i = 0; i < kTok; ++i) nc_max = max(nc_max, ncs[i]);
  const int n_ct = (nc_max + kCand - 1) / kCand;   // candidate tiles with a real block
  const int row_stride = n_ct * kCand;

  bool fail = false;
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && n_ct > 0) {
      mbar_arrive_expect_tx(&bars[0], qi_bytes);
      for (int hf = 0; hf < halves; ++hf)
        tma_load_2d(&tm_qi, &bars[0], qi_s + hf * (N * 128), hf * 64, (b * S.n_q + r0) * Hi);
      pdl_wait();  // the k̄ hi/lo planes come from the kernel before
      for (int ct = 0; ct < n_ct; ++ct) {
        const int st = ct & 1;
        if (ct >= 2 && !mbar_wait(&bars[3 + st], ((ct >> 1) & 1) ^ 1, kWaitNs)) {
          fail = true;
          break;
        }
        uint8_t *dst = kb_s + st * 2 * cand_bytes;
        mbar_arrive_expect_tx(&bars[1 + st], 2 * cand_bytes);
        const int y = b * S.nb_cap + ct * kCand;
        for (int hf = 0; hf < halves; ++hf) {
          tma_load_2d(&tm_hi, &bars[1 + st], dst + hf * (kCand * 128), hf * 64, y);
          tma_load_2d(&tm_lo, &bars[1 + st], dst + cand_bytes + hf * (kCand * 128), hf * 64, y);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop on warp-uniform values; one elected lane issues.
    if (n_ct > 0) {
      const uint32_t idesc = idesc_bf16_f32(kCand, N, false, false);
      fail = !mbar_wait_warp(&bars[0], 0, kWaitNs);
      tc_fence_after();
      const uint32_t qa = smem_u32(qi_s);
      for (int ct = 0; ct < n_ct && !fail; ++ct) {
        const int st = ct & 1, buf = ct & 1;
        if (ct >= 2 && !mbar_wait_warp(&bars[7 + buf], ((ct >> 1) & 1) ^ 1, kWaitNs)) { fail = true; break; }
        if (!mbar_wait_warp(&bars[1 + st], (ct >> 1) & 1, kWaitNs)) { fail = true; break; }
        tc_fence_after();
        const uint32_t ka = smem_u32(kb_s + st * 2 * cand_bytes);
        const uint32_t d = tbase + (uint32_t)(buf * N);
        int step = 0;
        for (int part = 0; part < 2; ++part)  // hi, then lo
          for (int hf = 0; hf < halves; ++hf)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk, ++step)
              mma_ss_w(d, sdesc_sw128(ka + part * cand_bytes + hf * (kCand * 128) + kk * 32, 16, 1024),
                       sdesc_sw128(qa + hf * (N * 128) + kk * 32, 16, 1024), idesc, step > 0 ? 1u : 0u);
        mma_commit_w(&bars[5 + buf]);
        mma_commit_w(&bars[3 + st]);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue: token scores
    const int row = 32 * (warp & 3) + lane;  // candidate within the tile
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
    for (int ct = 0; ct < n_ct; ++ct) {
      const int buf = ct & 1;
      const bool got = mbar_wait(&bars[5 + buf], (ct >> 1) & 1, kWaitNs);
      if (!__all_sync(0xffffffffu, got)) { fail = true; break; }
      tc_fence_after();
      const int j = ct * kCand + row;
      for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_addr + (uint32_t)(buf * N + c0), v);
        tmem_ld_wait();
        // columns c0 .. c0 + 31 are tokens c0 / Hi .. with Hi heads each
#pragma unroll
        for (int tq = 0; tq < 32 / Hi; ++tq) {
          const int tok = c0 / Hi + tq;
          float s = 0.f;
#pragma unroll
          for (int h = 0; h < Hi; ++h) {
            const float x = __uint_as_float(v[tq * Hi + h]);
            s += x > 0.f ? x : 0.f;
          }
          if (j < ncs[tok]) {
            if (P.scores_out) P.scores_out[((size_t)b * S.n_q + r0 + tok) * S.nb_cap + j] = s;
            else scores[tok * row_stride + j] = __float_as_uint(s);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[7 + buf]);
    }
  }
  if (fail && lane == 0) record_status(P.status, QSA_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }

  // ---------------------------------------------------------------- per-token top-k
  pdl_wait();  // (returns at once: the producer's wait already covered the kernel before)
  if (P.scores_out) return;  // partial scores only: the caller reduces and selects
  int *wh = hist + warp * 256;
  for (int tok = warp; tok < kTok; tok += kThreads / 32) {
    const int r = r0 + tok;
    if (r >= S.n_q) continue;
    const uint32_t *keys = scores + tok * row_stride;
    warp_select_row([&](int j) { return keys[j]; }, ncs[tok], D.k, P.sel + ((size_t)b * S.n_q + r) * D.k, wh);
  }
}

// Step 3 from a score matrix: one warp per query row reads the row's n_c candidate
// scores from scores [batch][n_q][nb_cap] (through the order-preserving map of fp32
// to uint32, so any finite value orders correctly; -0 counts as +0) and selects as
// the fused kernels do.
constexpr int kSelWarps = 8;
__global__ void __launch_bounds__(kSelWarps * 32)
k_select_topk(Dims D, Seqs S, const float *__restrict__ scores, int32_t *__restrict__ sel, int *status) {
  __shared__ int hist[kSelWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;  // over batch * n_q
  if (row >= (long long)S.batch * S.n_q) return;
  const int b = (int)(row / S.n_q), r = (int)(row % S.n_q);
  const bool ok = seq_ok(S, b, lane == 0 ? status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int t = seq_qfirst(S, b) + r;
  const int n = (ok && t >= 0 && t < len) ? (t + 1) / D.B : -1;
  const float *srow = scores + (size_t)row * S.nb_cap;
  warp_select_row(
      [&](int j) {
        float f = __ldg(srow + j);
        if (f == 0.f) f = 0.f;
        const uint32_t u = __float_as_uint(f);
        return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      },
      n, D.k, sel + (size_t)row * D.k, hist[warp]);
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

// 2-D bf16 map [rows][cols], 128-byte swizzle, boxes of 64 columns x box_rows.
bool make_map2d(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char what[192];
    snprintf(what, sizeof what, "tensor map [%llu rows][%llu cols] box %u rows at %p: driver error %d",
             (unsigned long long)rows, (unsigned long long)cols, box_rows, ptr, (int)r);
    note_error(what, cudaErrorInvalidValue);
  }
  return r == CUDA_SUCCESS;
}

int score_stages(int nb_tile_max) { return nb_tile_max <= kCand ? 1 : 2; }
size_t smem_bytes(const Dims &D, int nb_tile_max) {
  const int N = kTok * D.Hi;
  return 1024 + (size_t)N * D.di * 2 + 2 * (size_t)score_stages(nb_tile_max) * kCand * D.di * 2 + 16 * 8 + 16 +
         kTok * 4 + (size_t)kTok * nb_tile_max * 4;
}

}  // namespace

bool score_tc_supported(const Dims &D, const Seqs &S) {
  const int nb_tiles = ((S.nb_cap + kCand - 1) / kCand) * kCand;
  return D.bf16 && (D.di == 64 || D.di == 128) && (D.Hi == 1 || D.Hi == 2 || D.Hi == 4 || D.Hi == 8) &&
         S.nb_cap <= kMaxBlocks &&
         smem_bytes(D, nb_tiles) <= 227 * 1024;
}

size_t score_tc_workspace(const Dims &D, const Seqs &S) {
  return 2 * (((size_t)S.batch * S.nb_cap * D.di * 2 + 255) & ~(size_t)255);
}

cudaError_t launch_score_topk_tc(const Dims &D, const Seqs &S, const void *qi, const float *kbar, int32_t *sel,
                                 void *scratch, int *status, cudaStream_t st, float *scores_out, bool pdl) {
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  const size_t plane = ((size_t)S.batch * S.nb_cap * D.di * 2 + 255) & ~(size_t)255;
  __nv_bfloat16 *hi = (__nv_bfloat16 *)scratch;
  __nv_bfloat16 *lo = (__nv_bfloat16 *)((char *)scratch + plane);
  const size_t n = (size_t)S.batch * S.nb_cap * D.di;
  if (n > 0) {
    note_launch();
    cudaError_t e = launch_maybe_pdl(k_kbar_split, dim3((unsigned)min((n + 255) / 256, (size_t)4096)), dim3(256), 0,
                                     st, pdl, kbar, hi, lo, n);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tq, th, tl;
  const uint64_t rows_hl = (uint64_t)S.batch * (S.nb_cap > 0 ? S.nb_cap : 1);
  if (!make_map2d(&tq, qi, D.di, (uint64_t)S.batch * S.n_q * D.Hi, kTok * D.Hi) ||
      !make_map2d(&th, hi, D.di, rows_hl, kCand) || !make_map2d(&tl, lo, D.di, rows_hl, kCand))
    return cudaErrorInvalidValue;
  ScoreParams P;
  P.D = D;
  P.S = S;
  P.sel = sel;
  P.scores_out = scores_out;
  P.status = status;
  P.n_tiles = (S.n_q + kTok - 1) / kTok;
  P.N = kTok * D.Hi;
  const int nb_tiles = ((S.nb_cap + kCand - 1) / kCand) * kCand;
  P.stages = score_stages(nb_tiles);
  const size_t smem = smem_bytes(D, nb_tiles);
  auto kern = D.Hi == 1 ? k_score_topk_tc<1> : D.Hi == 2 ? k_score_topk_tc<2> : D.Hi == 4 ? k_score_topk_tc<4>
                                                                                  : k_score_topk_tc<8>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  note_launch();
  return launch_maybe_pdl(kern, dim3(P.n_tiles, S.batch), dim3(kThreads), smem, st, pdl, tq, th, tl, P);
}

cudaError_t launch_select_topk(const Dims &D, const Seqs &S, const float *scores, int32_t *sel, int *status,
                               cudaStream_t st) {
  const long long rows = (long long)S.batch * S.n_q;
  if (rows == 0) return cudaSuccess;
  const long long grid = (rows + kSelWarps - 1) / kSelWarps;
  if (grid > 0x7fffffffLL) return cudaErrorNotSupported;
  note_launch();
  k_select_topk<<<(unsigned)grid, kSelWarps * 32, 0, st>>>(D, S, scores, sel, status);
  return cudaGetLastError();
}

}  // namespace qsa
