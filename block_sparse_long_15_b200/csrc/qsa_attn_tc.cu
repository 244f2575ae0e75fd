// Step 4 on 5th-generation tensor cores (tcgen05) for prefill: exact attention
// over each query's selected blocks plus its trailing block (Hugging Face
// Transformers model doc "Qwen4-Exp", intro paragraph on QSA; GQA per
// Qwen4ExpTextConfig num_key_value_heads).
//
// Work unit: one KV head g of one sequence and 2 T consecutive query rows, T =
// 128 / G, held as two 128-row MMA tiles A and B whose rows are (token, query head
// of g) pairs -- the G heads that share a token's selection share every K/V tile,
// and both tiles share every K/V chunk in shared memory. The unit walks the union
// of its tokens' key sets in ascending 128-key chunks (two 64-key halves; a half
// lies inside one block). The kernel is persistent: one CTA per SM takes units from
// an atomic ticket, heaviest (latest) units first, and prepares the next unit while
// the current one ends, so the selection read, the Q load and the first K chunk of
// a unit overlap the previous unit's last chunks. The ticket and a count of CTAs
// done with tickets sit in the workspace's status page; the last CTA sets both back
// to zero, so the workspace is zero again after every call:
//   warp 18     unit builder: takes the next ticket when the producer nears the end
//               of the current unit, writes the unit's coordinates, its per-tile chunk
//               bitmaps and a copy of its selection lists into one of two slots, and
//               releases the slot to the other warps;
//   warp 0      TMA producer: Q of each unit once every QK of the unit before has
//               completed, and K and V chunks (128-byte swizzle) into a 2-deep ring
//               whose entry j holds K of chunk j and V of chunk j - 1 under one
//               barrier, released after the QK MMAs of chunk j; the ring and every
//               barrier phase run on across units;
//   warp 1      TMEM owner and MMA issuer (the warp runs the loop, one elected
//               lane issues). Tiles ping-pong: for
//               chunk i it issues O_A += P_A V_i, S_A = Q_A K_{i+1}^T, then the
//               same for B, so one tile's softmax overlaps the other tile's MMAs.
//               A tile with no row that sees a chunk skips it. MMAs run in issue
//               order, which orders a QK after the PV that read the same columns;
//               a tile's first PV of a unit overwrites O, after the softmax warps
//               have read the previous unit's O (their P of the new unit comes later);
//   warps 2-9   softmax of tile A, warps 10-17 tile B. Warp w reads TMEM lanes
//               32 (w % 4) + 16 s .. + 15 (s one bit of w) with 16x32bx2 accesses
//               split 64 columns apart, so it owns 16 rows whole: thread t < 16 holds
//               its row's first 64-key half of the chunk, thread t + 16 the second.
//               Per chunk: tcgen05.ld of the half's 64 S columns, the row's mask for
//               the half (a half of a selected block is visible whole, a trailing
//               half up to the query position, anything else not at all), the
//               half's max, the row max by one shuffle with the partner thread,
//               online softmax with a lazily rescaled reference max, P (bf16)
//               written over the half's first 32 S columns with tcgen05.st for the
//               PV MMA (A operand from TMEM); each thread rescales and writes out
//               its 64 columns of O, and the two partial row sums meet by a shuffle.
// TMEM (512 columns): S of tile w at 128 w, O of tile w at 256 + 128 w; P of half
// h of tile w at 128 w + 64 h.
// Every wait is bounded; on expiry the kernel records QSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>

#include <algorithm>
#include <math.h>
#include <stdio.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kD = 128;      // head dim served
constexpr int kRows = 128;   // MMA M: (token, head) rows per tile
constexpr int kTiles = 2;    // tiles per CTA sharing the K/V chunks
constexpr int kChunk = 128;  // keys per chunk (MMA N of S = Q K^T, K of O += P V)
constexpr int kHalf = 64;    // mask granularity (smallest block size served)
constexpr int kNE = 2;       // ring depth: entry j holds K of chunk j and V of chunk j - 1
constexpr int kThreads = 608;  // producer, MMA, 2 tiles x 4 lane groups x 2 sixteen-row groups, builder
constexpr int kBuilderWarp = 18;
constexpr int kSoftWarps = 16;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr uint32_t kQBytes = kRows * kD * 2;    // 32 KB per tile, two 64-column halves
constexpr uint32_t kKVBytes = kChunk * kD * 2;  // 32 KB per K (or V) chunk, two halves
constexpr uint32_t kSelSlotBytes = 8192;        // a unit's selection lists, if they fit
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kEntryBytes = 2 * kKVBytes;  // K at + 0, V at + kKVBytes
constexpr uint32_t kOffE = kOffQ + kTiles * kQBytes;
constexpr uint32_t kOffBar = kOffE + kNE * kEntryBytes;
constexpr uint32_t kOffMisc = kOffBar + 512;
constexpr uint32_t kOffInfo = kOffMisc + 64;                  // [slot] UnitInfo
constexpr uint32_t kOffSel = kOffInfo + 128;                  // [slot] selection lists
constexpr uint32_t kOffBitmap = kOffSel + 2 * kSelSlotBytes;  // [slot][tile] chunk bitmaps

// barrier slots
constexpr int kBarQ = 0;                        // Q of the unit landed
constexpr int kBarQEmpty = 1;                   // every QK of the unit completed
constexpr int kBarFull = 2;                     // [ring entry]
constexpr int kBarEmpty = kBarFull + kNE;       // [ring entry]
constexpr int kBarSFull = kBarEmpty + kNE;      // [tile]
constexpr int kBarPFull = kBarSFull + 2;        // [tile], 8 arrivals (one per softmax warp)
constexpr int kBarPVDone = kBarPFull + 2;       // [tile]
constexpr int kBarSlotFull = kBarPVDone + 2;    // [slot], 32 arrivals (the builder's lanes)
constexpr int kBarSlotFree = kBarSlotFull + 2;  // [slot], producer + MMA warp + softmax warps
constexpr int kBarLead = kBarSlotFree + 2;      // the producer is kLead entries from a unit's end
constexpr int kBarSel = kBarLead + 1;           // the builder's bulk copy of a unit's lists
constexpr int kNumBars = kBarSel + 1;
constexpr int kLead = 2;
static_assert(kNumBars * 8 <= 512, "barrier area");

// A unit as the builder hands it to the other warps.
struct UnitInfo {
  int live;  // 0: no unit left, the warps leave their loops
  int b, g, r0, len, start, qf, has_work, nwords, ok;
  int pad[6];
};
static_assert(sizeof(UnitInfo) * 2 == 128, "unit info area");

struct TcParams {
  Dims D;
  Seqs S;
  const int32_t *sel;
  __nv_bfloat16 *out;
  int *status;
  unsigned *sched;   // [0] next unit ticket, [1] CTAs done taking tickets; zero between launches
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

// A wait off the critical path that sleeps between polls, leaving the sub-partition's
// issue slots to the warps that are working.
__device__ __forceinline__ bool idle_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitNs) return false;
    __nanosleep(128);
  }
  return true;
}
__device__ __forceinline__ bool idle_wait_warp(uint64_t *bar, uint32_t parity) {
  return __all_sync(0xffffffffu, idle_wait(bar, parity));
}

// *p |= bits on a shared-memory word, when pred holds (predicated, no branch)
__device__ __forceinline__ void smem_or_if(uint32_t *p, uint32_t bits, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.shared.or.b32 [%0], %1;\n\t}\n" ::"r"(smem_u32(p)),
      "r"(bits), "r"((uint32_t)pred)
      : "memory");
}

// P for one 32-key quarter held in registers (fp32 bits), written back in place
// over sv[0 .. 15] as 16 packed bf16 pairs: p = 2^(s * sl2 - m) for keys below
// `lim`, 0 from there on. Pair u lands in slot u / 2 <= u, after it was read. The
// scaled logits and the running sum use packed fp32 pairs; returns the quarter's sum.
template <bool kAll>
__device__ __forceinline__ float p_quarter_regs(uint32_t (&sv)[32], int lim, uint64_t scale2, uint64_t negm2) {
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

// Max of the first `lim` of 32 fp32 values, three at a time in 4 independent chains.
template <bool kAll>
__device__ __forceinline__ float max_quarter(const uint32_t *sv, int lim) {
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

// ---------------------------------------------------------------- unit builder
// Warp 18. Unit su goes to slot su % 2 once the warps are done with unit su - 2. The
// first unit of CTA i is unit i; later ones come from the shared ticket, taken when
// the producer is kLead entries from the end of the unit before, so a unit goes to
// the SM that is about to need one. Kept out of line: its registers do not add to
// the softmax loop's.
__device__ __noinline__ void unit_builder(const TcParams &P, uint8_t *base, int lane) {
  uint64_t *bars = (uint64_t *)(base + kOffBar);
  volatile int *abort_flag = (volatile int *)(base + kOffMisc + 8);
  UnitInfo *infos = (UnitInfo *)(base + kOffInfo);
  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int HB = D.Hkv * S.batch;
  const int T = P.T, k = D.k, B = D.B;
  const int bw = P.bitmap_words;
  const bool sel_cached = kTiles * T * k * 4 <= (int)kSelSlotBytes;
  const int total = P.n_units * HB;
  bool fail = false;
  int n_bulk = 0;  // bulk copies so far (phases of kBarSel)
  for (int su = 0;; ++su) {
    const int s = su & 1;
    bool waited = true;
    if (su >= 1) waited = idle_wait(&bars[kBarLead], (su - 1) & 1);
    if (waited && su >= 2) waited = idle_wait(&bars[kBarSlotFree + s], ((su >> 1) - 1) & 1);
    if (!__all_sync(0xffffffffu, waited)) {
      fail = true;
      break;
    }
    int tk = su == 0 ? (int)blockIdx.x : total;
    if (su > 0 && lane == 0 && !*abort_flag) tk = (int)gridDim.x + (int)atomicAdd(&P.sched[0], 1u);
    tk = __shfl_sync(0xffffffffu, tk, 0);
    UnitInfo &I = infos[s];
    if (tk >= total) {
      if (lane == 0) I.live = 0;
      __syncwarp();
      mbar_arrive(&bars[kBarSlotFull + s]);
      break;
    }
    const int unit = P.n_units - 1 - tk / HB;  // heavy (late) units first
    const int g = (tk % HB) % D.Hkv;
    const int b = (tk % HB) / D.Hkv;
    const int r0 = unit * kTiles * T;
    const bool ok = seq_ok(S, b, lane == 0 ? P.status : nullptr);
    const int len = ok ? S.kv_len[b] : 0;
    const int start = ok ? seq_start(S, b) : 0;
    const int qf = seq_qfirst(S, b);
    const int r_end = min(r0 + kTiles * T, S.n_q);
    const int t_lo = max(0, qf + r0);
    const int t_hi = min(len - 1, qf + r_end - 1);
    const bool has_work = ok && r0 < S.n_q && t_lo <= t_hi;
    const int n_chunks = has_work ? t_hi / kChunk + 1 : 0;
    const int nwords = min((n_chunks + 31) >> 5, bw);
    if (has_work) {
      // Per-tile chunk sets (selected blocks and trailing ranges of the tile's
      // tokens) and a copy of the unit's selection lists.
      uint32_t *bm0 = (uint32_t *)(base + kOffBitmap) + (s * kTiles) * bw, *bm1 = bm0 + bw;
      int32_t *sel_s = (int32_t *)(base + kOffSel + s * kSelSlotBytes);
      for (int i = lane; i < 2 * nwords; i += 32) (i < nwords ? bm0 : bm1)[i % nwords] = 0;
      __syncwarp();
      // The unit's rows are consecutive, so its lists are one contiguous range of
      // the selection: one bulk copy into the slot when it is aligned and fits,
      // else plain loads.
      const int rows = min(kTiles * T, S.n_q - r0);
      const int32_t *src_all = P.sel + ((size_t)b * S.n_q + r0) * k;
      const uint32_t bytes = (uint32_t)(rows * k * 4);
      const bool bulk = sel_cached && ((reinterpret_cast<uintptr_t>(src_all) | bytes) & 15) == 0;
      if (bulk) {
        if (lane == 0) {
          fence_proxy_async_smem();  // the slot's last readers were generic-proxy loads
          mbar_arrive_expect_tx(&bars[kBarSel], bytes);
          bulk_load(sel_s, src_all, bytes, &bars[kBarSel]);
        }
        const bool got = mbar_wait(&bars[kBarSel], n_bulk & 1, kWaitNs);
        ++n_bulk;
        if (!__all_sync(0xffffffffu, got)) {
          fail = true;
          break;
        }
      }
      // One token per lane: its list is k block ids (ascending, -1 padded); the bits
      // of one bitmap word are gathered in a register and set with one reduction.
      for (int tok = lane; tok < kTiles * T; tok += 32) {
        const int r = r0 + tok, t = qf + r;
        if (r >= S.n_q || t < 0 || t >= len) continue;
        uint32_t *bm = tok < T ? bm0 : bm1;
        const int n_c = (t + 1) / B;
        uint32_t word = 0;
        int wi = -1;
        if (bulk && (k & 3) == 0 && (B & (B - 1)) == 0 && B <= 4096) {
          // A power-of-two block covers B / 128 aligned chunks (one, for B <= 128)
          // of one bitmap word: a branch-free step per list entry. Each lane starts
          // at its own point of its list (the lists sit k words apart, which would
          // put every lane on the same banks) and loads a step ahead.
          const int sh = __ffs(B) - 1;
          const uint32_t span = B >= 4096 ? 0xffffffffu : (1u << max(B >> 7, 1)) - 1u;
          const int4 *src4 = reinterpret_cast<const int4 *>(sel_s + tok * k);
          const int nv = k >> 2;
          int m = lane % nv;
          int4 x = src4[m];
          for (int step = 0; step < nv; ++step) {
            m = m + 1 == nv ? 0 : m + 1;
            const int4 xn = src4[m];
            const int js[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int j = js[q];
              const bool v = (unsigned)j < (unsigned)n_c;
              const int c = (j << sh) >> 7;
              const int cw = v ? (c >> 5) : wi;
              const uint32_t bits = v ? span << (c & 31) : 0u;
              smem_or_if(&bm[wi], word, cw != wi && wi >= 0);
              word = cw != wi ? bits : (word | bits);
              wi = cw;
            }
            x = xn;
          }
        } else {
          const int32_t *src = bulk ? sel_s + tok * k : src_all + tok * k;
          for (int i = 0; i < k; ++i) {
            const int j = src[i];
            if (sel_cached && !bulk) sel_s[tok * k + i] = j;
            if (j >= 0 && j < n_c)
              for (int c = (j * B) / kChunk; c <= (j * B + B - 1) / kChunk; ++c) {
                smem_or_if(&bm[wi], word, (c >> 5) != wi && wi >= 0);
                word = (c >> 5) != wi ? 0u : word;
                wi = c >> 5;
                word |= 1u << (c & 31);
              }
          }
        }
        // the trailing block's keys up to the query position
        const int lo = n_c * B;
        if (lo <= t)
          for (int c = lo / kChunk; c <= t / kChunk; ++c) {
            smem_or_if(&bm[wi], word, (c >> 5) != wi && wi >= 0);
            word = (c >> 5) != wi ? 0u : word;
            wi = c >> 5;
            word |= 1u << (c & 31);
          }
        smem_or_if(&bm[wi], word, wi >= 0);
      }
      __syncwarp();
    }
    if (lane == 0) {
      I.b = b;
      I.g = g;
      I.r0 = r0;
      I.len = len;
      I.start = start;
      I.qf = qf;
      I.has_work = has_work;
      I.nwords = nwords;
      I.ok = ok;
      I.live = 1;
    }
    __syncwarp();
    mbar_arrive(&bars[kBarSlotFull + s]);
  }
  if (fail) {
    if (lane == 0) record_status(P.status, QSA_ERR_TIMEOUT);
    *abort_flag = 1;
  }
  // The last CTA to stop taking tickets sets both counters back to zero for the
  // next launch (every CTA gets here, a failed one too).
  if (lane == 0) {
    __threadfence();
    if (atomicAdd(&P.sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&P.sched[0], 0u);
      atomicExch(&P.sched[1], 0u);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(base + kOffBar);
  uint32_t *tmem_slot = (uint32_t *)(base + kOffMisc);
  volatile int *abort_flag = (volatile int *)(base + kOffMisc + 8);
  UnitInfo *infos = (UnitInfo *)(base + kOffInfo);

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = P.T, G = D.G, k = D.k, B = D.B;
  const int bw = P.bitmap_words;
  const bool sel_cached = kTiles * T * k * 4 <= (int)kSelSlotBytes;
  // chunk bitmap of tile w and selection lists of the unit in slot s
  auto bitmap = [&](int s, int w) { return (uint32_t *)(base + kOffBitmap) + (s * kTiles + w) * bw; };
  auto sel_slot = [&](int s) { return (int32_t *)(base + kOffSel + s * kSelSlotBytes); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1;
      if (i == kBarPFull || i == kBarPFull + 1) count = 8;
      if (i == kBarSlotFull || i == kBarSlotFull + 1) count = 32;
      if (i == kBarSlotFree || i == kBarSlotFree + 1) count = 2 + kSoftWarps;
      mbar_init(&bars[i], count);
    }
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
  // sel comes from the kernel before (qsa_forward's scoring, when launched as its
  // programmatic dependent); everything above read only inputs
  pdl_wait();

  if (warp == kBuilderWarp) {
    unit_builder(P, base, lane);
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Ring entry j: K of union chunk j (if any) and V of chunk j - 1 (if any), one
    // barrier for both, so the MMA warp takes one wait per chunk for PV(j - 1) and
    // QK(j), which it issues together. Entries count on across units.
    if (lane == 0) {
      int j = 0, qn = 0;  // ring entries and Q loads so far
      bool fail = false;
      for (int su = 0; !fail; ++su) {
        const int s = su & 1;
        if (!idle_wait(&bars[kBarSlotFull + s], (su >> 1) & 1)) {
          fail = true;
          break;
        }
        const UnitInfo I = infos[s];
        if (!I.live) break;
        if (I.has_work) {
          const uint32_t *bm0 = bitmap(s, 0), *bm1 = bitmap(s, 1);
          // Q of this unit, once every QK of the unit before has completed
          if (qn > 0 && !mbar_wait(&bars[kBarQEmpty], (qn - 1) & 1, kWaitNs)) {
            fail = true;
            break;
          }
          mbar_arrive_expect_tx(&bars[kBarQ], kTiles * kQBytes);
          for (int w = 0; w < kTiles; ++w) {
            const int z = I.b * S.n_q + I.r0 + w * T;
            uint8_t *dst = base + kOffQ + w * kQBytes;
            tma_load_3d(&tm_q, &bars[kBarQ], dst, 0, I.g * G, z);
            tma_load_3d(&tm_q, &bars[kBarQ], dst + kQBytes / 2, 64, I.g * G, z);
          }
          ++qn;
          const int z = I.b * D.Hkv + I.g;
          // the unit's entries: one per union chunk, and one for the last chunk's V
          int left = 1;
          for (int i = 0; i < I.nwords; ++i) left += __popc(bm0[i] | bm1[i]);
          bool lead = false;
          int cp = -1;
          int c = next_chunk(bm0, bm1, I.nwords, 0);
          while (c >= 0 || cp >= 0) {
            if (!lead && left <= kLead) {
              mbar_arrive(&bars[kBarLead]);
              lead = true;
            }
            --left;
            const int se = j % kNE;
            if (j >= kNE && !mbar_wait(&bars[kBarEmpty + se], ((j / kNE) & 1) ^ 1, kWaitNs)) {
              fail = true;
              break;
            }
            uint8_t *es = base + kOffE + se * kEntryBytes;
            mbar_arrive_expect_tx(&bars[kBarFull + se], (c >= 0 ? kKVBytes : 0u) + (cp >= 0 ? kKVBytes : 0u));
            if (c >= 0) {
              const int y = I.start + c * kChunk;
              tma_load_3d(&tm_k, &bars[kBarFull + se], es, 0, y, z);
              tma_load_3d(&tm_k, &bars[kBarFull + se], es + kKVBytes / 2, 64, y, z);
            }
            if (cp >= 0) {
              const int y = I.start + cp * kChunk;
              tma_load_3d(&tm_v, &bars[kBarFull + se], es + kKVBytes, 0, y, z);
              tma_load_3d(&tm_v, &bars[kBarFull + se], es + kKVBytes + kKVBytes / 2, 64, y, z);
            }
            cp = c;
            c = c >= 0 ? next_chunk(bm0, bm1, I.nwords, c + 1) : -1;
            ++j;
            if (*abort_flag) {
              fail = true;
              break;
            }
          }
          if (!lead) mbar_arrive(&bars[kBarLead]);
        } else {
          mbar_arrive(&bars[kBarLead]);
        }
        mbar_arrive(&bars[kBarSlotFree + s]);
        if (*abort_flag) fail = true;
      }
      if (fail) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop on warp-uniform values; one elected lane issues.
    constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kChunk, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, kD, false, true);
    int j = 0, qn = 0;          // ring entries and units with work so far
    int n_pv0 = 0, n_pv1 = 0;   // PVs issued per tile
    bool fail = false;
    // Shared-memory descriptors are built once; a k-step moves the start address,
    // which is the low field of the descriptor, so it is a 64-bit add of
    // (byte offset >> 4).
    const uint64_t q_desc0 = sdesc_sw128(smem_u32(base + kOffQ), 16, 1024);
    const uint64_t k_desc0 = sdesc_sw128(smem_u32(base + kOffE), 16, 1024);
    const uint64_t v_desc0 = sdesc_sw128(smem_u32(base + kOffE + kKVBytes), kKVBytes / 2, 1024);
    // S_w = Q_w K^T from ring entry se
    auto issue_qk = [&](int w, int se) {
      const uint64_t qd = q_desc0 + (uint64_t)((w * kQBytes) >> 4);
      const uint64_t kd = k_desc0 + (uint64_t)((se * kEntryBytes) >> 4);
      const uint32_t d = tbase + (uint32_t)(w * 128);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint64_t off_q = (uint64_t)(((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4);
        const uint64_t off_k = (uint64_t)(((kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32) >> 4);
        mma_ss_w(d, qd + off_q, kd + off_k, idesc_qk, kk > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars[kBarSFull + w]);
    };
    // O_w (+)= P_w V from ring entry se, once P_w is written; the unit's first PV of
    // the tile overwrites O
    auto issue_pv = [&](int w, int se, bool first) -> bool {
      const int cnt = w ? n_pv1++ : n_pv0++;
      if (!warp_wait(&bars[kBarPFull + w], cnt & 1)) return false;
      tc_fence_after();
      const uint64_t vd = v_desc0 + (uint64_t)((se * kEntryBytes) >> 4);
      const uint32_t o = tbase + 256u + (uint32_t)(w * 128), pcol = tbase + (uint32_t)(w * 128);
      // keys 16 kk .. 16 kk + 15 of half kk / 4 sit at columns 64 (kk / 4) + 8 (kk % 4)
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk)
        mma_ts_w(o, pcol + (kk >> 2) * 64 + (kk & 3) * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                 (!first || kk > 0) ? 1u : 0u);
      mma_commit_w(&bars[kBarPVDone + w]);
      return true;
    };
    for (int su = 0; !fail; ++su) {
      const int s = su & 1;
      if (!idle_wait_warp(&bars[kBarSlotFull + s], (su >> 1) & 1)) {
        fail = true;
        break;
      }
      const int live = infos[s].live, has_work = infos[s].has_work, nwords = infos[s].nwords;
      const int len = infos[s].len, start = infos[s].start;
      if (!live) break;
      if (has_work) {
        const uint32_t *bm0 = bitmap(s, 0), *bm1 = bitmap(s, 1);
        bool first0 = true, first1 = true;  // the tile's next PV is the unit's first
        if (!warp_wait(&bars[kBarQ], qn & 1)) fail = true;
        ++qn;
        tc_fence_after();
        int c = next_chunk(bm0, bm1, nwords, 0);  // a unit with work has a chunk
        if (!fail) {
          const int se = j % kNE;
          if (!warp_wait(&bars[kBarFull + se], (j / kNE) & 1)) fail = true;
          tc_fence_after();
          for (int w = 0; w < kTiles && !fail; ++w)
            if (bit_of(w ? bm1 : bm0, c)) issue_qk(w, se);
          if (!fail) mma_commit_w(&bars[kBarEmpty + se]);
          ++j;
        }
        int cn = fail ? -1 : next_chunk(bm0, bm1, nwords, c + 1);
        // Q is free once the unit's last QK has completed
        if (!fail && cn < 0) mma_commit_w(&bars[kBarQEmpty]);
        while (!fail && c >= 0) {
          // entry j: V of chunk c and, if there is one, K of chunk cn. V rows past the
          // sequence end are zeroed: their P is zero but the buffer may hold anything
          // there, and 0 * NaN is NaN.
          const int se = j % kNE;
          if (!warp_wait(&bars[kBarFull + se], (j / kNE) & 1)) {
            fail = true;
            break;
          }
          tc_fence_after();
          const int valid_rows = len - c * kChunk;
          if (valid_rows < kChunk && start + len < S.kv_cap) {
            uint8_t *vs = base + kOffE + se * kEntryBytes + kKVBytes;
            for (int rr = max(valid_rows, 0) + lane; rr < kChunk; rr += 32) {
              uint4 *p0 = (uint4 *)(vs + rr * 128);
              uint4 *p1 = (uint4 *)(vs + kKVBytes / 2 + rr * 128);
#pragma unroll
              for (int q = 0; q < 8; ++q) p0[q] = p1[q] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          for (int w = 0; w < kTiles; ++w) {
            if (bit_of(w ? bm1 : bm0, c)) {
              if (!issue_pv(w, se, w ? first1 : first0)) {
                fail = true;
                break;
              }
              (w ? first1 : first0) = false;
            }
            if (cn >= 0 && bit_of(w ? bm1 : bm0, cn)) issue_qk(w, se);
          }
          if (fail) break;
          mma_commit_w(&bars[kBarEmpty + se]);
          ++j;
          const int cnn = cn >= 0 ? next_chunk(bm0, bm1, nwords, cn + 1) : -1;
          if (cn >= 0 && cnn < 0) mma_commit_w(&bars[kBarQEmpty]);
          c = cn;
          cn = cnn;
          if (__any_sync(0xffffffffu, *abort_flag != 0)) fail = true;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarSlotFree + s]);
    }
    if (fail && lane == 0) {
      record_status(P.status, QSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    // Warp (tile w, lane group q, sub-group s) owns rows 32 q + 16 s .. + 15 of tile w,
    // whole: thread t < 16 holds row 32 q + 16 s + t's first 64-key half of every
    // chunk (and the first 64 columns of its O), thread t + 16 the same row's second
    // half (16x32bx2 TMEM accesses with a 64-column split).
    const int sw = warp - 2;
    const int w = sw >> 3;          // tile
    const int sub = (sw >> 2) & 1;  // which 16 of the lane group's 32 rows
    const int lg = warp & 3;        // TMEM lane group
    const int hh = lane >> 4;       // this thread's 64-key half of every chunk, and 64 columns of O
    const int row = 32 * lg + 16 * sub + (lane & 15);
    const int tok = w * T + row / G, h = row % G;
    const uint32_t lane_addr = tbase + ((uint32_t)(32 * lg + 16 * sub) << 16);
    const uint32_t s_col = lane_addr + (uint32_t)(w * 128);        // this thread reads from + 64 hh
    const uint32_t o_col = lane_addr + 256u + (uint32_t)(w * 128);  // likewise
    const float sl2 = D.scale * 1.4426950408889634f;
    int n_all = 0;  // chunks of this tile over all units so far: S, P and PV phases
    bool fail = false;
    for (int su = 0; !fail; ++su) {
      const int s = su & 1;
      if (!idle_wait_warp(&bars[kBarSlotFull + s], (su >> 1) & 1)) {
        fail = true;
        break;
      }
      // the slot stays this warp's until it releases it after the epilogue
      const UnitInfo *I = &infos[s];
      if (!I->live) break;
      const uint32_t *bm0 = bitmap(s, 0), *bm1 = bitmap(s, 1);
      const uint32_t *bm = w ? bm1 : bm0;
      const int has_work = I->has_work, nwords = I->nwords, len = I->len;
      const int t = I->qf + I->r0 + tok;  // this row's query position
      const bool valid = has_work && I->r0 + tok < S.n_q && t >= 0 && t < len;
      const int n_c = valid ? (t + 1) / B : 0;
      const int32_t *srow =
          sel_cached ? sel_slot(s) + tok * k : P.sel + ((size_t)I->b * S.n_q + (valid ? I->r0 + tok : 0)) * k;
      float m_ref = -INFINITY, l = 0.f;
      int ptr = 0, n = 0;
      if (has_work) {
        for (int c = next_chunk(bm0, bm1, nwords, 0); c >= 0; c = next_chunk(bm0, bm1, nwords, c + 1)) {
          if (!bit_of(bm, c)) continue;
          int lim = 0;
          if (valid) {
            const int key0 = c * kChunk + hh * kHalf;
            const int jb = key0 / B;
            if (jb < n_c) {
              while (ptr < k && srow[ptr] >= 0 && srow[ptr] < jb) ++ptr;
              lim = (ptr < k && srow[ptr] == jb) ? kHalf : 0;
            } else {
              const int last = t - key0;
              lim = last >= 0 ? min(last + 1, kHalf) : 0;
            }
          }
          const bool z = __all_sync(0xffffffffu, lim == 0);
          // Masking per key is needed only where a thread sees part of its half (its
          // row's trailing block) or the chunk reaches past the sequence end (the cache
          // may hold NaN there). Otherwise each thread sees all 64 keys of its half or
          // none: one that sees none takes +inf as its reference, so its p = 2^(s - inf)
          // is 0.
          const bool part = __any_sync(0xffffffffu, lim > 0 && lim < kHalf) || c * kChunk + kChunk > len;
          if (!warp_wait(&bars[kBarSFull + w], n_all & 1)) { fail = true; break; }
          tc_fence_after();
          // pass 1: the half's max over its visible keys
          float hmax = -INFINITY;
          if (!z) {
            uint32_t sv0[32], sv1[32];
            tmem_ld32_split<64>(s_col, sv0);
            tmem_ld32_split<64>(s_col + 32, sv1);
            tmem_ld_wait();
            if (part) {
              hmax = fmaxf(max_quarter<false>(sv0, lim), max_quarter<false>(sv1, lim - 32));
            } else {
              const float mx = fmaxf(max_quarter<true>(sv0, 32), max_quarter<true>(sv1, 32));
              hmax = lim ? mx : -INFINITY;
            }
          }
          // the row's max over both halves: the other half is in thread lane ^ 16
          const float cmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, 16)) * sl2;
          bool rescale = false;
          float alpha = 1.f;
          if (cmax > -INFINITY) {  // the row sees a key in this chunk
            if (m_ref == -INFINITY) {
              m_ref = cmax;
            } else if (cmax > m_ref + 8.f) {
              rescale = true;
              alpha = ex2_approx(m_ref - cmax);
              m_ref = cmax;
            }
          }
          // pass 2: P (bf16 pairs) over each half's first 32 S columns, once all 64 are read
          float psum = 0.f;
          // lanes L and L ^ 8 hold the same half of the warp's two tokens (every lane takes
          // part in these shuffles, whatever branch it goes on to)
          const int lim_x = __shfl_xor_sync(0xffffffffu, lim, 8);
          const float m_x = __shfl_xor_sync(0xffffffffu, m_ref, 8);
          const bool pairable = !part && __all_sync(0xffffffffu, !(lim > 0 && lim_x > 0));
          if (z) {
            uint32_t zk[32];
  #pragma unroll
            for (int e = 0; e < 32; ++e) zk[e] = 0u;
            tmem_st32_split<64>(s_col, zk);
          } else if (pairable) {
            // Lanes L and L ^ 8 hold the same half of the warp's two tokens. When no such
            // pair has both lanes seeing their half, the blind lane of a pair takes the
            // seeing lane's keys 32..63 and computes them with that lane's reference:
            // every lane then runs 32 exponentials instead of 64 (MUFU costs the same per
            // warp instruction whatever the lanes that take part).
            const bool mine = lim > 0, other = lim_x > 0;
            const uint64_t scale2 = f2_splat(sl2);
            const uint64_t negm2 = f2_splat(mine ? -m_ref : other ? -m_x : -INFINITY);
            uint32_t sv0[32], sv1[32];
            tmem_ld32_split<64>(s_col + 32, sv1);
            tmem_ld_wait();
  #pragma unroll
            for (int u = 0; u < 32; ++u) sv1[u] = __shfl_xor_sync(0xffffffffu, sv1[u], 8);
            tmem_ld32_split<64>(s_col, sv0);
            tmem_ld_wait();
  #pragma unroll
            for (int u = 0; u < 32; ++u) sv0[u] = mine ? sv0[u] : sv1[u];
            const float ps = p_quarter_regs<true>(sv0, 32, scale2, negm2);
            // the seeing lane's P of keys 32..63 and their sum, back from its partner
  #pragma unroll
            for (int u = 0; u < 16; ++u) {
              const uint32_t back = __shfl_xor_sync(0xffffffffu, sv0[u], 8);
              sv1[u] = mine ? back : 0u;
            }
            const float ps_other = __shfl_xor_sync(0xffffffffu, ps, 8);
            psum = mine ? ps + ps_other : 0.f;
  #pragma unroll
            for (int u = 0; u < 16; ++u) sv0[u] = mine ? sv0[u] : 0u;
            tmem_st32_split_lo<64>(s_col, sv0, sv1);
          } else {
            const uint64_t scale2 = f2_splat(sl2);
            const uint64_t negm2 = f2_splat(part || lim ? -m_ref : -INFINITY);
            uint32_t sv0[32], sv1[32];
            tmem_ld32_split<64>(s_col, sv0);
            tmem_ld_wait();
            psum = part ? p_quarter_regs<false>(sv0, lim, scale2, negm2) : p_quarter_regs<true>(sv0, 32, scale2, negm2);
            tmem_ld32_split<64>(s_col + 32, sv1);
            tmem_ld_wait();
            psum += part ? p_quarter_regs<false>(sv1, lim - 32, scale2, negm2)
                         : p_quarter_regs<true>(sv1, 32, scale2, negm2);
            tmem_st32_split_lo<64>(s_col, sv0, sv1);
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // The reference max moved up: scale this thread's half of the row's O (and
            // its part of l) by alpha. O is stable once this tile's previous PV has
            // completed, and the next PV waits for this warp's arrival below.
            if (n >= 1 && !warp_wait(&bars[kBarPVDone + w], (n_all - 1) & 1)) { fail = true; break; }
            tc_fence_after();
  #pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
              uint32_t ov[32];
              tmem_ld32_split<64>(o_col + cb * 32, ov);
              tmem_ld_wait();
  #pragma unroll
              for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
              tmem_st32_split<64>(o_col + cb * 32, ov);
            }
            l *= alpha;
          }
          l += psum;
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarPFull + w]);
          ++n;
          ++n_all;
          if (*abort_flag) { fail = true; break; }
        }
      }
      // the row's sum over both halves
      const float l_other = __shfl_xor_sync(0xffffffffu, l, 16);
      if (fail) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // -------------------------------------------------------------- epilogue
      // The unit's last PV of the tile is the barrier's phase n_all - 1: the phase
      // before it completed before S of the last chunk did, and the next one needs
      // this warp's P of the next unit.
      const bool have_o = has_work && n > 0 && !fail && warp_wait(&bars[kBarPVDone + w], (n_all - 1) & 1);
      if (has_work && n > 0 && !fail && !have_o) {
        record_status(P.status, QSA_ERR_TIMEOUT);
        *abort_flag = 1;
        fail = true;
      }
      tc_fence_after();
      const int r = I->r0 + tok;
      const bool write = r < S.n_q && I->ok;
      __nv_bfloat16 *orow = P.out + (((size_t)I->b * S.n_q + (write ? r : 0)) * D.Hq + I->g * G + h) * kD + hh * 64;
      // A row that is not a query of the sequence (left padding) may hold NaN queries,
      // hence NaN in O: its output is written as zeros by selection, not by scaling.
      const float lt = l + l_other;
      const bool keep = valid && lt > 0.f;
      const float inv = keep ? 1.f / lt : 0.f;
      if (__all_sync(0xffffffffu, !have_o)) {
        if (write) {
          uint4 *o4 = (uint4 *)orow;
#pragma unroll
          for (int q = 0; q < 8; ++q) o4[q] = make_uint4(0, 0, 0, 0);
        }
      } else {
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t ov[16];
          tmem_ld16_split<64>(o_col + cb * 16, ov);
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
      // this warp is done with the slot
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarSlotFree + s]);
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

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 148;
  return n[dev];
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
  return D.bf16 && D.d == kD && D.G >= 1 && kRows % D.G == 0 && D.B % kHalf == 0;
}

size_t attn_tc_workspace(const Dims &, const Seqs &) { return 0; }

cudaError_t launch_attn_tc(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                           const int32_t *sel, void *out, unsigned *sched, int *status, cudaStream_t st, bool pdl) {
  if (!attn_tc_supported(D)) return cudaErrorNotSupported;
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const uint64_t rows_q = (uint64_t)S.batch * S.n_q;
  const int T = kRows / D.G;
  if (!encode_fn()) {
    note_error("cuTensorMapEncodeTiled entry point", cudaErrorNotSupported);
    return cudaErrorNotSupported;
  }
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
  P.sched = sched;
  P.T = T;
  P.n_units = (S.n_q + kTiles * T - 1) / (kTiles * T);
  const int max_chunks = (S.kv_cap + kChunk - 1) / kChunk;
  P.bitmap_words = (max_chunks + 31) / 32;
  const size_t smem = 1024 + kOffBitmap + (size_t)2 * kTiles * P.bitmap_words * 4;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  cudaError_t e = ensure_smem(k_attn_tc, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)P.n_units * D.Hkv * S.batch;
  if (units > 0x7fffffffLL) return cudaErrorNotSupported;
  const int grid = (int)std::min<long long>(units, sm_count());
  note_launch();
  e = launch_maybe_pdl(k_attn_tc, dim3((unsigned)grid), dim3(kThreads), smem, st, pdl, tq, tk, tv, P);
  if (e != cudaSuccess) {
    cudaFuncAttributes a;
    char what[160];
    if (cudaFuncGetAttributes(&a, k_attn_tc) == cudaSuccess)
      snprintf(what, sizeof what, "k_attn_tc launch (regs %d, max threads %d, smem %zu)", a.numRegs,
               a.maxThreadsPerBlock, smem);
    else
      snprintf(what, sizeof what, "k_attn_tc launch");
    note_error(what, e);
  }
  return e;
}

}  // namespace qsa
