// Step 4 for decode (one query row per sequence): split-KV attention over the
// selected blocks plus the trailing block, bound by HBM bandwidth (Hugging Face
// Transformers model doc "Qwen4-Exp": intro paragraph on QSA; cached generation in
// the Usage tips; GQA per Qwen4ExpTextConfig num_key_value_heads).
//
// The attended tokens of one (sequence, KV head) are its selected blocks (ascending)
// followed by the trailing block. They are cut into splits of kItems blocks; one
// CTA per (split, KV head, sequence) pulls its K and V blocks with TMA (a block of
// one head is a contiguous 64 x 128 bf16 tile, loaded as two 128-byte-swizzled
// boxes) into shared memory, all at once, and four warps run the G query heads of
// the group against them with warp-level bf16 MMAs (m16n8k16: heads as rows, keys
// as columns, fp32 accumulate) and an online softmax per warp. The warps merge in
// shared memory and the CTA writes an fp32 partial (m, l, O) to the workspace; the
// last CTA of each (sequence, KV head) to finish merges the splits with the
// log-sum-exp rule and writes bf16 (a counter in the workspace, reset after use). Rows of a partial block beyond the sequence end are masked in S and
// zeroed in V before use (the cache may hold anything there).
#include <cuda.h>
#include <math.h>
#include <stdio.h>

#include "qsa_internal.h"
#include "sm100_ptx.cuh"

namespace qsa {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kBlk = 64;          // keys per block tile (the block size served)
constexpr int kItems = 2;         // blocks per split
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kTileBytes = kBlk * kD * 2;  // 16 KB per K (or V) block
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxG = 8;          // query heads per KV head served (MMA rows 0..7)

struct DecParams {
  Dims D;
  Seqs S;
  const __nv_bfloat16 *q;
  const int32_t *sel;
  __nv_bfloat16 *out;
  float *part;      // [batch][Hkv][max_splits][G][d]: O of each split (unnormalised)
  float *part_ml;   // [batch][Hkv][max_splits][G][2]: m (log2 domain) and l of each split
  int *done;        // [batch][Hkv] splits finished in this call; the merging CTA resets it to 0
  int max_splits;
  int *status;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte chunk) inside a 128-byte-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads)
k_attn_decode(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, DecParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *ks = base;                                  // kItems x 16 KB
  uint8_t *vs = base + kItems * kTileBytes;            // kItems x 16 KB
  uint64_t *bars = (uint64_t *)(base + 2 * kItems * kTileBytes);
  float *red = (float *)base;  // merge scratch, reuses the K/V tiles once they are consumed

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool ok = seq_ok(S, b, threadIdx.x == 0 ? P.status : nullptr);
  const int len = ok ? S.kv_len[b] : 0;
  const int start = ok ? seq_start(S, b) : 0;
  const int t = seq_qfirst(S, b);
  if (!ok || t < 0 || t >= len) {
    // padding row: split 0 writes the group's output rows as zeros
    if (split == 0)
      for (int e = threadIdx.x; e < D.G * kD; e += kThreads)
        P.out[((size_t)b * S.n_q * D.Hq + (size_t)g * D.G) * kD + e] = __float2bfloat16_rn(0.f);
    return;
  }
  const int n_c = (t + 1) / D.B;
  const int n_sel = min(n_c, D.k);
  const bool trailing = n_c * D.B <= t;
  const int n_items = n_sel + (trailing ? 1 : 0);
  const int item0 = split * kItems;
  if (item0 >= n_items) return;
  const int n_mine = min(kItems, n_items - item0);
  const int32_t *srow = P.sel + (size_t)b * S.n_q * D.k;  // decode: one query row per sequence

  // block start (relative key position) and number of valid keys of item i
  auto item_block = [&](int i, int &key0, int &nkeys) {
    if (i < n_sel) {
      key0 = srow[i] * D.B;
      nkeys = kBlk;
    } else {
      key0 = n_c * D.B;
      nkeys = t + 1 - key0;
    }
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kItems; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int z = b * D.Hkv + g;
    for (int i = 0; i < n_mine; ++i) {
      int key0, nk;
      item_block(item0 + i, key0, nk);
      mbar_arrive_expect_tx(&bars[i], 4 * (kTileBytes / 2));
      uint8_t *kd = ks + i * kTileBytes, *vd = vs + i * kTileBytes;
      tma_load_3d(&tm_k, &bars[i], kd, 0, start + key0, z);
      tma_load_3d(&tm_k, &bars[i], kd + kTileBytes / 2, 64, start + key0, z);
      tma_load_3d(&tm_v, &bars[i], vd, 0, start + key0, z);
      tma_load_3d(&tm_v, &bars[i], vd + kTileBytes / 2, 64, start + key0, z);
    }
  }

  // q of the group as the A operand: rows = heads (0..G-1, rest zero), 8 k-steps of 16 dims.
  const int head = lane >> 2;  // A/C row owned by this lane (rows 8..15 are padding)
  const int G = D.G;
  uint32_t qa[8][2];
  {
    const __nv_bfloat16 *qrow = P.q + (((size_t)b * S.n_q) * D.Hq + (size_t)g * G + head) * kD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int c0 = kk * 16 + 2 * (lane & 3);
      if (head < G) {
        qa[kk][0] = *(const uint32_t *)(qrow + c0);
        qa[kk][1] = *(const uint32_t *)(qrow + c0 + 8);
      } else {
        qa[kk][0] = qa[kk][1] = 0u;
      }
    }
  }
  const float sl2 = D.scale * 1.4426950408889634f;
  float m = -INFINITY, l = 0.f;
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

  bool fail = false;
  for (int i = 0; i < n_mine; ++i) {
    int key0, nk;
    item_block(item0 + i, key0, nk);
    const bool got = mbar_wait(&bars[i], 0, kWaitNs);
    if (__syncthreads_or(!got)) {  // uniform across the CTA: no thread is left at a barrier
      fail = true;
      break;
    }
    const uint32_t kb = smem_u32(ks + i * kTileBytes), vb = smem_u32(vs + i * kTileBytes);
    if (nk < kBlk) {
      // zero V rows past the sequence end (generic writes, read below by ldmatrix)
      uint8_t *vd = vs + i * kTileBytes;
      for (int e = threadIdx.x; e < (kBlk - nk) * 16; e += kThreads) {
        const int rr = nk + e / 16, cc = e % 16;
        *(uint4 *)(vd + (cc >> 3) * (kTileBytes / 2) + rr * 128 + ((cc & 7) << 4)) = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
    }
    // this warp's 16 keys of the block: rows 16 warp .. 16 warp + 15
    const int r0 = warp * 16;
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      // B fragments (K^T, col-major) for 2 key tiles: rows = keys, 16-byte chunks of dims.
      const int half = kk >> 2;
      const int mtx = lane >> 3, rr = lane & 7;
      const int key = r0 + (mtx >> 1) * 8 + rr;
      const int chunk = (kk & 3) * 2 + (mtx & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + half * (kTileBytes / 2) + sw128(key, chunk), b0, b1, b2, b3);
      mma16816(s[0], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
      mma16816(s[1], qa[kk][0], 0u, qa[kk][1], 0u, b2, b3);
    }
    // mask and online softmax for row `head` over this warp's 16 keys
    float x[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = r0 + nt * 8 + 2 * (lane & 3) + e;
        x[nt * 2 + e] = key < nk ? s[nt][e] * sl2 : -INFINITY;
      }
    float cmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
    const float m_new = fmaxf(m, cmax);
    const float corr = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = (x[e] == -INFINITY) ? 0.f : ex2_approx(x[e] - m_new);
    float ps = (p[0] + p[1]) + (p[2] + p[3]);
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l = l * corr + ps;
    m = m_new;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= corr;
      o[nt][1] *= corr;
    }
    // P (rows = heads, 16 keys) as the A operand; rows 8..15 are zero.
    const uint32_t pa0 = pack_bf16x2(p[0], p[1]);
    const uint32_t pa2 = pack_bf16x2(p[2], p[3]);
    // O += P V: B = V (16 keys x 8 dims per tile), loaded transposed from [key][dim] rows.
#pragma unroll
    for (int nt2 = 0; nt2 < 8; ++nt2) {
      const int mtx = lane >> 3, rr = lane & 7;
      const int key = r0 + (mtx & 1) * 8 + rr;
      const int dim_chunk = nt2 * 2 + (mtx >> 1);  // 16-byte chunk of 8 dims (0..15)
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(vb + (dim_chunk >> 3) * (kTileBytes / 2) + sw128(key, dim_chunk & 7), v0, v1, v2, v3);
      mma16816(o[2 * nt2], pa0, 0u, pa2, 0u, v0, v1);
      mma16816(o[2 * nt2 + 1], pa0, 0u, pa2, 0u, v2, v3);
    }
  }
  if (fail) {
    record_status(P.status, QSA_ERR_TIMEOUT);
    return;
  }
  __syncthreads();  // every warp is done with the K/V tiles before they become merge scratch
  // merge the warps: each lane of a quad holds dims 8 nt + 2 (lane & 3) + {0,1} of row `head`
  float *wm = red;                        // [warps][8]
  float *wl = red + kWarps * 8;           // [warps][8]
  float *wo = red + 2 * kWarps * 8;       // [warps][8][128]
  if ((lane & 3) == 0 && head < kMaxG) {
    wm[warp * 8 + head] = m;
    wl[warp * 8 + head] = l;
  }
  if (head < kMaxG) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int dcol = nt * 8 + 2 * (lane & 3);
      wo[(warp * 8 + head) * kD + dcol] = o[nt][0];
      wo[(warp * 8 + head) * kD + dcol + 1] = o[nt][1];
    }
  }
  __syncthreads();
  const size_t unit = (size_t)b * D.Hkv + g;
  float *dst = P.part + (unit * P.max_splits + split) * G * kD;
  float *dst_ml = P.part_ml + (unit * P.max_splits + split) * G * 2;
  for (int e = threadIdx.x; e < G * kD; e += kThreads) {
    const int hh = e / kD, dd = e % kD;
    float mm = -INFINITY;
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, wm[w * 8 + hh]);
    float acc = 0.f, ll = 0.f;
    for (int w = 0; w < kWarps; ++w) {
      const float f = (wm[w * 8 + hh] == -INFINITY) ? 0.f : ex2_approx(wm[w * 8 + hh] - mm);
      acc += f * wo[(w * 8 + hh) * kD + dd];
      ll += f * wl[w * 8 + hh];
    }
    dst[e] = acc;
    if (dd == 0) {
      dst_ml[hh * 2] = mm;
      dst_ml[hh * 2 + 1] = ll;
    }
  }
  // The last split of this (sequence, KV head) to finish merges all of them:
  // O = sum_s 2^(m_s - m) O_s / sum_s 2^(m_s - m) l_s, then resets the counter.
  const int n_splits = (n_items + kItems - 1) / kItems;
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&P.done[unit], 1) == n_splits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float *fw = red;                     // [n_splits][G] weights 2^(m_s - m)
  float *inv_l = red + P.max_splits * kMaxG;  // [G]
  const float *ml = P.part_ml + unit * P.max_splits * G * 2;
  if (threadIdx.x < G) {
    const int hh = threadIdx.x;
    float mm = -INFINITY;
    for (int sp = 0; sp < n_splits; ++sp) mm = fmaxf(mm, __ldcg(&ml[(sp * G + hh) * 2]));
    float ll = 0.f;
    for (int sp = 0; sp < n_splits; ++sp) {
      const float ms = __ldcg(&ml[(sp * G + hh) * 2]);
      const float f = (ms == -INFINITY) ? 0.f : ex2_approx(ms - mm);
      fw[sp * G + hh] = f;
      ll += f * __ldcg(&ml[(sp * G + hh) * 2 + 1]);
    }
    inv_l[hh] = ll > 0.f ? 1.f / ll : 0.f;
  }
  __syncthreads();
  const float4 *src = (const float4 *)(P.part + unit * P.max_splits * G * kD);
  __nv_bfloat16 *orow = P.out + ((size_t)b * S.n_q * D.Hq + (size_t)g * G) * kD;
  for (int e4 = threadIdx.x; e4 < G * kD / 4; e4 += kThreads) {
    const int hh = (e4 * 4) / kD;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int sp = 0; sp < n_splits; ++sp) {
      const float4 o4 = __ldcg(&src[(size_t)sp * (G * kD / 4) + e4]);
      const float f = fw[sp * G + hh];
      acc.x = fmaf(f, o4.x, acc.x);
      acc.y = fmaf(f, o4.y, acc.y);
      acc.z = fmaf(f, o4.z, acc.z);
      acc.w = fmaf(f, o4.w, acc.w);
    }
    const float il = inv_l[hh];
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * il, acc.y * il);
    pk.y = pack_bf16x2(acc.z * il, acc.w * il);
    *(uint2 *)(orow + e4 * 4) = pk;
  }
  if (threadIdx.x == 0) P.done[b * D.Hkv + g] = 0;
}

// ---------------------------------------------------------------------------
// Persistent streaming variant. The items (attended blocks) of all (sequence,
// KV head) units, in unit order, form one list; CTA c of C streams the contiguous
// range [floor(c T / C), floor((c+1) T / C)) of it through a kStages-deep ring of
// K+V blocks filled by a producer warp, so that HBM always has loads in flight.
// Four compute warps process each block as the split kernel does (16 keys per
// warp, online softmax per warp); at every unit boundary inside its range the CTA
// merges its warps and writes one partial to slot (unit + c), and the last CTA
// to finish a unit merges that unit's partials into the bf16 output.
// ---------------------------------------------------------------------------
constexpr int kStages = 6;
constexpr int kPThreads = (kWarps + 1) * 32;  // warp kWarps is the producer
constexpr int kMaxUnits = 2048;

struct PstParams {
  Dims D;
  Seqs S;
  const __nv_bfloat16 *q;
  const int32_t *sel;
  __nv_bfloat16 *out;
  float *part;      // [n_units + C][G][d]
  float *part_ml;   // [n_units + C][G][2]
  int *done;        // [n_units]
  int n_units, C;
  int *status;
};

// n_items of the unit's sequence: selected blocks plus the trailing block (0 for padding rows).
__device__ __forceinline__ int unit_items(const Dims &D, const Seqs &S, int b, int &t, int &n_c) {
  t = -1;
  n_c = 0;
  const int st = seq_start(S, b), len = S.kv_len[b];
  if (st < 0 || len < 0 || (long long)st + len > (long long)S.kv_cap) return 0;
  t = seq_qfirst(S, b);
  if (t < 0 || t >= len) return 0;
  n_c = (t + 1) / D.B;
  return min(n_c, D.k) + ((n_c * D.B <= t) ? 1 : 0);
}

// CTA owning item i: floor(c T / C) <= i < floor((c+1) T / C)  <=>  c = ceil((i+1) C / T) - 1.
__device__ __forceinline__ int cta_of(long long i, int C, long long T) {
  return (int)(((i + 1) * C + T - 1) / T) - 1;
}

__global__ void __launch_bounds__(kPThreads, 1)
k_attn_decode_pst(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, PstParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *ring = base;                                            // kStages x (K 16 KB + V 16 KB)
  uint64_t *full = (uint64_t *)(base + kStages * 2 * kTileBytes);  // [kStages]
  uint64_t *empty = full + kStages;                                // [kStages]
  float *mrg = (float *)(empty + kStages);                         // warp merge scratch
  int *pre = (int *)(mrg + 2 * kWarps * 8 + kWarps * 8 * kD);  // [n_units + 1]
  __shared__ int s_last, s_fail;

  const Dims &D = P.D;
  const Seqs &S = P.S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, U = P.n_units, G = D.G;

  // Everything up to the grid-dependency wait below reads only the sequence
  // geometry (kv_len, kv_start, q_first), which the kernel before this one in the
  // stream (the decode append + selection) does not write, so with programmatic
  // dependent launch it overlaps that kernel's tail.
  __shared__ int s_wsum[kPThreads / 32];
  if (threadIdx.x == 0) {
    pre[0] = 0;
    s_fail = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    fence_mbar_init();
  }
  if (warp == kWarps && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  {
    // unit prefix sums, every CTA for itself: each thread counts a contiguous run
    // of units, then a scan over the threads' run totals gives each run's offset
    const int per = (U + kPThreads - 1) / kPThreads;
    const int u_a = min(U, (int)threadIdx.x * per), u_z = min(U, u_a + per);
    int run = 0;
    for (int u = u_a; u < u_z; ++u) {
      int t, n_c;
      const int v = unit_items(D, S, u / D.Hkv, t, n_c);
      pre[u + 1] = v;
      run += v;
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int acc = incl - run;
    for (int w = 0; w < warp; ++w) acc += s_wsum[w];
    for (int u = u_a; u < u_z; ++u) {
      acc += pre[u + 1];
      pre[u + 1] = acc;
    }
  }
  __syncthreads();
  const long long T = pre[U];
  // sel and the cache rows appended this step come from the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // padding units: CTA (u mod grid) writes their output rows as zeros
  for (int u = c; u < U; u += P.C) {
    if (pre[u + 1] != pre[u]) continue;
    const int b = u / D.Hkv, g = u % D.Hkv;
    for (int e = threadIdx.x; e < G * kD; e += kPThreads)
      P.out[((size_t)b * S.n_q * D.Hq + (size_t)g * G) * kD + e] = __float2bfloat16_rn(0.f);
  }
  // With C <= T every CTA range is non-empty, so the CTAs between a unit's first and
  // last part all hold a part of it.
  const int C = (int)min((long long)P.C, T);
  if (c >= C) return;
  const long long lo = (long long)c * T / C, hi = (long long)(c + 1) * T / C;
  // first unit of the range: largest u with pre[u] <= lo
  int u0 = 0;
  {
    int a = 0, z = U;
    while (z - a > 1) {
      const int mid = (a + z) >> 1;
      if (pre[mid] <= lo) a = mid;
      else z = mid;
    }
    u0 = a;
    while (u0 < U && pre[u0 + 1] <= lo) ++u0;
  }

  // item -> (unit, key0, valid keys)
  auto locate = [&](int &u, long long i, int &key0, int &nk) {
    while (pre[u + 1] <= i) ++u;
    const int b = u / D.Hkv;
    const int t = seq_qfirst(S, b);
    const int n_c = (t + 1) / D.B, n_sel = min(n_c, D.k);
    const int j = (int)(i - pre[u]);
    if (j < n_sel) {
      key0 = P.sel[(size_t)b * S.n_q * D.k + j] * D.B;
      nk = kBlk;
    } else {
      key0 = n_c * D.B;
      nk = t + 1 - key0;
    }
  };

  if (warp == kWarps) {
    // ---------------------------------------------------------------- producer
    // The warp resolves the coordinates of the next 32 items in parallel (one per
    // lane, so the global reads of kv_len and sel overlap), then lane 0 issues them.
    int u = u0;
    for (long long i0 = lo; i0 < hi; i0 += 32) {
      const long long i = i0 + lane;
      int y = 0, z = 0;
      if (i < hi) {
        int ul = u;
        int key0, nk;
        locate(ul, i, key0, nk);
        const int b = ul / D.Hkv;
        y = seq_start(S, b) + key0;
        z = b * D.Hkv + ul % D.Hkv;
      }
      // the unit of the last item of this batch starts the next batch's search
      const long long last = min(hi, i0 + 32) - 1;
      while (pre[u + 1] <= last) ++u;
      const int cnt = (int)min((long long)32, hi - i0);
      bool fail = false;
      for (int j = 0; j < cnt; ++j) {
        const int yj = __shfl_sync(0xffffffffu, y, j), zj = __shfl_sync(0xffffffffu, z, j);
        const int n = (int)(i0 - lo) + j, st = n % kStages;
        if (lane == 0) {
          if (n >= kStages && !mbar_wait(&empty[st], ((n / kStages) & 1) ^ 1, kWaitNs)) {
            record_status(P.status, QSA_ERR_TIMEOUT);
            fail = true;
          } else {
            uint8_t *kd = ring + st * 2 * kTileBytes, *vd = kd + kTileBytes;
            mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
            tma_load_3d(&tm_k, &full[st], kd, 0, yj, zj);
            tma_load_3d(&tm_k, &full[st], kd + kTileBytes / 2, 64, yj, zj);
            tma_load_3d(&tm_v, &full[st], vd, 0, yj, zj);
            tma_load_3d(&tm_v, &full[st], vd + kTileBytes / 2, 64, yj, zj);
          }
        }
        if (__shfl_sync(0xffffffffu, (int)fail, 0)) break;
      }
      if (__shfl_sync(0xffffffffu, (int)fail, 0)) break;
    }
    return;  // the producer takes no part in the named barriers below
  }

  // ---------------------------------------------------------------- compute warps
  const int head = lane >> 2;
  const float sl2 = D.scale * 1.4426950408889634f;
  float m = -INFINITY, l = 0.f;
  float o[16][4];
  uint32_t qa[8][2];
  int u = u0, u_loaded = -1;
  bool fail = false;
  float *wm = mrg, *wl = mrg + kWarps * 8, *wo = mrg + 2 * kWarps * 8;
  int u_t = 0, u_nc = 0, u_nsel = 0;  // geometry of the current unit
  for (long long i = lo; i < hi; ++i) {
    const int n = (int)(i - lo), st = n % kStages;
    while (pre[u + 1] <= i) ++u;
    const int b = u / D.Hkv, g = u % D.Hkv;
    if (u != u_loaded) {  // a new unit starts: its geometry and queries, fresh softmax state
      u_loaded = u;
      u_t = seq_qfirst(S, b);
      u_nc = (u_t + 1) / D.B;
      u_nsel = min(u_nc, D.k);
      const __nv_bfloat16 *qrow = P.q + (((size_t)b * S.n_q) * D.Hq + (size_t)g * G + head) * kD;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int c0 = kk * 16 + 2 * (lane & 3);
        if (head < G) {
          qa[kk][0] = *(const uint32_t *)(qrow + c0);
          qa[kk][1] = *(const uint32_t *)(qrow + c0 + 8);
        } else {
          qa[kk][0] = qa[kk][1] = 0u;
        }
      }
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    }
    const int j_item = (int)(i - pre[u]);
    const int nk = j_item < u_nsel ? kBlk : u_t + 1 - u_nc * D.B;  // valid keys of this block
    const bool got = mbar_wait(&full[st], (n / kStages) & 1, kWaitNs);
    if (!__all_sync(0xffffffffu, got) && lane == 0) s_fail = 1;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (s_fail) {  // every compute warp sees the same flag after the barrier and leaves together
      fail = true;
      break;
    }
    uint8_t *kd = ring + st * 2 * kTileBytes, *vd = kd + kTileBytes;
    if (nk < kBlk) {
      for (int e = threadIdx.x; e < (kBlk - nk) * 16; e += kWarps * 32) {
        const int rr = nk + e / 16, cc = e % 16;
        *(uint4 *)(vd + (cc >> 3) * (kTileBytes / 2) + rr * 128 + ((cc & 7) << 4)) = make_uint4(0, 0, 0, 0);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    const uint32_t kb = smem_u32(kd), vb = smem_u32(vd);
    const int r0 = warp * 16;
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int half = kk >> 2;
      const int mtx = lane >> 3, rr = lane & 7;
      const int key = r0 + (mtx >> 1) * 8 + rr;
      const int chunk = (kk & 3) * 2 + (mtx & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + half * (kTileBytes / 2) + sw128(key, chunk), b0, b1, b2, b3);
      mma16816(sacc[0], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
      mma16816(sacc[1], qa[kk][0], 0u, qa[kk][1], 0u, b2, b3);
    }
    float x[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = r0 + nt * 8 + 2 * (lane & 3) + e;
        x[nt * 2 + e] = key < nk ? sacc[nt][e] * sl2 : -INFINITY;
      }
    float cmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
    const float m_new = fmaxf(m, cmax);
    const float corr = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = (x[e] == -INFINITY) ? 0.f : ex2_approx(x[e] - m_new);
    float ps = (p[0] + p[1]) + (p[2] + p[3]);
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l = l * corr + ps;
    m = m_new;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= corr;
      o[nt][1] *= corr;
    }
    const uint32_t pa0 = pack_bf16x2(p[0], p[1]);
    const uint32_t pa2 = pack_bf16x2(p[2], p[3]);
#pragma unroll
    for (int nt2 = 0; nt2 < 8; ++nt2) {
      const int mtx = lane >> 3, rr = lane & 7;
      const int key = r0 + (mtx & 1) * 8 + rr;
      const int dim_chunk = nt2 * 2 + (mtx >> 1);
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(vb + (dim_chunk >> 3) * (kTileBytes / 2) + sw128(key, dim_chunk & 7), v0, v1, v2, v3);
      mma16816(o[2 * nt2], pa0, 0u, pa2, 0u, v0, v1);
      mma16816(o[2 * nt2 + 1], pa0, 0u, pa2, 0u, v2, v3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);

    const bool unit_end = (i + 1 == pre[u + 1]) || (i + 1 == hi);
    if (!unit_end) continue;
    // ---- flush this unit's segment: merge the warps, write the partial to slot (u + c)
    if ((lane & 3) == 0 && head < kMaxG) {
      wm[warp * 8 + head] = m;
      wl[warp * 8 + head] = l;
    }
    if (head < kMaxG) {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int dcol = nt * 8 + 2 * (lane & 3);
        wo[(warp * 8 + head) * kD + dcol] = o[nt][0];
        wo[(warp * 8 + head) * kD + dcol + 1] = o[nt][1];
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const size_t slot = (size_t)u + c;
    float *dst = P.part + slot * G * kD;
    float *dst_ml = P.part_ml + slot * G * 2;
    for (int e = threadIdx.x; e < G * kD; e += kWarps * 32) {
      const int hh = e / kD, dd = e % kD;
      float mm = -INFINITY;
      for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, wm[w * 8 + hh]);
      float acc = 0.f, ll = 0.f;
      for (int w = 0; w < kWarps; ++w) {
        const float f = (wm[w * 8 + hh] == -INFINITY) ? 0.f : ex2_approx(wm[w * 8 + hh] - mm);
        acc += f * wo[(w * 8 + hh) * kD + dd];
        ll += f * wl[w * 8 + hh];
      }
      dst[e] = acc;
      if (dd == 0) {
        dst_ml[hh * 2] = mm;
        dst_ml[hh * 2 + 1] = ll;
      }
    }
    const int c_first = cta_of(pre[u], C, T), c_last = cta_of(pre[u + 1] - 1, C, T);
    const int n_parts = c_last - c_first + 1;
    // The barrier orders this CTA's partial writes before thread 0's release on
    // the unit counter; the CTA that brings the count to n_parts acquires the
    // other parts' writes and, after the next barrier, all its threads read them.
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 0) {
      int old;
      asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(old) : "l"(&P.done[u]) : "memory");
      s_last = old == n_parts - 1;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (s_last) {
      // O = sum_p 2^(m_p - m) O_p / sum_p 2^(m_p - m) l_p, merged part by part
      // with a running max; each thread reads the (m, l) of its head and its O
      // slice of every part at once (one round trip to L2)
      const float *ml = P.part_ml + ((size_t)u + c_first) * G * 2;
      const float4 *src = (const float4 *)(P.part + ((size_t)u + c_first) * G * kD);
      __nv_bfloat16 *orow = P.out + ((size_t)b * S.n_q * D.Hq + (size_t)g * G) * kD;
      for (int e4 = threadIdx.x; e4 < G * kD / 4; e4 += kWarps * 32) {
        const int hh = (e4 * 4) / kD;
        float m_run = -INFINITY, l_run = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int pp = 0; pp < n_parts; ++pp) {
          const float ms = __ldcg(&ml[(pp * G + hh) * 2]), ls = __ldcg(&ml[(pp * G + hh) * 2 + 1]);
          const float4 o4 = __ldcg(&src[(size_t)pp * (G * kD / 4) + e4]);
          if (ms == -INFINITY) continue;  // a part that saw no key of this head
          const float m_new = fmaxf(m_run, ms);
          const float a = ex2_approx(m_run - m_new), f = ex2_approx(ms - m_new);
          acc.x = fmaf(f, o4.x, acc.x * a);
          acc.y = fmaf(f, o4.y, acc.y * a);
          acc.z = fmaf(f, o4.z, acc.z * a);
          acc.w = fmaf(f, o4.w, acc.w * a);
          l_run = fmaf(f, ls, l_run * a);
          m_run = m_new;
        }
        const float il = l_run > 0.f ? 1.f / l_run : 0.f;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * il, acc.y * il);
        pk.y = pack_bf16x2(acc.z * il, acc.w * il);
        *(uint2 *)(orow + e4 * 4) = pk;
      }
      if (threadIdx.x == 0) P.done[u] = 0;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  if (fail) record_status(P.status, QSA_ERR_TIMEOUT);
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

bool make_kv_map(CUtensorMap *m, const void *ptr, const Dims &D, const Seqs &S) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)S.kv_cap, (cuuint64_t)S.batch * D.Hkv};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)S.kv_cap * kD * 2};
  cuuint32_t box[3] = {64, kBlk, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int max_splits_for(const Dims &D) { return (D.k + 1 + kItems - 1) / kItems; }

}  // namespace

bool attn_decode_supported(const Dims &D) { return D.bf16 && D.d == kD && D.B == kBlk && D.G <= kMaxG; }

// Workspace: [batch][Hkv] int unit counters (rounded up to 256 bytes), then fp32
// partial outputs [slots][G][d], then their (m, l) pairs [slots][G][2]. The split
// kernel uses batch * Hkv * max_splits slots; the persistent kernel n_units + C,
// C <= kMaxCtas.
constexpr int kMaxCtas = 1024;
size_t counters_bytes(const Dims &D, const Seqs &S) {
  return (((size_t)S.batch * D.Hkv * sizeof(int)) + 255) & ~(size_t)255;
}
bool use_persistent(const Dims &D, const Seqs &S) { return (long long)S.batch * D.Hkv <= kMaxUnits; }
size_t partial_slots(const Dims &D, const Seqs &S) {
  return use_persistent(D, S) ? (size_t)S.batch * D.Hkv + kMaxCtas
                              : (size_t)S.batch * D.Hkv * max_splits_for(D);
}
size_t partial_o_bytes(const Dims &D, const Seqs &S) { return partial_slots(D, S) * D.G * kD * sizeof(float); }
size_t attn_decode_workspace(const Dims &D, const Seqs &S) {
  return counters_bytes(D, S) + partial_o_bytes(D, S) + partial_slots(D, S) * D.G * 2 * sizeof(float);
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n[dev] = 148;
  return n[dev];
}

cudaError_t launch_attn_decode(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                               const int32_t *sel, void *out, void *scratch, size_t scratch_bytes, int *status,
                               cudaStream_t st, bool pdl) {
  if (!attn_decode_supported(D) || S.n_q != 1) return cudaErrorNotSupported;
  if (S.batch == 0) return cudaSuccess;
  if (scratch_bytes < attn_decode_workspace(D, S)) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_kv_map(&tk, k, D, S) || !make_kv_map(&tv, v, D, S)) return cudaErrorInvalidValue;
  if (use_persistent(D, S)) {
    PstParams Q;
    Q.D = D;
    Q.S = S;
    Q.q = (const __nv_bfloat16 *)q;
    Q.sel = sel;
    Q.out = (__nv_bfloat16 *)out;
    Q.done = (int *)scratch;
    Q.part = (float *)((char *)scratch + counters_bytes(D, S));
    Q.part_ml = (float *)((char *)scratch + counters_bytes(D, S) + partial_o_bytes(D, S));
    Q.n_units = S.batch * D.Hkv;
    Q.C = min(sm_count(), kMaxCtas);
    Q.status = status;
    const size_t smem = 1024 + (size_t)kStages * 2 * kTileBytes + 2 * kStages * 8 +
                        sizeof(float) * (2 * kWarps * 8 + kWarps * 8 * kD) +
                        sizeof(int) * (Q.n_units + 1);
    cudaError_t e = ensure_smem(k_attn_decode_pst, smem);
    if (e != cudaSuccess) return e;
    note_launch();
    // With pdl, a programmatic dependent launch: the kernel may start while the
    // previous kernel in the stream finishes; it waits for that kernel's results
    // (griddepcontrol.wait) after its prologue. Without it, griddepcontrol.wait
    // returns at once.
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(Q.C);
    lc.blockDim = dim3(kPThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&lc, k_attn_decode_pst, tk, tv, Q);
  }
  DecParams P;
  P.D = D;
  P.S = S;
  P.q = (const __nv_bfloat16 *)q;
  P.sel = sel;
  P.out = (__nv_bfloat16 *)out;
  P.done = (int *)scratch;
  P.part = (float *)((char *)scratch + counters_bytes(D, S));
  P.part_ml = (float *)((char *)scratch + counters_bytes(D, S) + partial_o_bytes(D, S));
  P.max_splits = max_splits_for(D);
  P.status = status;
  static_assert(sizeof(float) * (2 * kWarps * 8 + kWarps * 8 * kD) <= 2 * kItems * kTileBytes, "merge scratch");
  const size_t smem = 1024 + 2 * kItems * kTileBytes + 64;
  cudaError_t e = ensure_smem(k_attn_decode, smem);
  if (e != cudaSuccess) return e;
  note_launch();
  k_attn_decode<<<dim3(P.max_splits, D.Hkv, S.batch), kThreads, smem, st>>>(tk, tv, P);
  return cudaGetLastError();
}

}  // namespace qsa

// ---------------------------------------------------------------------------
// Decode attention without a caller workspace.
//
// Some callers cannot hand this library any device memory beyond their inputs
// and outputs: for example a plugin that a host framework invokes with only its
// input and output buffers, or a serving process whose device memory is all
// reserved up front by its own pool, so that a cudaMalloc would fail or bypass
// that pool. For them this entry point keeps the split partials of the decode
// kernel in a fixed array in the library's device memory instead of a workspace.
// ---------------------------------------------------------------------------
namespace {

// Status word and split partials of qsa_sparse_attn_decode_noalloc: every GPU that
// loads the library holds this array until the process exits. Layout: [0, 256) the
// status word the decode kernels record a timed-out wait in, then the decode
// workspace (unit counters, then the partials).
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" qsa_status_t qsa_sparse_attn_decode_noalloc(const qsa_config_t *cfg, const void *q, const void *k,
                                                       const void *v, const int32_t *sel,
                                                       const int32_t *kv_start, const int32_t *kv_len,
                                                       int32_t batch, int32_t kv_cap, void *out,
                                                       qsa_stream_t stream) {
  using namespace qsa;
  Dims D;
  qsa_status_t s = resolve_config(cfg, &D);
  if (s != QSA_OK) return s;
  if (batch < 0 || kv_cap < 0) return QSA_ERR_INVALID_ARG;
  if (batch == 0) return QSA_OK;
  if (!q || !k || !v || !sel || !kv_start || !kv_len || !out) return QSA_ERR_INVALID_ARG;
  const void *ptrs[] = {q, k, v, sel, out};
  for (const void *p : ptrs)
    if (((uintptr_t)p & 15u) != 0) return QSA_ERR_INVALID_ARG;
  if (!attn_decode_supported(D)) return QSA_ERR_UNSUPPORTED;
  Seqs S;
  S.kv_start = kv_start;
  S.kv_len = kv_len;
  S.q_first = nullptr;  // the query of sequence b sits at kv_len[b] - 1
  S.batch = batch;
  S.n_q = 1;
  S.kv_cap = kv_cap;
  S.nb_cap = kv_cap / D.B;
  const size_t need = kStatusBytes + attn_decode_workspace(D, S);
  if (need > (size_t)QSA_NOALLOC_SCRATCH_BYTES) {
    char what[160];
    snprintf(what, sizeof what, "decode partials need %zu bytes, more than the %d-byte static scratch", need,
             (int)QSA_NOALLOC_SCRATCH_BYTES);
    note_error(what, cudaErrorInvalidValue);
    return QSA_ERR_UNSUPPORTED;
  }
  // In host code the array's name only stands in for it; its device address on the
  // current device comes from the runtime. The lookup is made on every call (a
  // host-side table lookup once the module is loaded), so that an address is never
  // reused after the device's context was torn down and the module loaded again.
  void *arr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&arr, g_noalloc_scratch);
  if (e != cudaSuccess) {
    note_error("cudaGetSymbolAddress of the static decode scratch", e);
    return QSA_ERR_CUDA;
  }
  // Clear the status word and the unit counters, ordered before the kernel on the
  // stream: a call whose bounded wait ran out leaves counters set, and this keeps
  // that from reaching any later call.
  e = cudaMemsetAsync(arr, 0, kStatusBytes + counters_bytes(D, S), (cudaStream_t)stream);
  if (e != cudaSuccess) {
    note_error("qsa_sparse_attn_decode_noalloc: clearing the static scratch", e);
    return QSA_ERR_CUDA;
  }
  e = launch_attn_decode(D, S, q, k, v, sel, out, (char *)arr + kStatusBytes, need - kStatusBytes, (int *)arr,
                         (cudaStream_t)stream);
  if (e != cudaSuccess) {
    note_error("qsa_sparse_attn_decode_noalloc launch", e);
    return e == cudaErrorNotSupported ? QSA_ERR_UNSUPPORTED : QSA_ERR_CUDA;
  }
  return QSA_OK;
}
