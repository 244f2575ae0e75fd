// CUDA-core kernels of the QSA path: block compression, fp32 scoring with exact
// top-k selection, a CUDA-core attention kernel (fp32 config and shapes the
// tensor-core kernel does not take) and the decode prologue.
//
// Definitions: Hugging Face Transformers model doc "Qwen4-Exp", intro paragraph
// on QSA and Qwen4ExpTextConfig indexer_* parameters (see include/qsa.h).
#include <math.h>

#include "qsa_internal.h"
#include "qsa_rowselect.cuh"

namespace qsa {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}

// ---------------------------------------------------------------------------
// Step 1: block compression. One warp per (sequence, block); each lane owns
// adjacent column pairs, so one load instruction of the warp reads a whole
// 128-byte row (di = 64, bf16), and up to 64 rows are in flight before any is added.
// kbar[b][j][c] = (sum_{u<B} ki[start + jB + u][c]) / B, summed in key order.
// ---------------------------------------------------------------------------
template <typename T> struct Pair;
template <> struct Pair<__nv_bfloat16> {
  typedef __nv_bfloat162 type;
  __device__ static float lo(type v) { return __low2float(v); }
  __device__ static float hi(type v) { return __high2float(v); }
};
template <> struct Pair<float> {
  typedef float2 type;
  __device__ static float lo(type v) { return v.x; }
  __device__ static float hi(type v) { return v.y; }
};

constexpr int kCompressWarps = 8;  // warps per CTA (2 per CTA measured slower at 8K)

template <typename T>
__global__ void __launch_bounds__(kCompressWarps * 32)
k_compress(Dims D, Seqs S, const T *__restrict__ ki, const int32_t *__restrict__ blocks_done,
           float *__restrict__ kbar, int32_t *__restrict__ blocks_out, int *status) {
  typedef typename Pair<T>::type P2;
  constexpr int kRows = sizeof(T) == 2 ? 64 : 32;  // rows loaded before they are summed
  // a programmatic dependent (qsa_forward's next stage) may start its prologue now;
  // it waits for this grid before it reads k̄
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!seq_ok(S, b, status)) return;
  const int start = seq_start(S, b), len = S.kv_len[b];
  const int hi = len / D.B;
  if (blocks_out && blockIdx.x == 0 && threadIdx.x == 0) blocks_out[b] = hi;
  const int lo = blocks_done ? max(blocks_done[b], 0) : 0;
  const int pairs = D.di / 2;
  for (int j = lo + blockIdx.x * kCompressWarps + warp; j < hi; j += gridDim.x * kCompressWarps) {
    const P2 *src = (const P2 *)(ki + ((size_t)b * S.kv_cap + start + (size_t)j * D.B) * D.di);
    float *dst = kbar + ((size_t)b * S.nb_cap + j) * D.di;
    for (int cp = lane; cp < pairs; cp += 32) {
      float a0 = 0.f, a1 = 0.f;
      for (int u0 = 0; u0 < D.B; u0 += kRows) {
        P2 v[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
          if (u0 + u < D.B) v[u] = src[(size_t)(u0 + u) * pairs + cp];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
          if (u0 + u < D.B) {
            a0 += Pair<T>::lo(v[u]);
            a1 += Pair<T>::hi(v[u]);
          }
      }
      dst[2 * cp] = a0 / (float)D.B;
      dst[2 * cp + 1] = a1 / (float)D.B;
    }
  }
}

// ---------------------------------------------------------------------------
// Steps 2+3 on CUDA cores. A CTA holds `warps` consecutive query rows of one
// sequence, one warp per row. Compressed keys stream through shared memory in
// chunks of 32 blocks shared by all rows; each lane scores one block:
//   s_j = sum_h max(0, qi[h] . kbar[j])    (fp32, dot in index order)
// Selection is an exact radix select on the fp32 bit patterns (scores are >= +0,
// so the bit order is the value order): the k-th largest key tau is found bit by
// bit, then blocks with key > tau are kept together with the lowest-index blocks
// whose key equals tau -- the (-score, index) order with ties to the lower index.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_score_topk_simt(Dims D, Seqs S, const T *__restrict__ qi,
                                  const float *__restrict__ kbar, int32_t *__restrict__ sel,
                                  int *status, int warps, int nc_cap, float *__restrict__ scores_out) {
  extern __shared__ float smem[];
  const int HD = D.Hi * D.di;
  float *qi_s = smem;                                  // [warps][Hi*di]
  float *kb_s = qi_s + warps * HD;                     // [32][di+1]
  uint32_t *sc_s = (uint32_t *)(kb_s + 32 * (D.di + 1));  // [warps][nc_cap]
  __shared__ int s_ncmax;

  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * warps + warp;
  const bool ok = seq_ok(S, b, status);
  const int len = ok ? S.kv_len[b] : 0;
  const int t = (r < S.n_q) ? seq_qfirst(S, b) + r : -1;
  const bool valid = ok && r < S.n_q && t >= 0 && t < len;
  const int n_c = valid ? (t + 1) / D.B : 0;

  if (threadIdx.x == 0) s_ncmax = 0;
  if (valid) {
    const T *src = qi + ((size_t)b * S.n_q + r) * HD;
    for (int i = lane; i < HD; i += 32) qi_s[warp * HD + i] = to_f(src[i]);
  }
  __syncthreads();
  if (lane == 0 && n_c > 0) atomicMax(&s_ncmax, n_c);
  __syncthreads();
  const int nc_max = s_ncmax;
  uint32_t *keys = sc_s + (size_t)warp * nc_cap;

  for (int j0 = 0; j0 < nc_max; j0 += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * D.di; i += blockDim.x) {
      const int jj = i / D.di, c = i - jj * D.di, j = j0 + jj;
      kb_s[jj * (D.di + 1) + c] = (j < nc_max) ? kbar[((size_t)b * S.nb_cap + j) * D.di + c] : 0.f;
    }
    __syncthreads();
    const int j = j0 + lane;
    if (j < n_c) {
      float s = 0.f;
      const float *kr = kb_s + lane * (D.di + 1);
      for (int h = 0; h < D.Hi; ++h) {
        const float *qh = qi_s + warp * HD + h * D.di;
        float dot = 0.f;
        for (int c = 0; c < D.di; ++c) dot = fmaf(qh[c], kr[c], dot);
        s += dot > 0.f ? dot : 0.f;
      }
      keys[j] = __float_as_uint(s);
      if (scores_out) scores_out[((size_t)b * S.n_q + r) * S.nb_cap + j] = s;
    }
  }
  __syncwarp();
  if (r >= S.n_q || scores_out) return;  // with scores_out: scores only, no selection
  int32_t *out = sel + ((size_t)b * S.n_q + r) * D.k;
  if (!valid || n_c <= D.k) {
    for (int i = lane; i < D.k; i += 32) out[i] = (i < n_c) ? i : -1;
    return;
  }
  uint32_t prefix = 0;
  int remaining = D.k;
  for (int bit = 30; bit >= 0; --bit) {
    const uint32_t want = (prefix >> bit) | 1u;
    int cnt = 0;
    for (int j = lane; j < n_c; j += 32) cnt += ((keys[j] >> bit) == want);
    cnt = __reduce_add_sync(kFull, cnt);
    if (cnt >= remaining) prefix |= (1u << bit);
    else remaining -= cnt;
  }
  int base = 0, tie_base = 0;
  const unsigned lt = lanemask_lt();
  for (int j0 = 0; j0 < n_c; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < n_c ? keys[j] : 0u;
    const bool gt = j < n_c && key > prefix;
    const bool eq = j < n_c && key == prefix;
    const unsigned eq_mask = __ballot_sync(kFull, eq);
    const bool take = gt || (eq && tie_base + __popc(eq_mask & lt) < remaining);
    const unsigned take_mask = __ballot_sync(kFull, take);
    if (take) out[base + __popc(take_mask & lt)] = j;
    base += __popc(take_mask);
    tie_base += __popc(eq_mask);
  }
}

// ---------------------------------------------------------------------------
// Steps 2+3 with one CTA per query row (few rows, e.g. a decode step): the row's
// candidates are spread over all threads, and the same exact radix select runs
// with block-wide counts; selected ids are written in ascending order.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 512;

// Decode prologue for sequence b, run by one CTA: append the new token at L-1
// and, if that completes block j = L/B - 1, compress it and advance kbar_blocks.
// The indexer state must be in step (kbar_blocks == (L-1)/B; larger means the
// cache was cropped, which QSA does not support). Every thread reads the sequence
// state itself, and the new rows are loaded before anything waits on it, so the
// global reads of the prologue overlap. A completed block's k̄ row is also left in
// `kbar_new` (shared) for the scoring that follows in the same kernel; the caller
// synchronises the CTA before reading it. Returns the completed block, or -1.
template <typename T>
__device__ int decode_append_row(const Dims &D, const Seqs &S, const DecodeAppend &A, float *kbar, int b,
                                 int *status, float *kbar_new) {
  T *k_cache = (T *)A.k_cache, *v_cache = (T *)A.v_cache, *ki_cache = (T *)A.ki_cache;
  const T *k_new = (const T *)A.k_new, *v_new = (const T *)A.v_new, *ki_new = (const T *)A.ki_new;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int HD = D.Hkv * D.d;
  // the first two elements of this thread's share of the new K/V rows and its
  // element of the new indexer key, in flight with the state loads
  T kn0 = T(), vn0 = T(), kn1 = T(), vn1 = T(), kin = T();
  if (tid < HD) {
    kn0 = k_new[(size_t)b * HD + tid];
    vn0 = v_new[(size_t)b * HD + tid];
  }
  if (tid + nt < HD) {
    kn1 = k_new[(size_t)b * HD + tid + nt];
    vn1 = v_new[(size_t)b * HD + tid + nt];
  }
  if (tid < D.di) kin = ki_new[(size_t)b * D.di + tid];
  const int start = seq_start(S, b), L = S.kv_len[b], have = A.kbar_blocks[b];
  const bool geo = start >= 0 && L >= 1 && (long long)start + L <= (long long)S.kv_cap;
  const int need = geo ? (L - 1) / D.B : 0;
  if (tid == 0) {
    if (!geo) record_status(status, QSA_ERR_DEVICE_CHECK);
    else if (have != need) record_status(status, have > need ? QSA_ERR_UNSUPPORTED : QSA_ERR_DEVICE_CHECK);
  }
  if (!geo || have != need) return -1;
  const size_t pos = (size_t)start + L - 1;
  auto put = [&](int i, T kv, T vv) {
    const int g = i / D.d, c = i - g * D.d;
    const size_t dst = (((size_t)b * D.Hkv + g) * S.kv_cap + pos) * D.d + c;
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  };
  if (tid < HD) put(tid, kn0, vn0);
  if (tid + nt < HD) put(tid + nt, kn1, vn1);
  for (int i = tid + 2 * nt; i < HD; i += nt) put(i, k_new[(size_t)b * HD + i], v_new[(size_t)b * HD + i]);
  for (int c = tid; c < D.di; c += nt)
    ki_cache[((size_t)b * S.kv_cap + pos) * D.di + c] = c == tid ? kin : ki_new[(size_t)b * D.di + c];
  if (L % D.B != 0) return -1;
  // the new token completes block j: its mean, rows in key order, the last one
  // being the token just appended (taken from ki_new rather than re-read)
  const int j = L / D.B - 1;
  const T *src = ki_cache + ((size_t)b * S.kv_cap + start + (size_t)j * D.B) * D.di;
  for (int c = tid; c < D.di; c += nt) {
    float acc = 0.f;
    for (int u = 0; u < D.B - 1; ++u) acc += to_f(src[(size_t)u * D.di + c]);
    acc += to_f(c == tid ? kin : ki_new[(size_t)b * D.di + c]);
    const float m = acc / (float)D.B;
    kbar[((size_t)b * S.nb_cap + j) * D.di + c] = m;
    kbar_new[c] = m;
  }
  if (tid == 0) A.kbar_blocks[b] = L / D.B;
  return j;
}

template <typename T, bool kAppend>
__global__ void __launch_bounds__(kRowThreads)
k_score_topk_row(Dims D, Seqs S, const T *__restrict__ qi, const float *kbar, int32_t *__restrict__ sel,
                 int *status, DecodeAppend A) {
  extern __shared__ float smem[];
  // The decode attention kernel that follows is launched as a programmatic
  // dependent: let it start its prologue now; it waits for this grid's completion
  // before it reads anything this kernel writes.
  if (kAppend) asm volatile("griddepcontrol.launch_dependents;");
  const int HD = D.Hi * D.di;
  float *qi_s = smem;                               // [Hi*di]
  float *kbar_new = qi_s + HD;                      // [di]: k̄ of a block completed by the append
  uint32_t *keys = (uint32_t *)(kbar_new + D.di);   // [nb_cap]
  __shared__ int red[kRowThreads / 32];
  __shared__ int wbase[kRowThreads / 32 + 1];
  const int r = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Loads that depend on nothing are issued first: the query's indexer row and
  // the sequence state. As soon as the length is known every thread prefetches
  // the k̄ rows of its candidates into L2, so that those DRAM reads are in flight
  // during the decode append and the barrier below.
  const T *src = qi + ((size_t)b * S.n_q + r) * HD;
  const T q0 = tid < HD ? src[tid] : T();
  const int start0 = seq_start(S, b), len0 = S.kv_len[b], t = seq_qfirst(S, b) + r;
  const bool geo = start0 >= 0 && len0 >= 0 && (long long)start0 + len0 <= (long long)S.kv_cap;
  const bool valid = geo && t >= 0 && t < len0;
  const int n_c = valid ? (t + 1) / D.B : 0;
  const float *kb = kbar + (size_t)b * S.nb_cap * D.di;
  if (n_c > D.k)
    for (int j = tid; j < n_c; j += kRowThreads)
      for (int o = 0; o < D.di * 4; o += 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"((const char *)(kb + (size_t)j * D.di) + o));
  const int j_new = kAppend ? decode_append_row<T>(D, S, A, (float *)kbar, b, status, kbar_new) : -1;
  if (tid < HD) qi_s[tid] = to_f(q0);
  for (int i = tid + kRowThreads; i < HD; i += kRowThreads) qi_s[i] = to_f(src[i]);
  seq_ok(S, b, tid == 0 ? status : nullptr);  // records a bad geometry
  int32_t *out = sel + ((size_t)b * S.n_q + r) * D.k;
  if (n_c <= D.k) {
    for (int i = tid; i < D.k; i += kRowThreads) out[i] = (i < n_c) ? i : -1;
    return;
  }
  __syncthreads();
  for (int j = tid; j < n_c; j += kRowThreads) {
    const float4 *kr = (const float4 *)(j == j_new ? kbar_new : kb + (size_t)j * D.di);
    keys[j] = __float_as_uint(block_score_fp32(qi_s, D.Hi, D.di, kr));
  }
  __syncthreads();
  // Radix select of the k-th largest key, 8 bits at a time from the top: count the
  // keys that match the prefix found so far per value of the next byte, then keep
  // the byte at which the running count from the top reaches `remaining`.
  __shared__ int hist[256];
  __shared__ int s_digit, s_above, s_cnt, s_ncand;
  __shared__ uint32_t s_cand[32], s_val;
  __shared__ unsigned s_min, s_max;
  // Bits above the highest one in which the row's keys differ are common to all
  // keys: the radix passes start below them, 8 bits at a time, so that no pass
  // piles every key into one histogram bin.
  if (tid == 0) {
    s_min = 0xffffffffu;
    s_max = 0u;
  }
  __syncthreads();
  {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j = tid; j < n_c; j += kRowThreads) {
      kmin = min(kmin, keys[j]);
      kmax = max(kmax, keys[j]);
    }
    kmin = __reduce_min_sync(kFull, kmin);
    kmax = __reduce_max_sync(kFull, kmax);
    if (lane == 0) {
      atomicMin(&s_min, kmin);
      atomicMax(&s_max, kmax);
    }
  }
  __syncthreads();
  const uint32_t diff = s_min ^ s_max;
  const int top = diff ? 31 - __clz(diff) : -1;
  uint32_t pmask = top >= 31 ? 0u : (0xffffffffu << (top + 1));
  uint32_t prefix = s_max & pmask;
  int remaining = D.k;
  for (int hi_bit = top; hi_bit >= 0; hi_bit -= 8) {
    const int shift = hi_bit >= 7 ? hi_bit - 7 : 0;
    const uint32_t dmask = (2u << (hi_bit - shift)) - 1u;
    for (int i = tid; i < 256; i += kRowThreads) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n_c; j += kRowThreads) {
      const uint32_t key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns digits 255-8L .. 248-8L (descending)
      int c[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * lane - q];
        tot += c[q];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - tot;  // keys in higher digits than this lane's range
      if (excl < remaining && incl >= remaining) {
        int above = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (above + c[q] >= remaining) {
            s_digit = 255 - 8 * lane - q;
            s_above = above;
            s_cnt = c[q];
            break;
          }
          above += c[q];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    pmask |= dmask << shift;
    remaining -= s_above;
    const int cnt = s_cnt;
    __syncthreads();
    if (shift > 0 && cnt <= 32) {
      // The k-th largest key lies among the at most 32 keys still matching the
      // prefix: gather them, sort them across warp 0 (bitonic, descending) and read
      // the remaining-th; the keys above it among them leave `remaining` ties.
      if (tid == 0) s_ncand = 0;
      __syncthreads();
      for (int j = tid; j < n_c; j += kRowThreads) {
        const uint32_t key = keys[j];
        if ((key & pmask) == prefix) s_cand[atomicAdd(&s_ncand, 1)] = key;
      }
      __syncthreads();
      if (warp == 0) {
        const int nc = s_ncand;
        uint32_t v = lane < nc ? s_cand[lane] : 0u;
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(kFull, v, stride);
            const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0 || size == 32);
            v = keep_max ? max(v, o) : min(v, o);
          }
        }
        const uint32_t val = __shfl_sync(kFull, v, remaining - 1);
        const int gt = __popc(__ballot_sync(kFull, lane < nc && v > val));
        if (lane == 0) {
          s_val = val;
          s_above = gt;
        }
      }
      __syncthreads();
      prefix = s_val;
      pmask = 0xffffffffu;
      remaining -= s_above;
      __syncthreads();
      break;
    }
  }
  // ascending compaction: chunks of kRowThreads consecutive ids in thread order
  const unsigned lt = lanemask_lt();
  int base = 0, tie_base = 0;
  for (int j0 = 0; j0 < n_c; j0 += kRowThreads) {
    const int j = j0 + tid;
    const uint32_t key = j < n_c ? keys[j] : 0u;
    const bool gt = j < n_c && key > prefix;
    const bool eq = j < n_c && key == prefix;
    // ranks of the ties in id order decide which ties are kept
    const unsigned eq_mask = __ballot_sync(kFull, eq);
    __syncthreads();
    if (lane == 0) red[warp] = __popc(eq_mask);
    __syncthreads();
    int eq_before = tie_base;
    for (int w = 0; w < warp; ++w) eq_before += red[w];
    int eq_tot = 0;
    for (int w = 0; w < kRowThreads / 32; ++w) eq_tot += red[w];
    const bool take = gt || (eq && eq_before + __popc(eq_mask & lt) < remaining);
    const unsigned take_mask = __ballot_sync(kFull, take);
    if (lane == 0) wbase[warp] = __popc(take_mask);
    __syncthreads();
    int take_before = base;
    for (int w = 0; w < warp; ++w) take_before += wbase[w];
    int take_tot = 0;
    for (int w = 0; w < kRowThreads / 32; ++w) take_tot += wbase[w];
    if (take) out[take_before + __popc(take_mask & lt)] = j;
    base += take_tot;
    tie_base += eq_tot;
  }
}

// ---------------------------------------------------------------------------
// Step 4 on CUDA cores. One CTA per (query row, KV head, sequence); one warp per
// query head of the group. Keys stream in chunks of 32 through shared memory
// (selected blocks in ascending order, then the trailing range); each warp keeps
// an online softmax (running max m, sum l, fp32 output in registers).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_attn_simt(Dims D, Seqs S, const T *__restrict__ q, const T *__restrict__ k,
                            const T *__restrict__ v, const int32_t *__restrict__ sel,
                            T *__restrict__ out, int *status) {
  extern __shared__ float smem[];
  const int d = D.d;
  float *q_s = smem;                 // [G][d]
  float *k_s = q_s + D.G * d;        // [32][d+1]
  float *v_s = k_s + 32 * (d + 1);   // [32][d]
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = g * D.G + warp;
  const bool ok = seq_ok(S, b, status);
  const int len = ok ? S.kv_len[b] : 0;
  const int start = ok ? seq_start(S, b) : 0;
  const int t = seq_qfirst(S, b) + r;
  T *o_row = out + (((size_t)b * S.n_q + r) * D.Hq + h) * d;
  if (!ok || t < 0 || t >= len) {
    for (int c = lane; c < d; c += 32) o_row[c] = from_f<T>(0.f);
    return;
  }
  const T *q_row = q + (((size_t)b * S.n_q + r) * D.Hq + h) * d;
  for (int c = lane; c < d; c += 32) q_s[warp * d + c] = to_f(q_row[c]);
  const size_t plane = ((size_t)b * D.Hkv + g) * S.kv_cap + start;
  const T *kb = k + plane * d;
  const T *vb = v + plane * d;
  const int32_t *srow = sel + ((size_t)b * S.n_q + r) * D.k;
  const int n_c = (t + 1) / D.B;

  float m = -INFINITY, l = 0.f;
  float o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0.f;

  for (int s = 0; s <= D.k; ++s) {
    int lo, hi;
    if (s < D.k) {
      const int blk = srow[s];
      if (blk < 0 || blk >= n_c) continue;
      lo = blk * D.B;
      hi = lo + D.B;
    } else {
      lo = n_c * D.B;
      hi = t + 1;
    }
    for (int c0 = lo; c0 < hi; c0 += 32) {
      const int nk = min(32, hi - c0);
      __syncthreads();
      for (int i = threadIdx.x; i < nk * d; i += blockDim.x) {
        const int u = i / d, c = i - u * d;
        k_s[u * (d + 1) + c] = to_f(kb[(size_t)(c0 + u) * d + c]);
        v_s[u * d + c] = to_f(vb[(size_t)(c0 + u) * d + c]);
      }
      __syncthreads();
      float logit = -INFINITY;
      if (lane < nk) {
        float dot = 0.f;
        const float *kr = k_s + lane * (d + 1);
        const float *qr = q_s + warp * d;
        for (int c = 0; c < d; ++c) dot = fmaf(qr[c], kr[c], dot);
        logit = dot * D.scale;
      }
      const float m_new = fmaxf(m, warp_max(logit));
      const float corr = expf(m - m_new);
      const float p = lane < nk ? expf(logit - m_new) : 0.f;
      l = l * corr + warp_sum(p);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] *= corr;
      for (int u = 0; u < nk; ++u) {
        const float pu = __shfl_sync(kFull, p, u);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (lane + 32 * i < d) o[i] = fmaf(pu, v_s[u * d + lane + 32 * i], o[i]);
      }
      m = m_new;
    }
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i < d) o_row[lane + 32 * i] = from_f<T>(o[i] * inv);
}

// ---------------------------------------------------------------------------
// Decode prologue, one CTA per sequence: check the indexer state is in step
// with the cache (kbar_blocks == (L-1)/B; a larger value means the cache was
// cropped, which QSA does not support), append the new token at L-1, and if
// that completes block j = L/B - 1, compress it and advance kbar_blocks.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
k_decode_append(Dims D, Seqs S, T *__restrict__ k_cache, T *__restrict__ v_cache,
                T *__restrict__ ki_cache, float *__restrict__ kbar, int32_t *__restrict__ kbar_blocks,
                const T *__restrict__ k_new, const T *__restrict__ v_new,
                const T *__restrict__ ki_new, int *status) {
  const int b = blockIdx.x;
  if (!seq_ok(S, b, status)) return;
  const int L = S.kv_len[b], start = seq_start(S, b);
  if (L < 1) {
    record_status(status, QSA_ERR_DEVICE_CHECK);
    return;
  }
  const int have = kbar_blocks[b], need = (L - 1) / D.B;
  if (have != need) {
    record_status(status, have > need ? QSA_ERR_UNSUPPORTED : QSA_ERR_DEVICE_CHECK);
    return;
  }
  const size_t pos = (size_t)start + L - 1;
  for (int i = threadIdx.x; i < D.Hkv * D.d; i += blockDim.x) {
    const int g = i / D.d, c = i - g * D.d;
    const size_t dst = (((size_t)b * D.Hkv + g) * S.kv_cap + pos) * D.d + c;
    k_cache[dst] = k_new[(size_t)b * D.Hkv * D.d + i];
    v_cache[dst] = v_new[(size_t)b * D.Hkv * D.d + i];
  }
  for (int c = threadIdx.x; c < D.di; c += blockDim.x)
    ki_cache[((size_t)b * S.kv_cap + pos) * D.di + c] = ki_new[(size_t)b * D.di + c];
  if (L % D.B != 0) return;
  __syncthreads();
  const int j = L / D.B - 1;
  const T *src = ki_cache + ((size_t)b * S.kv_cap + start + (size_t)j * D.B) * D.di;
  for (int c = threadIdx.x; c < D.di; c += blockDim.x) {
    float acc = 0.f;
    for (int u = 0; u < D.B; ++u) acc += to_f(src[(size_t)u * D.di + c]);
    kbar[((size_t)b * S.nb_cap + j) * D.di + c] = acc / (float)D.B;
  }
  if (threadIdx.x == 0) kbar_blocks[b] = L / D.B;
}

}  // namespace

cudaError_t launch_compress(const Dims &D, const Seqs &S, const void *ki, const int32_t *blocks_done,
                            float *kbar, int32_t *blocks_out, int *status, cudaStream_t st) {
  if (S.batch == 0) return cudaSuccess;
  int gx = (S.nb_cap + kCompressWarps - 1) / kCompressWarps;
  gx = max(1, min(gx, 4096));
  dim3 grid(gx, S.batch);
  note_launch();
  if (D.bf16)
    k_compress<__nv_bfloat16><<<grid, kCompressWarps * 32, 0, st>>>(D, S, (const __nv_bfloat16 *)ki, blocks_done, kbar,
                                                    blocks_out, status);
  else
    k_compress<float><<<grid, kCompressWarps * 32, 0, st>>>(D, S, (const float *)ki, blocks_done, kbar, blocks_out,
                                            status);
  return cudaGetLastError();
}

static size_t score_smem(const Dims &D, int warps, int nc_cap) {
  return sizeof(float) * ((size_t)warps * D.Hi * D.di + 32 * (D.di + 1) + (size_t)warps * nc_cap);
}

// With scores_out set: the warp-per-row kernel writes each row's scores there and
// selects nothing (the CTA-per-row kernel is not used).
static cudaError_t launch_score_topk_simt_impl(const Dims &D, const Seqs &S, const void *qi, const float *kbar,
                                               int32_t *sel, int *status, cudaStream_t st, float *scores_out) {
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  if (!scores_out && (long long)S.batch * S.n_q <= 4096 && D.di % 4 == 0) {
    // few rows: one CTA per row
    const size_t smem = sizeof(float) * ((size_t)D.Hi * D.di + D.di + S.nb_cap);
    if (smem <= 200 * 1024) {
      dim3 grid(S.n_q, S.batch);
      note_launch();
      cudaError_t e;
      if (D.bf16) {
        auto kern = k_score_topk_row<__nv_bfloat16, false>;
        if ((e = ensure_smem(kern, smem)) != cudaSuccess) return e;
        kern<<<grid, kRowThreads, smem, st>>>(D, S, (const __nv_bfloat16 *)qi, kbar, sel, status, DecodeAppend{});
      } else {
        auto kern = k_score_topk_row<float, false>;
        if ((e = ensure_smem(kern, smem)) != cudaSuccess) return e;
        kern<<<grid, kRowThreads, smem, st>>>(D, S, (const float *)qi, kbar, sel, status, DecodeAppend{});
      }
      return cudaGetLastError();
    }
  }
  const int nc_cap = S.nb_cap;
  int warps = S.n_q < 8 ? S.n_q : 8;
  const size_t limit = 200 * 1024;
  while (warps > 1 && score_smem(D, warps, nc_cap) > limit) --warps;
  const size_t smem = score_smem(D, warps, nc_cap);
  if (smem > limit) return cudaErrorNotSupported;
  dim3 grid((S.n_q + warps - 1) / warps, S.batch);
  note_launch();
  cudaError_t e;
  if (D.bf16) {
    auto kern = k_score_topk_simt<__nv_bfloat16>;
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, warps * 32, smem, st>>>(D, S, (const __nv_bfloat16 *)qi, kbar, sel, status, warps, nc_cap,
                                         scores_out);
  } else {
    auto kern = k_score_topk_simt<float>;
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, warps * 32, smem, st>>>(D, S, (const float *)qi, kbar, sel, status, warps, nc_cap, scores_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_index_scores_simt(const Dims &D, const Seqs &S, const void *qi, const float *kbar,
                                     float *scores, int *status, cudaStream_t st) {
  return launch_score_topk_simt_impl(D, S, qi, kbar, nullptr, status, st, scores);
}

cudaError_t launch_score_topk_simt(const Dims &D, const Seqs &S, const void *qi, const float *kbar,
                                   int32_t *sel, int *status, cudaStream_t st) {
  return launch_score_topk_simt_impl(D, S, qi, kbar, sel, status, st, nullptr);
}

cudaError_t launch_decode_append_score(const Dims &D, const Seqs &S, const DecodeAppend &A, const void *qi,
                                       float *kbar, int32_t *sel, int *status, cudaStream_t st) {
  if (S.batch == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)D.Hi * D.di + D.di + S.nb_cap);
  if (S.n_q != 1 || D.di % 4 != 0 || smem > 200 * 1024) {
    // general path: separate prologue, then the scoring launch
    cudaError_t e = launch_decode_append(D, S, A.k_cache, A.v_cache, A.ki_cache, kbar, A.kbar_blocks, A.k_new,
                                         A.v_new, A.ki_new, status, st);
    if (e != cudaSuccess) return e;
    return launch_score_topk_simt(D, S, qi, kbar, sel, status, st);
  }
  dim3 grid(1, S.batch);
  note_launch();
  cudaError_t e;
  if (D.bf16) {
    auto kern = k_score_topk_row<__nv_bfloat16, true>;
    if ((e = ensure_smem(kern, smem)) != cudaSuccess) return e;
    kern<<<grid, kRowThreads, smem, st>>>(D, S, (const __nv_bfloat16 *)qi, kbar, sel, status, A);
  } else {
    auto kern = k_score_topk_row<float, true>;
    if ((e = ensure_smem(kern, smem)) != cudaSuccess) return e;
    kern<<<grid, kRowThreads, smem, st>>>(D, S, (const float *)qi, kbar, sel, status, A);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const Dims &D, const Seqs &S, const void *q, const void *k,
                             const void *v, const int32_t *sel, void *out, int *status,
                             cudaStream_t st) {
  if (S.batch == 0 || S.n_q == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)D.G * D.d + 32 * (D.d + 1) + 32 * D.d);
  dim3 grid(S.n_q, D.Hkv, S.batch);
  note_launch();
  cudaError_t e;
  if (D.bf16) {
    auto kern = k_attn_simt<__nv_bfloat16>;
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, D.G * 32, smem, st>>>(D, S, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                       (const __nv_bfloat16 *)v, sel, (__nv_bfloat16 *)out, status);
  } else {
    auto kern = k_attn_simt<float>;
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, D.G * 32, smem, st>>>(D, S, (const float *)q, (const float *)k, (const float *)v, sel,
                                       (float *)out, status);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_append(const Dims &D, const Seqs &S, void *k_cache, void *v_cache,
                                 void *ki_cache, float *kbar, int32_t *kbar_blocks,
                                 const void *k_new, const void *v_new, const void *ki_new,
                                 int *status, cudaStream_t st) {
  if (S.batch == 0) return cudaSuccess;
  note_launch();
  if (D.bf16)
    k_decode_append<__nv_bfloat16><<<S.batch, 256, 0, st>>>(
        D, S, (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache, (__nv_bfloat16 *)ki_cache, kbar,
        kbar_blocks, (const __nv_bfloat16 *)k_new, (const __nv_bfloat16 *)v_new,
        (const __nv_bfloat16 *)ki_new, status);
  else
    k_decode_append<float><<<S.batch, 256, 0, st>>>(D, S, (float *)k_cache, (float *)v_cache,
                                                    (float *)ki_cache, kbar, kbar_blocks,
                                                    (const float *)k_new, (const float *)v_new,
                                                    (const float *)ki_new, status);
  return cudaGetLastError();
}

}  // namespace qsa
