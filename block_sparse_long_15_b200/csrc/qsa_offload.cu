// Cache offloading for decode: the attention K/V cache stays in host memory and
// only the blocks a step attends cross PCIe, while the indexer state (k̄ and the
// indexer keys) stays on the device ("Qwen4-Exp" model doc, Usage tips: the
// indexer state is kept apart from the attention K/V cache, which QSA reads only
// at the selected blocks and the trailing block).
//
// After the decode append/selection kernel has written this step's token into the
// host cache and the selection into `sel`, one CTA per (attended item, KV head,
// sequence) copies that item's rows into a compact device staging cache of
// capacity (k + 1) * B per (sequence, KV head): the selected blocks in ascending
// order at slots 0 .. n_sel - 1, the trailing block at slot n_sel. Attending
// query t = L - 1 over the staging cache with length n_sel * B + (L - n_c * B) and
// selection 0 .. n_sel - 1 visits the same keys in the same order as attending the
// full cache with the original selection, so the results are identical.
#include <stdint.h>

#include "qsa_internal.h"

namespace qsa {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;  // 16-byte pieces in flight per thread

template <typename T>
__global__ void __launch_bounds__(kGatherThreads)
k_offload_gather(Dims D, Seqs S, const T *k_cache, const T *v_cache, const T *__restrict__ k_new,
                 const T *__restrict__ v_new, const int32_t *__restrict__ sel, T *__restrict__ k_stage,
                 T *__restrict__ v_stage, int32_t *__restrict__ sel_stage, int32_t *__restrict__ len_stage,
                 int cap) {
  const int j = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int start = seq_start(S, b), L = S.kv_len[b];
  const bool ok = start >= 0 && L >= 1 && (long long)start + L <= (long long)S.kv_cap;
  const int n_c = ok ? L / D.B : 0;
  const int n_sel = min(n_c, D.k);
  const int tl = ok ? L - n_c * D.B : 0;  // trailing rows, the last being this step's token
  if (j == 0 && g == 0) {
    for (int i = threadIdx.x; i < D.k; i += blockDim.x) sel_stage[(size_t)b * D.k + i] = i < n_sel ? i : -1;
    if (threadIdx.x == 0) len_stage[b] = ok ? n_sel * D.B + tl : 0;
  }
  int blk, rows;
  if (j < n_sel) {
    blk = sel[(size_t)b * D.k + j];
    rows = D.B;
    if (blk < 0 || blk >= n_c) return;  // not a complete block: nothing to copy
  } else if (j == n_sel && tl > 0) {
    blk = n_c;
    rows = tl;
  } else {
    return;
  }
  const size_t src_row0 = ((size_t)b * D.Hkv + g) * S.kv_cap + start + (size_t)blk * D.B;
  const size_t dst_row0 = ((size_t)b * D.Hkv + g) * cap + (size_t)j * D.B;
  const uint4 *ks = (const uint4 *)(k_cache + src_row0 * D.d);
  const uint4 *vs = (const uint4 *)(v_cache + src_row0 * D.d);
  const uint4 *kn = (const uint4 *)(k_new + ((size_t)b * D.Hkv + g) * D.d);
  const uint4 *vn = (const uint4 *)(v_new + ((size_t)b * D.Hkv + g) * D.d);
  uint4 *kd = (uint4 *)(k_stage + dst_row0 * D.d);
  uint4 *vd = (uint4 *)(v_stage + dst_row0 * D.d);
  const int per_row = D.d * (int)sizeof(T) / 16;
  const int n = rows * per_row;
  const int new_from = (j == n_sel) ? (rows - 1) * per_row : n;  // pieces of this step's token
  for (int e0 = threadIdx.x; e0 < n; e0 += kGatherThreads * kGatherUnroll) {
    uint4 kv[kGatherUnroll], vv[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int e = e0 + u * kGatherThreads;
      if (e < new_from) {
        kv[u] = ks[e];
        vv[u] = vs[e];
      } else if (e < n) {
        kv[u] = kn[e - new_from];
        vv[u] = vn[e - new_from];
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int e = e0 + u * kGatherThreads;
      if (e < n) {
        kd[e] = kv[u];
        vd[e] = vv[u];
      }
    }
  }
}

}  // namespace

size_t offload_cap(const Dims &D) { return (size_t)(D.k + 1) * D.B; }

cudaError_t launch_offload_gather(const Dims &D, const Seqs &S, const void *k_cache, const void *v_cache,
                                  const void *k_new, const void *v_new, const int32_t *sel, void *k_stage,
                                  void *v_stage, int32_t *sel_stage, int32_t *len_stage, cudaStream_t st) {
  if (S.batch == 0) return cudaSuccess;
  if (S.batch > 65535 || D.Hkv > 65535) return cudaErrorNotSupported;
  const dim3 grid(D.k + 1, D.Hkv, S.batch);
  const int cap = (int)offload_cap(D);
  note_launch();
  if (D.bf16)
    k_offload_gather<__nv_bfloat16><<<grid, kGatherThreads, 0, st>>>(
        D, S, (const __nv_bfloat16 *)k_cache, (const __nv_bfloat16 *)v_cache, (const __nv_bfloat16 *)k_new,
        (const __nv_bfloat16 *)v_new, sel, (__nv_bfloat16 *)k_stage, (__nv_bfloat16 *)v_stage, sel_stage,
        len_stage, cap);
  else
    k_offload_gather<float><<<grid, kGatherThreads, 0, st>>>(
        D, S, (const float *)k_cache, (const float *)v_cache, (const float *)k_new, (const float *)v_new, sel,
        (float *)k_stage, (float *)v_stage, sel_stage, len_stage, cap);
  return cudaGetLastError();
}

}  // namespace qsa
