// Internal declarations shared by the QSA CUDA translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qsa.h"

namespace qsa {

// Resolved problem shape (from qsa_config_t after validation).
struct Dims {
  int Hq, Hkv, G, d;  // G = Hq / Hkv query heads per KV head
  int Hi, di;         // indexer heads / dim
  int B, k;           // block size (compress ratio) and blocks kept per query
  float scale;        // softmax scale
  bool bf16;          // element type of q, k, v, qi, ki, out
};

// Sequence geometry of one call (all device pointers).
struct Seqs {
  const int32_t *kv_start, *kv_len, *q_first;
  int batch, n_q, kv_cap;
  int nb_cap;  // kv_cap / B: rows of kbar per sequence
};

// Workspace layout: [0, 256) status word area, then kernel scratch. Within the status
// area, the two words at kSchedOffset are the unit counters of the persistent prefill
// attention kernel, which its last CTA sets back to zero.
constexpr size_t kStatusBytes = 256;
constexpr size_t kSchedOffset = 128;

__device__ __forceinline__ void record_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// A null kv_start means every sequence starts at storage index 0; a null q_first
// means the single query row of each sequence sits at kv_len - 1 (decode).
__device__ __forceinline__ int seq_start(const Seqs &s, int b) { return s.kv_start ? s.kv_start[b] : 0; }
__device__ __forceinline__ int seq_qfirst(const Seqs &s, int b) {
  return s.q_first ? s.q_first[b] : s.kv_len[b] - 1;
}

// True when the sequence's geometry fits its buffers; records a device check otherwise.
__device__ __forceinline__ bool seq_ok(const Seqs &s, int b, int *status) {
  const int st = seq_start(s, b), len = s.kv_len[b];
  const bool ok = st >= 0 && len >= 0 && (long long)st + len <= (long long)s.kv_cap;
  if (!ok) record_status(status, QSA_ERR_DEVICE_CHECK);
  return ok;
}

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Validates a config and fills the resolved shape (the rules of qsa_config_validate).
qsa_status_t resolve_config(const qsa_config_t *cfg, Dims *D);

// Host-side count of kernel launches issued by this library.
void note_launch(int n = 1);

// Remember a failed CUDA call for qsa_last_error() (what + the CUDA error text).
void note_error(const char *what, cudaError_t e);

// Raise a kernel's dynamic shared memory limit once per (device, kernel) -- the
// attribute is sticky -- so that launches stay legal while a stream is being
// captured into a CUDA graph. Keyed by the kernel's address: instantiations of one
// template share a type but not their attributes.
cudaError_t ensure_smem_for(const void *kernel, size_t bytes);
template <typename K>
cudaError_t ensure_smem(K kernel, size_t bytes) {
  return ensure_smem_for(reinterpret_cast<const void *>(kernel), bytes);
}

// Launch `kernel` on `st`; with pdl, as a programmatic dependent of the kernel before
// it in the stream (it may start while that kernel finishes and must griddepcontrol.wait
// before reading that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                             Args &&...args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&lc, kernel, static_cast<KArgs>(args)...);
}

// ---- launches (each returns the launch error, cudaSuccess otherwise) ----

// Step 1: kbar[b][j] for blocks_done[b] <= j < kv_len[b] / B; optionally records
// kv_len[b] / B into blocks_out[b].
cudaError_t launch_compress(const Dims &D, const Seqs &S, const void *ki, const int32_t *blocks_done,
                            float *kbar, int32_t *blocks_out, int *status, cudaStream_t st);

// Steps 2+3 (CUDA cores, fp32): scores and top-k for every query row.
cudaError_t launch_score_topk_simt(const Dims &D, const Seqs &S, const void *qi, const float *kbar,
                                   int32_t *sel, int *status, cudaStream_t st);

// Steps 2+3 on tcgen05 tensor cores (bf16 indexer, kbar as a bf16 hi/lo pair); scratch
// holds the hi/lo planes (score_tc_workspace bytes).
bool score_tc_supported(const Dims &D, const Seqs &S);
size_t score_tc_workspace(const Dims &D, const Seqs &S);
// With scores_out set, writes each row's scores s[b][r][j] (j < n_c of the row) to
// scores_out [batch][n_q][nb_cap] instead of selecting (sel is not touched).
// pdl: the k̄ split and the scoring kernel are launched as programmatic dependents of
// the kernel before them (qsa_forward's compression).
cudaError_t launch_score_topk_tc(const Dims &D, const Seqs &S, const void *qi, const float *kbar, int32_t *sel,
                                 void *scratch, int *status, cudaStream_t st, float *scores_out = nullptr,
                                 bool pdl = false);

// Steps 2 alone on CUDA cores (fp32): each row's scores s[b][r][j], j < n_c, into
// scores [batch][n_q][nb_cap]; other entries are not written.
cudaError_t launch_index_scores_simt(const Dims &D, const Seqs &S, const void *qi, const float *kbar,
                                     float *scores, int *status, cudaStream_t st);

// Step 3 alone: top-k of each row of a score matrix [batch][n_q][nb_cap] (any finite
// fp32 values, e.g. the sum of head-sharded partial scores), ties to the lower block.
cudaError_t launch_select_topk(const Dims &D, const Seqs &S, const float *scores, int32_t *sel, int *status,
                               cudaStream_t st);

// The decode prologue (append the new token at kv_len - 1, compress a block it
// completes, advance kbar_blocks; see launch_decode_append) fused with steps 2+3
// for the single query row of each sequence.
struct DecodeAppend {
  void *k_cache, *v_cache, *ki_cache;
  int32_t *kbar_blocks;
  const void *k_new, *v_new, *ki_new;
};
cudaError_t launch_decode_append_score(const Dims &D, const Seqs &S, const DecodeAppend &A, const void *qi,
                                       float *kbar, int32_t *sel, int *status, cudaStream_t st);

// Input projections with RoPE (tcgen05 GEMM, bf16): see qsa_project in qsa.h.
bool proj_supported(const Dims &D, int hidden, int rd_attn, int rd_idx);
cudaError_t launch_proj_rope(const Dims &D, int hidden, float rope_theta, int rd_attn, int rd_idx, const void *x,
                             const void *w, const int32_t *pos0, int batch, int n_tok, void *q, void *qi, void *k,
                             void *v, void *ki, int kv_cap, int kv_row0, int *status, cudaStream_t st);

// Checks every row of a selection list (ids in [0, n_c), strictly ascending, then -1
// padding; padding rows all -1) and records QSA_ERR_DEVICE_CHECK on a violation.
// Launched before the attention in the QSA_DEBUG build.
cudaError_t launch_validate_sel(const Dims &D, const Seqs &S, const int32_t *sel, int *status, cudaStream_t st);

// Step 4 on CUDA cores (fp32 accumulate), any supported shape.
cudaError_t launch_attn_simt(const Dims &D, const Seqs &S, const void *q, const void *k,
                             const void *v, const int32_t *sel, void *out, int *status,
                             cudaStream_t st);

// Step 4 on tcgen05 tensor cores (bf16, d = 128, G divides 128); returns
// cudaErrorNotSupported when the shape is not served.
bool attn_tc_supported(const Dims &D);
size_t attn_tc_workspace(const Dims &D, const Seqs &S);
// pdl: launched as a programmatic dependent of the kernel before it (qsa_forward's scoring).
// sched: two zeroed words (unit ticket, CTAs done) the kernel leaves at zero.
cudaError_t launch_attn_tc(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                           const int32_t *sel, void *out, unsigned *sched, int *status, cudaStream_t st,
                           bool pdl = false);

// Step 4 on tcgen05 tensor cores, one 128-row tile per CTA with double-buffered S
// (bf16, d = 256, G divides 128, block size a multiple of 64); no scratch.
bool attn_tc1_supported(const Dims &D);
cudaError_t launch_attn_tc1(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                            const int32_t *sel, void *out, int *status, cudaStream_t st);

// Decode prologue: append the new token, check the indexer state is in step,
// compress a just-completed block, advance kbar_blocks.
cudaError_t launch_decode_append(const Dims &D, const Seqs &S, void *k_cache, void *v_cache,
                                 void *ki_cache, float *kbar, int32_t *kbar_blocks,
                                 const void *k_new, const void *v_new, const void *ki_new,
                                 int *status, cudaStream_t st);

// Split-KV decode attention (one query per sequence), HBM-bound.
bool attn_decode_supported(const Dims &D);
size_t attn_decode_workspace(const Dims &D, const Seqs &S);
// pdl: launch as a programmatic dependent of the previous kernel in the stream, whose
// prologue (the unit prefix sums over kv_len, kv_start, q_first) overlaps that
// kernel's tail. Only for a predecessor that writes none of those (the decode
// append/selection kernel of qsa_forward).
cudaError_t launch_attn_decode(const Dims &D, const Seqs &S, const void *q, const void *k,
                               const void *v, const int32_t *sel, void *out, void *scratch,
                               size_t scratch_bytes, int *status, cudaStream_t st, bool pdl = false);

// Cache offloading (decode with K/V in host memory): copy each sequence's attended
// blocks -- its selection, then its trailing block, whose last row is this step's
// token taken from k_new / v_new -- from the caches into a compact device staging
// cache of capacity (k + 1) * B per (sequence, KV head), and write the selection
// (0 .. n_sel - 1, -1 padded) and the lengths that address it there.
size_t offload_cap(const Dims &D);
cudaError_t launch_offload_gather(const Dims &D, const Seqs &S, const void *k_cache, const void *v_cache,
                                  const void *k_new, const void *v_new, const int32_t *sel, void *k_stage,
                                  void *v_stage, int32_t *sel_stage, int32_t *len_stage, cudaStream_t st);

}  // namespace qsa
