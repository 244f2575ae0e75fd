// Host side of the QSA C ABI (include/qsa.h): argument validation, workspace
// sizing and kernel dispatch. Nothing here allocates device memory.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "qsa_internal.h"

#include <atomic>
#include <mutex>

using namespace qsa;

#include <stdio.h>

namespace qsa {
static std::atomic<uint64_t> g_launches{0};
static thread_local char g_last_error[256] = "";
static thread_local uint64_t g_error_serial = 0;
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
cudaError_t ensure_smem_for(const void *kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  struct Grant {
    const void *kernel;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static Grant table[256];
  static int n = 0;
  std::lock_guard<std::mutex> lock(mu);
  Grant *g = nullptr;
  for (int i = 0; i < n; ++i)
    if (table[i].kernel == kernel && table[i].dev == dev) g = &table[i];
  if (g && g->bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (!g && n < 256) g = &table[n++];
  if (g) *g = Grant{kernel, dev, bytes};
  return cudaSuccess;
}

void note_error(const char *what, cudaError_t e) {
  snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
  ++g_error_serial;
}
}  // namespace qsa

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Qwen4ExpTextConfig indexer fields are all-or-nothing (Usage tips: "the complete
// set of QSA indexer fields enables sparse token selection"); QSA needs exactly one
// indexer key head (indexer_kv_heads parameter).
qsa_status_t resolve(const qsa_config_t *c, Dims *D) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (c->indexer_n_heads <= 0 || c->indexer_kv_heads <= 0 || c->indexer_head_dim <= 0 ||
      c->indexer_budget <= 0 || c->indexer_compress_ratio <= 0)
    return QSA_ERR_INVALID_ARG;
  if (c->indexer_kv_heads != 1) return QSA_ERR_UNSUPPORTED;
  if (c->num_attention_heads <= 0 || c->num_key_value_heads <= 0 ||
      c->num_attention_heads % c->num_key_value_heads != 0)
    return QSA_ERR_INVALID_ARG;
  if (c->head_dim <= 0 || c->head_dim % 8 != 0 || c->indexer_head_dim % 8 != 0)
    return QSA_ERR_INVALID_ARG;
  if (c->dtype != QSA_DTYPE_BF16 && c->dtype != QSA_DTYPE_FP32) return QSA_ERR_INVALID_ARG;
  if (c->indexer_budget < c->indexer_compress_ratio) return QSA_ERR_INVALID_ARG;
  if (!(c->softmax_scale == c->softmax_scale)) return QSA_ERR_INVALID_ARG;  // NaN
  const int G = c->num_attention_heads / c->num_key_value_heads;
  if (c->head_dim > 256 || c->indexer_head_dim > 256 || c->indexer_n_heads > 64 || G > 32 ||
      c->indexer_compress_ratio > 256 || c->indexer_budget / c->indexer_compress_ratio > 4096)
    return QSA_ERR_UNSUPPORTED;
  if (D) {
    D->Hq = c->num_attention_heads;
    D->Hkv = c->num_key_value_heads;
    D->G = G;
    D->d = c->head_dim;
    D->Hi = c->indexer_n_heads;
    D->di = c->indexer_head_dim;
    D->B = c->indexer_compress_ratio;
    D->k = c->indexer_budget / c->indexer_compress_ratio;
    D->scale = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / sqrtf((float)c->head_dim);
    D->bf16 = c->dtype == QSA_DTYPE_BF16;
  }
  return QSA_OK;
}

qsa_status_t check_sizes(const Dims &D, int batch, int n_q, int kv_cap) {
  if (batch < 0 || n_q < 0 || kv_cap < 0) return QSA_ERR_INVALID_ARG;
  if ((long long)kv_cap / D.B > 32768) return QSA_ERR_UNSUPPORTED;
  return QSA_OK;
}

Seqs make_seqs(const Dims &D, const int32_t *kv_start, const int32_t *kv_len, const int32_t *q_first,
               int batch, int n_q, int kv_cap) {
  Seqs S;
  S.kv_start = kv_start;
  S.kv_len = kv_len;
  S.q_first = q_first;
  S.batch = batch;
  S.n_q = n_q;
  S.kv_cap = kv_cap;
  S.nb_cap = kv_cap / D.B;
  return S;
}

// One query row per sequence (a decode step, or a stage call with n_q == 1) goes to
// the split-KV decode kernel when it serves the shape; more rows go to a
// tensor-core prefill kernel: the two-tile kernel for head_dim 128, the one-tile
// kernel for head_dim 256; everything else to the CUDA-core kernel.
enum AttnKernel { kAttnSimt, kAttnTc, kAttnTc1, kAttnDecode };
AttnKernel pick_attn(const Dims &D, const Seqs &S) {
  if (S.n_q == 1 && attn_decode_supported(D)) return kAttnDecode;
  if (attn_tc_supported(D)) return kAttnTc;
  if (attn_tc1_supported(D)) return kAttnTc1;
  return kAttnSimt;
}

// Scoring: few rows (a decode step) take the CTA-per-row kernel; otherwise the
// tensor-core kernel when it serves the shape, else the warp-per-row kernel.
bool use_score_tc(const Dims &D, const Seqs &S) {
  return (long long)S.batch * S.n_q > 4096 && score_tc_supported(D, S);
}

// Scratch after the status word. Scoring and attention run one after the other on
// the stream, so they share it.
size_t scratch_need(const Dims &D, const Seqs &S) {
  size_t s = 0;
  switch (pick_attn(D, S)) {
    case kAttnDecode: s = attn_decode_workspace(D, S); break;
    case kAttnTc: s = attn_tc_workspace(D, S); break;
    default: break;
  }
  if (use_score_tc(D, S)) s = s > score_tc_workspace(D, S) ? s : score_tc_workspace(D, S);
  return (s + 255) & ~(size_t)255;
}


// Status of a launch; the launch sites record a detailed message, this records a
// generic one only when no message was recorded since the call began.
thread_local uint64_t g_serial_at_entry = 0;
qsa_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QSA_OK;
  if (g_error_serial == g_serial_at_entry) note_error("kernel launch", e);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    return QSA_ERR_UNSUPPORTED;
  }
  return QSA_ERR_CUDA;
}

int *status_word(void *ws) { return (int *)ws; }

qsa_status_t score_dispatch(const Dims &D, const Seqs &S, const void *qi, const float *kbar, int32_t *sel,
                            void *ws, cudaStream_t st, bool pdl = false) {
  int *status = (int *)ws;
  if (use_score_tc(D, S))
    return cuda_status(launch_score_topk_tc(D, S, qi, kbar, sel, (char *)ws + kStatusBytes, status, st, nullptr, pdl));
  return cuda_status(launch_score_topk_simt(D, S, qi, kbar, sel, status, st));
}

qsa_status_t attn_dispatch(const Dims &D, const Seqs &S, const void *q, const void *k, const void *v,
                           const int32_t *sel, void *out, void *ws, size_t ws_bytes, cudaStream_t st,
                           bool pdl = false) {
  char *scratch = (char *)ws + kStatusBytes;
  const size_t scratch_bytes = ws_bytes - kStatusBytes;
#ifdef QSA_DEBUG
  // debug build: check the selection the attention is about to read
  if (cudaError_t e = launch_validate_sel(D, S, sel, status_word(ws), st)) return cuda_status(e);
#endif
  switch (pick_attn(D, S)) {
    case kAttnDecode:
      return cuda_status(
          launch_attn_decode(D, S, q, k, v, sel, out, scratch, scratch_bytes, status_word(ws), st, pdl));
    case kAttnTc:
      return cuda_status(
          launch_attn_tc(D, S, q, k, v, sel, out, (unsigned *)((char *)ws + kSchedOffset), status_word(ws), st, pdl));
    case kAttnTc1:
      return cuda_status(launch_attn_tc1(D, S, q, k, v, sel, out, status_word(ws), st));
    default:
      return cuda_status(launch_attn_simt(D, S, q, k, v, sel, out, status_word(ws), st));
  }
}

}  // namespace

qsa_status_t qsa::resolve_config(const qsa_config_t *cfg, Dims *D) { return resolve(cfg, D); }

// ---------------------------------------------------------------- cache offloading
namespace {
struct StagingLayout {
  size_t k_off, v_off, sel_off, len_off, total;
};
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
StagingLayout staging_layout(const Dims &D, int batch) {
  const size_t esz = D.bf16 ? 2 : 4;
  const size_t kv = round256((size_t)batch * D.Hkv * offload_cap(D) * D.d * esz);
  StagingLayout L;
  L.k_off = 0;
  L.v_off = kv;
  L.sel_off = 2 * kv;
  L.len_off = L.sel_off + round256((size_t)batch * D.k * sizeof(int32_t));
  L.total = L.len_off + round256((size_t)batch * sizeof(int32_t));
  return L;
}
// The device address of a cache the caller keeps in host memory: page-locked host
// memory (or device memory) is reachable from kernels, pageable memory is not.
void *device_view(void *p) {
  cudaPointerAttributes a;
  if (!p || cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type == cudaMemoryTypeUnregistered) return nullptr;
  return a.devicePointer;
}
}  // namespace

extern "C" {

int32_t qsa_abi_version(void) { return QSA_ABI_VERSION; }

uint64_t qsa_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *qsa_last_error(void) { return g_last_error; }

qsa_status_t qsa_config_validate(const qsa_config_t *cfg) { return resolve(cfg, nullptr); }

int32_t qsa_topk_blocks(const qsa_config_t *cfg) {
  Dims D;
  return resolve(cfg, &D) == QSA_OK ? D.k : 0;
}

const char *qsa_status_string(qsa_status_t s) {
  switch (s) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported configuration or operation";
    case QSA_ERR_CUDA: return "CUDA error";
    case QSA_ERR_TIMEOUT: return "device wait timed out";
    case QSA_ERR_DEVICE_CHECK: return "device-side argument check failed";
  }
  return "unknown status";
}

const char *qsa_attn_kernel_name(const qsa_config_t *cfg, int32_t mode) {
  Dims D;
  if (resolve(cfg, &D) != QSA_OK) return "none";
  Seqs S = make_seqs(D, nullptr, nullptr, nullptr, 1, mode == QSA_DECODE ? 1 : 2, 0);
  switch (pick_attn(D, S)) {
    case kAttnDecode: return "split-kv decode";
    case kAttnTc: return "tcgen05";
    case kAttnTc1: return "tcgen05 one-tile";
    default: return "simt";
  }
}

qsa_status_t qsa_workspace_size(const qsa_config_t *cfg, int32_t mode, int32_t batch, int32_t n_q,
                                int32_t kv_cap, size_t *bytes) {
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if (!bytes || (mode != QSA_PREFILL && mode != QSA_DECODE)) return QSA_ERR_INVALID_ARG;
  if ((s = check_sizes(D, batch, n_q, kv_cap)) != QSA_OK) return s;
  Seqs S = make_seqs(D, nullptr, nullptr, nullptr, batch, n_q, kv_cap);
  if (mode == QSA_DECODE) S.n_q = 1;
  *bytes = kStatusBytes + scratch_need(D, S);
  return QSA_OK;
}

qsa_status_t qsa_compress_blocks(const qsa_config_t *cfg, const void *ki, const int32_t *kv_start,
                                 const int32_t *kv_len, const int32_t *blocks_done, int32_t batch,
                                 int32_t kv_cap, float *kbar, int32_t *kbar_blocks, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if ((s = check_sizes(D, batch, 1, kv_cap)) != QSA_OK) return s;
  if (batch == 0) return QSA_OK;
  // With kv_cap < B no block can complete: the k̄ buffer is empty and may be null.
  if (!ki || !kv_start || !kv_len || (!kbar && kv_cap / D.B > 0)) return QSA_ERR_INVALID_ARG;
  if (!aligned16(ki) || !aligned16(kbar)) return QSA_ERR_INVALID_ARG;
  Seqs S = make_seqs(D, kv_start, kv_len, nullptr, batch, 0, kv_cap);
  return cuda_status(launch_compress(D, S, ki, blocks_done, kbar, kbar_blocks, nullptr, (cudaStream_t)stream));
}

qsa_status_t qsa_index_score_topk(const qsa_config_t *cfg, const void *qi, const float *kbar,
                                  const int32_t *kv_len, const int32_t *q_first, int32_t batch,
                                  int32_t n_q, int32_t kv_cap, int32_t *sel, void *workspace,
                                  size_t workspace_bytes, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if ((s = check_sizes(D, batch, n_q, kv_cap)) != QSA_OK) return s;
  if (batch == 0 || n_q == 0) return QSA_OK;
  if (!qi || (!kbar && kv_cap / D.B > 0) || !kv_len || !q_first || !sel || !workspace)
    return QSA_ERR_INVALID_ARG;
  if (!aligned16(qi) || !aligned16(kbar) || !aligned16(sel) || !aligned16(workspace))
    return QSA_ERR_INVALID_ARG;
  // Scoring reads no keys, only k̄ rows (indexed by block from the sequence start),
  // so kv_start is not needed here.
  Seqs S = make_seqs(D, nullptr, kv_len, q_first, batch, n_q, kv_cap);
  if (workspace_bytes < kStatusBytes + scratch_need(D, S)) return QSA_ERR_INVALID_ARG;
  return score_dispatch(D, S, qi, kbar, sel, workspace, (cudaStream_t)stream);
}

qsa_status_t qsa_project(const qsa_config_t *cfg, const qsa_proj_config_t *pc, const void *x, const void *w,
                         const int32_t *q_first, int32_t batch, int32_t n_tok, void *q, void *qi, void *k,
                         void *v, void *ki, int32_t kv_cap, int32_t kv_row0, void *workspace,
                         size_t workspace_bytes, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if (!pc || batch < 0 || n_tok < 0 || kv_cap < 0 || kv_row0 < 0) return QSA_ERR_INVALID_ARG;
  if (batch == 0 || n_tok == 0) return QSA_OK;
  if ((long long)kv_row0 + n_tok > kv_cap) return QSA_ERR_INVALID_ARG;
  if (!(pc->rope_theta > 0.f) || pc->hidden_size <= 0) return QSA_ERR_INVALID_ARG;
  if (!proj_supported(D, pc->hidden_size, pc->rotary_dim, pc->indexer_rotary_dim)) return QSA_ERR_UNSUPPORTED;
  if (!x || !w || !q_first || !q || !qi || !k || !v || !ki || !workspace) return QSA_ERR_INVALID_ARG;
  const void *ptrs[] = {x, w, q, qi, k, v, ki, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return QSA_ERR_INVALID_ARG;
  if (workspace_bytes < kStatusBytes) return QSA_ERR_INVALID_ARG;
  return cuda_status(launch_proj_rope(D, pc->hidden_size, pc->rope_theta, pc->rotary_dim, pc->indexer_rotary_dim,
                                      x, w, q_first, batch, n_tok, q, qi, k, v, ki, kv_cap, kv_row0,
                                      status_word(workspace), (cudaStream_t)stream));
}

qsa_status_t qsa_index_scores(const qsa_config_t *cfg, const void *qi, const float *kbar, const int32_t *kv_len,
                              const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap, float *scores,
                              void *workspace, size_t workspace_bytes, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if ((s = check_sizes(D, batch, n_q, kv_cap)) != QSA_OK) return s;
  if (batch == 0 || n_q == 0 || kv_cap / D.B == 0) return QSA_OK;  // no complete block: nothing to score
  if (!qi || !kbar || !kv_len || !q_first || !scores || !workspace) return QSA_ERR_INVALID_ARG;
  if (!aligned16(qi) || !aligned16(kbar) || !aligned16(scores) || !aligned16(workspace)) return QSA_ERR_INVALID_ARG;
  Seqs S = make_seqs(D, nullptr, kv_len, q_first, batch, n_q, kv_cap);
  if (workspace_bytes < kStatusBytes + scratch_need(D, S)) return QSA_ERR_INVALID_ARG;
  int *status = status_word(workspace);
  if (use_score_tc(D, S))
    return cuda_status(launch_score_topk_tc(D, S, qi, kbar, nullptr, (char *)workspace + kStatusBytes, status,
                                            (cudaStream_t)stream, scores));
  return cuda_status(launch_index_scores_simt(D, S, qi, kbar, scores, status, (cudaStream_t)stream));
}

qsa_status_t qsa_select_topk(const qsa_config_t *cfg, const float *scores, const int32_t *kv_len,
                             const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap, int32_t *sel,
                             void *workspace, size_t workspace_bytes, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if ((s = check_sizes(D, batch, n_q, kv_cap)) != QSA_OK) return s;
  if (batch == 0 || n_q == 0) return QSA_OK;
  if ((!scores && kv_cap / D.B > 0) || !kv_len || !q_first || !sel || !workspace) return QSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(sel) || !aligned16(workspace)) return QSA_ERR_INVALID_ARG;
  if (workspace_bytes < kStatusBytes) return QSA_ERR_INVALID_ARG;
  Seqs S = make_seqs(D, nullptr, kv_len, q_first, batch, n_q, kv_cap);
  return cuda_status(launch_select_topk(D, S, scores, sel, status_word(workspace), (cudaStream_t)stream));
}

qsa_status_t qsa_sparse_attn(const qsa_config_t *cfg, const void *q, const void *k, const void *v,
                             const int32_t *sel, const int32_t *kv_start, const int32_t *kv_len,
                             const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap,
                             void *out, void *workspace, size_t workspace_bytes,
                             qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if ((s = check_sizes(D, batch, n_q, kv_cap)) != QSA_OK) return s;
  if (batch == 0 || n_q == 0) return QSA_OK;
  if (!q || !k || !v || !sel || !kv_start || !kv_len || !q_first || !out || !workspace)
    return QSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(sel) ||
      !aligned16(workspace))
    return QSA_ERR_INVALID_ARG;
  Seqs S = make_seqs(D, kv_start, kv_len, q_first, batch, n_q, kv_cap);
  if (workspace_bytes < kStatusBytes + scratch_need(D, S)) return QSA_ERR_INVALID_ARG;
  return attn_dispatch(D, S, q, k, v, sel, out, workspace, workspace_bytes, (cudaStream_t)stream);
}

qsa_status_t qsa_forward(const qsa_config_t *cfg, int32_t mode, const qsa_tensors_t *t,
                         void *workspace, size_t workspace_bytes, qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if (!t || (mode != QSA_PREFILL && mode != QSA_DECODE)) return QSA_ERR_INVALID_ARG;
  if ((s = check_sizes(D, t->batch, t->n_q, t->kv_cap)) != QSA_OK) return s;
  if (t->batch == 0 || t->n_q == 0) return QSA_OK;
  if (!t->q || !t->qi || !t->k_cache || !t->v_cache || !t->ki_cache ||
      (!t->kbar_cache && t->kv_cap / D.B > 0) ||
      !t->kbar_blocks || !t->kv_start || !t->kv_len || !t->sel || !t->out || !workspace)
    return QSA_ERR_INVALID_ARG;
  if (mode == QSA_PREFILL && !t->q_first) return QSA_ERR_INVALID_ARG;
  if (mode == QSA_DECODE && (t->n_q != 1 || !t->k_new || !t->v_new || !t->ki_new))
    return QSA_ERR_INVALID_ARG;
  const void *ptrs[] = {t->q, t->qi, t->k_cache, t->v_cache, t->ki_cache, t->kbar_cache, t->sel,
                        t->out, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return QSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int32_t *q_first = t->q_first;
  Seqs S = make_seqs(D, t->kv_start, t->kv_len, q_first, t->batch, t->n_q, t->kv_cap);
  if (workspace_bytes < kStatusBytes + scratch_need(D, S)) return QSA_ERR_INVALID_ARG;
  int *status = status_word(workspace);
  if (mode == QSA_PREFILL) {
    // compress -> (k̄ split) -> score -> attention, each a programmatic dependent of the
    // one before: a kernel's prologue overlaps its predecessor's tail, and it waits for
    // that predecessor before it reads its results
    s = cuda_status(launch_compress(D, S, t->ki_cache, nullptr, t->kbar_cache, t->kbar_blocks,
                                    status, st));
    if (s != QSA_OK) return s;
    s = score_dispatch(D, S, t->qi, t->kbar_cache, t->sel, workspace, st, true);
  } else {
    // The decode query sits at kv_len - 1; a null q_first tells the kernels so.
    S.q_first = nullptr;
    DecodeAppend A{t->k_cache, t->v_cache, t->ki_cache, t->kbar_blocks, t->k_new, t->v_new, t->ki_new};
    s = cuda_status(launch_decode_append_score(D, S, A, t->qi, t->kbar_cache, t->sel, status, st));
  }
  if (s != QSA_OK) return s;
  // The kernel before the attention is this call's scoring (prefill) or append and
  // selection (decode), which writes none of what the attention's prologue reads.
  return attn_dispatch(D, S, t->q, t->k_cache, t->v_cache, t->sel, t->out, workspace, workspace_bytes, st, true);
}


qsa_status_t qsa_offload_staging_size(const qsa_config_t *cfg, int32_t batch, size_t *bytes) {
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if (!bytes || batch < 0) return QSA_ERR_INVALID_ARG;
  *bytes = staging_layout(D, batch).total;
  return QSA_OK;
}

qsa_status_t qsa_decode_offload(const qsa_config_t *cfg, const qsa_tensors_t *t, void *staging,
                                size_t staging_bytes, void *workspace, size_t workspace_bytes,
                                qsa_stream_t stream) {
  g_serial_at_entry = g_error_serial;
  Dims D;
  qsa_status_t s = resolve(cfg, &D);
  if (s != QSA_OK) return s;
  if (!t) return QSA_ERR_INVALID_ARG;
  if ((s = check_sizes(D, t->batch, 1, t->kv_cap)) != QSA_OK) return s;
  if (t->batch == 0) return QSA_OK;
  if (t->n_q != 1 || !t->q || !t->qi || !t->ki_cache || (!t->kbar_cache && t->kv_cap / D.B > 0) ||
      !t->kbar_blocks || !t->kv_start || !t->kv_len || !t->sel || !t->out || !t->k_new || !t->v_new ||
      !t->ki_new || !staging || !workspace)
    return QSA_ERR_INVALID_ARG;
  void *k_dev = device_view(t->k_cache), *v_dev = device_view(t->v_cache);
  if (!k_dev || !v_dev) {
    note_error("qsa_decode_offload: k_cache / v_cache must be page-locked host memory or device memory",
               cudaErrorInvalidValue);
    return QSA_ERR_INVALID_ARG;
  }
  const void *ptrs[] = {t->q, t->qi, k_dev, v_dev, t->ki_cache, t->kbar_cache, t->sel, t->out,
                        t->k_new, t->v_new, staging, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return QSA_ERR_INVALID_ARG;
  const StagingLayout L = staging_layout(D, t->batch);
  if (staging_bytes < L.total) return QSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  Seqs S = make_seqs(D, t->kv_start, t->kv_len, nullptr, t->batch, 1, t->kv_cap);
  char *stg = (char *)staging;
  int32_t *sel_st = (int32_t *)(stg + L.sel_off), *len_st = (int32_t *)(stg + L.len_off);
  Seqs S2 = make_seqs(D, nullptr, len_st, nullptr, t->batch, 1, (int)offload_cap(D));
  if (workspace_bytes < kStatusBytes + scratch_need(D, S) || workspace_bytes < kStatusBytes + scratch_need(D, S2))
    return QSA_ERR_INVALID_ARG;
  int *status = status_word(workspace);
  DecodeAppend A{k_dev, v_dev, t->ki_cache, t->kbar_blocks, t->k_new, t->v_new, t->ki_new};
  s = cuda_status(launch_decode_append_score(D, S, A, t->qi, t->kbar_cache, t->sel, status, st));
  if (s != QSA_OK) return s;
  s = cuda_status(launch_offload_gather(D, S, k_dev, v_dev, t->k_new, t->v_new, t->sel, stg + L.k_off,
                                        stg + L.v_off, sel_st, len_st, st));
  if (s != QSA_OK) return s;
  return attn_dispatch(D, S2, t->q, stg + L.k_off, stg + L.v_off, sel_st, t->out, workspace, workspace_bytes, st);
}

qsa_status_t qsa_read_device_status(void *workspace, qsa_stream_t stream, qsa_status_t *status) {
  if (!workspace || !status) return QSA_ERR_INVALID_ARG;
  int h = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return QSA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return QSA_ERR_CUDA;
  *status = (qsa_status_t)h;
  return QSA_OK;
}

}  // extern "C"
