/*
 * qsa.h -- C ABI of the Qwen Sparse Attention (QSA) hot path for NVIDIA B200.
 *
 * QSA as documented on the Hugging Face Transformers model page "Qwen4-Exp":
 *   intro paragraph -- several indexer query heads score compressed key blocks,
 *     the most relevant contiguous token blocks are selected, and the incomplete
 *     trailing block stays uncompressed;
 *   Qwen4ExpTextConfig parameters indexer_n_heads, indexer_kv_heads,
 *     indexer_head_dim, indexer_budget, indexer_compress_ratio -- the fields of
 *     qsa_config_t below;
 *   Usage tips -- a complete indexer field set enables QSA on full-attention
 *     layers; cache cropping is unsupported; the indexer state (compressed keys)
 *     is kept apart from the attention K/V cache.
 *
 * The path, for a query at relative position t (L = t + 1 visible tokens,
 * B = indexer_compress_ratio, k = indexer_budget / B, n_c = L / B):
 *   1. compress   kbar[j] = mean of the B indexer keys of block j (complete blocks)
 *   2. score      s[j] = sum over indexer heads h of max(0, qi[h] . kbar[j]), j < n_c
 *   3. select     all j < n_c if n_c <= k, else the k best by (-s[j], j), ascending;
 *                 plus the trailing range [n_c * B, t] (empty iff L % B == 0)
 *   4. attend     softmax(scale * q . k_u) v_u over the selected tokens u, per query
 *                 head; query head h reads KV head h / (Hq / Hkv)
 * The score formula, the tie order (lower block index wins) and the trailing
 * rule at block boundaries are readings of the page, which gives no formula.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory. Every pointer argument except `cfg`, `t` and `bytes` is a DEVICE
 * pointer owned by the caller; the library never allocates, frees or keeps a
 * pointer past the call, and only qsa_read_device_status synchronises. All work
 * is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream),
 * so results are ready when the stream is. Base pointers must be 16-byte
 * aligned and rows dense (layouts below).
 *
 * Layouts (row-major, innermost index last; "bf16" per cfg->dtype, else fp32):
 *   q, out  [batch][n_q][Hq][d]        queries / attention output
 *   qi      [batch][n_q][Hi][di]       indexer query heads
 *   k, v    [batch][Hkv][kv_cap][d]    attention keys / values (one plane per KV head)
 *   ki      [batch][kv_cap][di]        the single indexer key head
 *   kbar    [batch][kv_cap / B][di]    compressed keys, always fp32
 *   sel     [batch][n_q][k]            selected block ids, int32, ascending, -1 padded
 *   kv_start[batch]  storage index of relative position 0 (a left pad)
 *   kv_len  [batch]  visible tokens: relative positions 0 .. kv_len-1
 *   q_first [batch]  relative position of query row 0; query row r sits at
 *                    t = q_first + r and is a padding row unless 0 <= t < kv_len
 *                    (its out row is written 0 and its sel row -1).
 * Prefill with left padding: n_q = kv_cap, kv_start = pad, kv_len = kv_cap - pad,
 * q_first = -pad. Decode: n_q = 1, kv_start = 0, q_first = kv_len - 1.
 *
 * Errors. Host-side checks return QSA_ERR_INVALID_ARG (null pointer, bad size,
 * misalignment, inconsistent config) or QSA_ERR_UNSUPPORTED (a configuration the
 * page rules out, e.g. indexer_kv_heads != 1, or a shape no kernel here serves)
 * before anything is enqueued. A failed launch returns QSA_ERR_CUDA. Checks that
 * need device data (lengths beyond capacity, a decode length that went
 * backwards, a device wait that ran out) are recorded in the workspace status
 * word, skip the affected work, and are read with qsa_read_device_status.
 * No C++ exception crosses this boundary.
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_ABI_VERSION 2

typedef struct CUstream_st *qsa_stream_t; /* same type as cudaStream_t */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,
  QSA_ERR_UNSUPPORTED = 2,
  QSA_ERR_CUDA = 3,
  QSA_ERR_TIMEOUT = 4,
  QSA_ERR_DEVICE_CHECK = 5
} qsa_status_t;

enum { QSA_DTYPE_BF16 = 0, QSA_DTYPE_FP32 = 1 };
enum { QSA_PREFILL = 0, QSA_DECODE = 1 };

/* Attention and indexer fields of Qwen4ExpTextConfig that the path reads. */
typedef struct {
  int32_t num_attention_heads;    /* Hq */
  int32_t num_key_value_heads;    /* Hkv; Hq % Hkv == 0 (grouped-query attention) */
  int32_t head_dim;               /* d; multiple of 8, <= 256 */
  int32_t indexer_n_heads;        /* Hi >= 1; setting it enables QSA */
  int32_t indexer_kv_heads;       /* must be 1: QSA uses a single indexer key head */
  int32_t indexer_head_dim;       /* di; multiple of 8, <= 256 */
  int32_t indexer_budget;         /* tokens from complete blocks per query; k = budget / B >= 1 */
  int32_t indexer_compress_ratio; /* B: keys averaged per block; 1 .. 256 */
  float softmax_scale;            /* <= 0 selects 1 / sqrt(head_dim) */
  int32_t dtype;                  /* QSA_DTYPE_BF16 or QSA_DTYPE_FP32 for q, k, v, qi, ki, out */
} qsa_config_t;

/* Everything qsa_forward touches. Caches double as prefill inputs: in prefill
 * mode k_cache / v_cache / ki_cache already hold the prompt. */
typedef struct {
  int32_t batch, n_q, kv_cap;
  const void *q;        /* [batch][n_q][Hq][d] */
  const void *qi;       /* [batch][n_q][Hi][di] */
  void *k_cache;        /* [batch][Hkv][kv_cap][d] */
  void *v_cache;        /* [batch][Hkv][kv_cap][d] */
  void *ki_cache;       /* [batch][kv_cap][di] */
  float *kbar_cache;    /* [batch][kv_cap / B][di] fp32: indexer state */
  int32_t *kbar_blocks; /* [batch] compressed blocks held in kbar_cache: indexer state */
  const void *k_new;    /* decode: [batch][Hkv][d], appended at kv_len - 1 */
  const void *v_new;    /* decode: [batch][Hkv][d] */
  const void *ki_new;   /* decode: [batch][di] */
  const int32_t *kv_start, *kv_len, *q_first; /* [batch]; q_first unused in decode */
  int32_t *sel;         /* [batch][n_q][k] out */
  void *out;            /* [batch][n_q][Hq][d] out */
} qsa_tensors_t;

/* Checks a config (Qwen4ExpTextConfig, indexer fields all-or-nothing; indexer_kv_heads
 * must be 1). Returns QSA_OK, QSA_ERR_INVALID_ARG or QSA_ERR_UNSUPPORTED. */
qsa_status_t qsa_config_validate(const qsa_config_t *cfg);

/* Blocks kept per query, k = indexer_budget / indexer_compress_ratio (0 on a bad config). */
int32_t qsa_topk_blocks(const qsa_config_t *cfg);

/* Static description of a status code; never NULL. */
const char *qsa_status_string(qsa_status_t status);

/* Bytes of workspace the calls below need for these sizes (mode QSA_PREFILL or
 * QSA_DECODE). The workspace is caller-owned device memory, 256-byte aligned, and
 * must be all zero before its first use; the library leaves the parts it relies on
 * at zero again after each call, except after a call whose device wait ran out
 * (status QSA_ERR_TIMEOUT): zero the workspace again before reusing it. Its first
 * 256 bytes hold the status word (qsa_read_device_status reads and clears it) and the
 * prefill attention's unit counters. One workspace must not serve two
 * calls that run concurrently. */
qsa_status_t qsa_workspace_size(const qsa_config_t *cfg, int32_t mode, int32_t batch, int32_t n_q,
                                int32_t kv_cap, size_t *bytes);

/* Step 1, block compression (Qwen4ExpTextConfig indexer_compress_ratio: B consecutive
 * indexer keys averaged into one block). For each sequence writes kbar[b][j] for the
 * complete blocks blocks_done[b] <= j < kv_len[b] / B (blocks_done may be NULL: all
 * complete blocks). fp32 sum in key order, then divided by B. kbar_blocks (may be
 * NULL) receives kv_len[b] / B, the count of compressed blocks the indexer state
 * then holds -- what a decode step expects in qsa_tensors_t.kbar_blocks when the
 * cache holds kv_len[b] tokens. */
qsa_status_t qsa_compress_blocks(const qsa_config_t *cfg, const void *ki, const int32_t *kv_start,
                                 const int32_t *kv_len, const int32_t *blocks_done, int32_t batch,
                                 int32_t kv_cap, float *kbar, int32_t *kbar_blocks, qsa_stream_t stream);

/* Steps 2 and 3, scoring and causal top-k selection (intro paragraph: multiple query
 * heads score compressed key blocks, the most relevant blocks are selected;
 * indexer_budget). Writes sel[b][r][0..k) for every query row: the selected complete
 * blocks in ascending order, -1 padded; padding rows are all -1. Scores are fp32;
 * ties go to the lower block index. */
qsa_status_t qsa_index_score_topk(const qsa_config_t *cfg, const void *qi, const float *kbar,
                                  const int32_t *kv_len, const int32_t *q_first, int32_t batch,
                                  int32_t n_q, int32_t kv_cap, int32_t *sel, void *workspace,
                                  size_t workspace_bytes, qsa_stream_t stream);

/* Step 4, exact attention over the selected tokens (Usage tips: sparse token selection
 * with ordinary softmax attention; num_key_value_heads: grouped-query attention).
 * Query row r of sequence b attends the blocks listed in sel[b][r] plus its trailing
 * range [n_c * B, t]. out rows of padding queries are zero. Accumulation is fp32;
 * bf16 outputs are rounded once at the end. */
qsa_status_t qsa_sparse_attn(const qsa_config_t *cfg, const void *q, const void *k, const void *v,
                             const int32_t *sel, const int32_t *kv_start, const int32_t *kv_len,
                             const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap,
                             void *out, void *workspace, size_t workspace_bytes,
                             qsa_stream_t stream);

/* The steps before the path: input projections and rotary position embedding
 * ("Qwen4-Exp" Qwen4ExpTextConfig: hidden_size; attention_bias = False, so no bias;
 * rope_parameters holding rope_theta; the head counts and dims of qsa_config_t).
 * Readings (the page fixes neither): RoPE in rotate-half form on the first rotary_dim
 * dims of every q and k head -- dims (i, i + r/2), i < r/2, turn by
 * pos * rope_theta^(-2i/r) -- and, with indexer_rotary_dim > 0, likewise on the
 * indexer query heads and the indexer key head; v is never rotated. */
typedef struct {
  int32_t hidden_size;        /* D: length of an input row and of every weight row; multiple of 64 */
  float rope_theta;           /* base of the rotary frequencies (rope_parameters["rope_theta"]) */
  int32_t rotary_dim;         /* dims of each q / k head that rotate: multiple of 32, <= head_dim */
  int32_t indexer_rotary_dim; /* same for the indexer heads (<= indexer_head_dim); 0: they do not rotate */
} qsa_proj_config_t;

/* Projects the token rows x [batch][n_tok][D] (bf16) by the stacked weight rows
 * w [Hq*d + 2*Hkv*d + Hi*di + di][D] (bf16: W_q, W_k, W_v, W_qi, W_ki one after the
 * other, each [out][D]) in fp32, applies RoPE at position q_first[b] + r to token row r
 * of sequence b, and writes bf16: q [batch][n_tok][Hq][d], qi [batch][n_tok][Hi][di],
 * and k, v [batch][Hkv][kv_cap][d], ki [batch][kv_cap][di] at storage row kv_row0 + r.
 * Prefill: q_first as for qsa_forward (-pad), kv_cap = n_tok, kv_row0 = 0. A decode
 * step: n_tok = 1, q_first[b] = kv_len[b] - 1, and k / v / ki are qsa_tensors_t's
 * k_new / v_new / ki_new (kv_cap = 1, kv_row0 = 0). Runs on tcgen05 tensor cores;
 * bf16 only, head_dim and indexer_head_dim multiples of 64 up to 256. Returns
 * QSA_ERR_UNSUPPORTED for other shapes. workspace: at least the 256-byte status word. */
qsa_status_t qsa_project(const qsa_config_t *cfg, const qsa_proj_config_t *pc, const void *x, const void *w,
                         const int32_t *q_first, int32_t batch, int32_t n_tok, void *q, void *qi, void *k,
                         void *v, void *ki, int32_t kv_cap, int32_t kv_row0, void *workspace,
                         size_t workspace_bytes, qsa_stream_t stream);

/* Head-sharded tensor parallelism ("Qwen4-Exp" Usage tips: tp_plan="auto" shards QSA;
 * the QSA projection dims must be divisible by the TP size). The block score is a sum
 * over indexer heads, so a rank holding a shard of the indexer query heads computes a
 * partial score; the partials summed over ranks (an all-reduce of the score matrix,
 * the caller's collective) are the full scores, from which every rank selects the same
 * blocks and attends its own shard of query / KV heads with qsa_sparse_attn.
 *
 * qsa_index_scores: step 2 alone. With cfg describing this rank's shard
 * (indexer_n_heads = the shard's head count, qi holding those heads), writes
 * scores[b][r][j] = sum over the shard's heads h of max(0, qi[b][r][h] . kbar[b][j])
 * for j < n_c(t) of every real query row; entries j >= n_c(t) and padding rows are not
 * written (they are never read by qsa_select_topk). Layout scores [batch][n_q][kv_cap / B]
 * fp32, device memory, 16-byte aligned. bf16 shapes with many rows run on the tensor
 * cores with the same precision as qsa_index_score_topk (kbar as a bf16 hi/lo pair);
 * others in fp32 on CUDA cores. workspace as for qsa_index_score_topk.
 *
 * qsa_select_topk: step 3 alone. Reads each real row's n_c(t) scores (any finite
 * fp32 values; -0 counts as +0) and writes sel[b][r][0..k) exactly as
 * qsa_index_score_topk does: the k best blocks by (-score, block id), ascending, -1
 * padded; padding rows all -1. workspace: at least the 256-byte status word. */
qsa_status_t qsa_index_scores(const qsa_config_t *cfg, const void *qi, const float *kbar, const int32_t *kv_len,
                              const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap, float *scores,
                              void *workspace, size_t workspace_bytes, qsa_stream_t stream);
qsa_status_t qsa_select_topk(const qsa_config_t *cfg, const float *scores, const int32_t *kv_len,
                             const int32_t *q_first, int32_t batch, int32_t n_q, int32_t kv_cap, int32_t *sel,
                             void *workspace, size_t workspace_bytes, qsa_stream_t stream);

/* The whole path.
 * QSA_PREFILL: compress every complete block of each prompt into kbar_cache (and set
 *   kbar_blocks[b] = kv_len[b] / B), then score, select and attend all n_q query rows.
 * QSA_DECODE (n_q == 1): kv_len[b] is the length AFTER this step's token. Appends
 *   k_new / v_new / ki_new at relative position kv_len[b] - 1; if that completes a
 *   block, compresses it; then scores, selects and attends the query at kv_len[b] - 1.
 *   The indexer state must be in step: kbar_blocks[b] == (kv_len[b] - 1) / B. A smaller
 *   kv_len (cache cropping, unsupported with QSA per the Usage tips) records
 *   QSA_ERR_UNSUPPORTED in the status word and leaves that sequence untouched. */
qsa_status_t qsa_forward(const qsa_config_t *cfg, int32_t mode, const qsa_tensors_t *t,
                         void *workspace, size_t workspace_bytes, qsa_stream_t stream);

/* Synchronises `stream`, returns the first device-side status recorded in the
 * workspace since the last read (QSA_OK if none) in *status, and clears it. */
qsa_status_t qsa_read_device_status(void *workspace, qsa_stream_t stream, qsa_status_t *status);

/* Library ABI version (QSA_ABI_VERSION) and the name of the kernel family that
 * qsa_sparse_attn would launch for this config in this mode (QSA_PREFILL: many query
 * rows; QSA_DECODE: one row per sequence): "tcgen05" (head_dim 128), "tcgen05
 * one-tile" (head_dim 256), "split-kv decode" (decode, head_dim 128, B = 64, G <= 8)
 * or "simt" (fp32 and every other shape). */
int32_t qsa_abi_version(void);
const char *qsa_attn_kernel_name(const qsa_config_t *cfg, int32_t mode);

/* Number of kernels this library has launched in the process so far (a host-side
 * counter bumped at every launch; diagnostics and benchmarking). */
uint64_t qsa_kernel_launch_count(void);

/* Text of the last CUDA error this library saw on the calling thread ("" if none). */
const char *qsa_last_error(void);

/* Self-test of the bounded device waits (failure detection): enqueues one CTA that
 * waits on a barrier nothing completes, gives up after limit_ns (1 ms .. 5 s) and
 * records QSA_ERR_TIMEOUT in the workspace status word, exactly as a pipelined
 * kernel does when a copy never lands. Read the result with qsa_read_device_status;
 * the CUDA context stays usable. */
qsa_status_t qsa_selftest_wait_timeout(void *workspace, int64_t limit_ns, qsa_stream_t stream);

/* Size of the fixed device array that qsa_sparse_attn_decode_noalloc uses. */
#define QSA_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)

/* Decode attention (step 4 for one query row per sequence, at kv_len[b] - 1) for
 * callers that cannot hand the library any device memory besides their inputs and
 * outputs -- for example a plugin that its host framework calls with nothing but
 * input and output buffers, or a serving process that reserves all device memory
 * for its own pool, so that a cudaMalloc would fail or go around that pool. It
 * computes what qsa_sparse_attn computes for n_q == 1 with q_first[b] = kv_len[b] - 1,
 * and allocates nothing: a status word and the split partials of the decode kernel
 * live in a fixed array of QSA_NOALLOC_SCRATCH_BYTES inside the library, which every
 * GPU that loads the library holds until the process exits (the paper has no
 * counterpart; this is an interface convenience).
 *   Arguments and layouts as for qsa_sparse_attn with n_q = 1 (q, out [batch][1][Hq][d];
 *   k, v [batch][Hkv][kv_cap][d]; sel [batch][1][k]); bf16, head_dim 128, B = 64, G <= 8.
 *   Each call looks up the array's device address on the current device (a host-side
 *   lookup; the first one on a device may load the library's device code, so make
 *   that first call before any stream capture), then enqueues on `stream` a clear of
 *   the array's status word and unit counters followed by the kernel: a call never
 *   sees what an earlier one left there.
 *   Every call on a device shares the one array; calls that overlap on the GPU (e.g.
 *   on two streams) race on it and must be serialised by the caller.
 *   Returns QSA_ERR_UNSUPPORTED (and sets qsa_last_error) when the partials of this
 *   batch exceed the array -- with batch * Hkv <= 2048 they take about
 *   (batch * Hkv + 1024) * G * (d + 2) * 4 bytes, which fits up to that limit for
 *   G = 8, d = 128 -- and for shapes the decode kernel does not serve. The caller
 *   cannot read the array's status word: lengths that do not fit the cache are
 *   skipped, and a device wait that runs out (each is bounded at 2 s) leaves that
 *   call's output rows unspecified, without a report. */
qsa_status_t qsa_sparse_attn_decode_noalloc(const qsa_config_t *cfg, const void *q, const void *k,
                                            const void *v, const int32_t *sel, const int32_t *kv_start,
                                            const int32_t *kv_len, int32_t batch, int32_t kv_cap, void *out,
                                            qsa_stream_t stream);

/* Cache offloading for decode ("Qwen4-Exp" Usage tips: the indexer state is kept
 * apart from the attention K/V cache). The attention K/V cache lives in host memory;
 * the indexer state (ki_cache, kbar_cache, kbar_blocks) and everything else stay on
 * the device, and only the blocks a step attends cross the host link.
 *
 * qsa_offload_staging_size: bytes of the device staging buffer that
 * qsa_decode_offload needs for `batch` sequences -- K and V of (k + 1) * B tokens per
 * (sequence, KV head) plus the remapped selection and lengths. Caller-owned device
 * memory, 256-byte aligned, no initialisation needed.
 *
 * qsa_decode_offload: the QSA_DECODE step of qsa_forward with t->k_cache and
 * t->v_cache in page-locked host memory (cudaHostAlloc or cudaHostRegister; device
 * memory also works). Appends k_new / v_new at kv_len - 1 in the host cache and
 * ki_new in the device indexer cache, compresses a completed block, scores and
 * selects on the device, copies the selected blocks and the trailing block of every
 * (sequence, KV head) into the staging buffer, and attends there. out and sel equal
 * what qsa_forward(QSA_DECODE) gives for the same inputs.
 *   Returns QSA_ERR_INVALID_ARG if a cache pointer is pageable host memory (the device
 *   cannot reach it) or the staging or workspace buffer is too small; otherwise as
 *   qsa_forward. The workspace is sized as for qsa_forward(QSA_DECODE). */
qsa_status_t qsa_offload_staging_size(const qsa_config_t *cfg, int32_t batch, size_t *bytes);
qsa_status_t qsa_decode_offload(const qsa_config_t *cfg, const qsa_tensors_t *t, void *staging,
                                size_t staging_bytes, void *workspace, size_t workspace_bytes,
                                qsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */
