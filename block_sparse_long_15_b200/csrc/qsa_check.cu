// Device-side checks of a selection list (the QSA_DEBUG build runs them before every
// attention launch): for each query row, the ids in sel[b][r][0 .. k) are the row's
// min(n_c, k) selected complete blocks -- each in [0, n_c), strictly ascending, so
// unique -- followed by -1 padding; a padding row holds -1 only (Hugging Face
// Transformers model doc "Qwen4-Exp", intro paragraph on QSA: the selected blocks
// are complete blocks before the query's trailing block). A violation records
// QSA_ERR_DEVICE_CHECK in the status word; nothing traps. The attention kernels skip
// ids outside [0, n_c) on their own, so a bad list never leads them out of bounds.
#include "qsa_internal.h"

namespace qsa {
namespace {

__global__ void k_validate_sel(Dims D, Seqs S, const int32_t *__restrict__ sel, int *status) {
  const long long rows = (long long)S.batch * S.n_q;
  for (long long row = blockIdx.x * (long long)blockDim.x + threadIdx.x; row < rows;
       row += (long long)gridDim.x * blockDim.x) {
    const int b = (int)(row / S.n_q), r = (int)(row % S.n_q);
    const int st = seq_start(S, b), len = S.kv_len[b];
    const bool geo = st >= 0 && len >= 0 && (long long)st + len <= (long long)S.kv_cap;
    const int t = seq_qfirst(S, b) + r;
    const int n_c = (geo && t >= 0 && t < len) ? (t + 1) / D.B : 0;
    const int want = n_c < D.k ? n_c : D.k;
    const int32_t *s = sel + (size_t)row * D.k;
    bool ok = true;
    int prev = -1;
    for (int i = 0; i < D.k; ++i) {
      const int j = s[i];
      if (i < want) {
        ok = ok && j > prev && j < n_c;
        prev = j;
      } else {
        ok = ok && j == -1;
      }
    }
    if (!ok) record_status(status, QSA_ERR_DEVICE_CHECK);
  }
}

}  // namespace

cudaError_t launch_validate_sel(const Dims &D, const Seqs &S, const int32_t *sel, int *status, cudaStream_t st) {
  const long long rows = (long long)S.batch * S.n_q;
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + 255) / 256;
  note_launch();
  k_validate_sel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(D, S, sel, status);
  return cudaGetLastError();
}

}  // namespace qsa
