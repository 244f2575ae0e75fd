// Split-KV decode attention (placeholder until the decode kernel lands).
#include "qsa_internal.h"

namespace qsa {
bool attn_decode_supported(const Dims &) { return false; }
size_t attn_decode_workspace(const Dims &, const Seqs &) { return 0; }
cudaError_t launch_attn_decode(const Dims &, const Seqs &, const void *, const void *, const void *,
                               const int32_t *, void *, void *, size_t, int *, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace qsa
