// Stage 1 of MSA: offline memory encoding (placeholder until the tcgen05 path lands).
#include "internal.h"

namespace msa {
struct EncodeWs {};
size_t encode_workspace(const msa_dims&, int64_t, int, int, void*, EncodeWs*) { return 0; }
msa_status encode_launch(const msa_dims&, const void*, int64_t, const int64_t*, int, const int32_t*, int,
                         const void*, const void*, const void*, void*, void*, void*, void*, cudaStream_t) {
  return fail(MSA_ERR_UNSUPPORTED, "msa_encode_memory is not available in this build");
}
}  // namespace msa
