// Causal MuSe with retrieval (placeholder).
#include "internal.h"

namespace muse {
size_t muse_retrieval_ws(const muse_dims &, int, int, int, int, int) { return 0; }
}  // namespace muse

extern "C" muse_status muse_retrieve_exact(const void *, const void *, const void *, muse_dims,
                                           int, int, int, int, int, int, int32_t *, int32_t *,
                                           int32_t *, void *, void *, size_t, muse_stream_t) {
  return MUSE_ERR_SHAPE;
}
