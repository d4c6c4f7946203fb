// Scratch needed by the tensor-core paths: the largest of the cache build's
// folded-weight image and the XOR layer's buffers (scoring needs none).
#include "lime_fast.cuh"

namespace lime {

size_t fast_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist) {
  const size_t a = fast_cache_ws_bytes(D), b = fast_layer_ws_bytes(D, B, total_hist);
  return a > b ? a : b;
}

}  // namespace lime
