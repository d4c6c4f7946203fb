#include "lime_fast.cuh"
namespace lime {
size_t fast_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist) {
  size_t a = fast_cache_ws_bytes(D), b = fast_layer_ws_bytes(D, B, total_hist);
  return a > b ? a : b;
}
bool fast_score_supported(const lime_dims&) { return false; }
int fast_score(const lime_dims&, int64_t, const void*, int64_t, const int32_t*, const int64_t*,
               int64_t, const void*, void*, float*, unsigned*, cudaStream_t) { return LIME_ERR_SHAPE; }
}
