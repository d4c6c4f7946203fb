#include "lime_fast.cuh"
namespace lime {
size_t fast_ws_bytes(const lime_dims& D, int64_t, int64_t) { return fast_cache_ws_bytes(D); }
bool fast_score_supported(const lime_dims&) { return false; }
int fast_score(const lime_dims&, int64_t, const void*, int64_t, const int32_t*, const int64_t*,
               int64_t, const void*, void*, float*, unsigned*, cudaStream_t) { return LIME_ERR_SHAPE; }
bool fast_layer_supported(const lime_dims&) { return false; }
int fast_xor_layer(const lime_dims&, int64_t, const int64_t*, int64_t, const void*, const void*,
                   const lime_layer_w&, void*, void*, float*, unsigned*, cudaStream_t) { return LIME_ERR_SHAPE; }
}
