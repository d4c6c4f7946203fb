// Tensor-core (tcgen05) and vectorised bf16 kernels of the LIME hot path.
#pragma once
#include "lime_common.cuh"

namespace lime {

// Launches a kernel that follows the pdl_launch / pdl_wait protocol with
// programmatic stream serialization (its launch and prologue overlap the
// previous kernel's tail), optionally as clusters of cluster_y CTAs along y.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, unsigned cluster_y, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  // the stream's priority travels with the launch (and into a captured graph's
  // kernel node), so a low-priority stream's CTAs yield SMs to a high one's
  int prio = 0;
  if (cudaStreamGetPriority(st, &prio) == cudaSuccess && prio != 0) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = prio;
    ++n;
  }
  if (cluster_y > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = cluster_y;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) return LIME_ERR_CUDA;
  note_launches(1);
  return LIME_OK;
}

size_t fast_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist);
size_t fast_cache_ws_bytes(const lime_dims& D);
size_t fast_layer_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist);

bool fast_cache_supported(const lime_dims& D);
int fast_build_qk_cache(const lime_dims& D, const void* T, int64_t n, const void* L,
                        const void* Wq, const void* Wk, void* cache, float* ws,
                        unsigned* status, cudaStream_t st);

// the two stages of fast_build_qk_cache (bf16 cache): G^T image, catalogue
int fast_fold_qk(const lime_dims& D, const void* L, const void* Wq, const void* Wk, void* image,
                 cudaStream_t st);
int fast_build_qk_cache_folded(const lime_dims& D, const void* T, int64_t n, const void* image,
                               void* cache, int tiles_per_cta, unsigned* status, cudaStream_t st);

// uncached (online) scoring from the item table and the folded G image
bool fast_online_supported(const lime_dims& D);
int fast_score_online(const lime_dims& D, int64_t B, const void* T, int64_t n_items,
                      const void* image, const int32_t* ids, const int64_t* off, int64_t total,
                      const void* LP, void* O, unsigned* status, cudaStream_t st);

// int8 cache (bytes q = round(255 w)); needs H*l >= 128
bool fast_cache_u8_supported(const lime_dims& D);
int fast_build_qk_cache_u8(const lime_dims& D, const void* T, int64_t n, const void* L,
                           const void* Wq, const void* Wk, void* cache, float* ws,
                           unsigned* status, cudaStream_t st);

bool fast_score_supported(const lime_dims& D);
int fast_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
               const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
               float* ws, unsigned* status, cudaStream_t st);

bool fast_ctx_supported(const lime_dims& D);
int fast_context_links(const lime_dims& D, int64_t B, const void* L, const void* ctx,
                       const lime_ctx_mlp& w, void* LC, unsigned* status, cudaStream_t st);

bool fast_score_u8_supported(const lime_dims& D);
int fast_score_u8(const lime_dims& D, int64_t B, const uint8_t* cache, int64_t n_items,
                  const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
                  unsigned* status, cudaStream_t st);

bool fast_layer_supported(const lime_dims& D);
int fast_xor_layer(const lime_dims& D, int64_t B, const int64_t* off, int64_t nh,
                   const void* E_in, const void* Z_in, const lime_layer_w& w, void* E_out,
                   void* Z_out, float* ws, unsigned* status, cudaStream_t st);

}  // namespace lime
