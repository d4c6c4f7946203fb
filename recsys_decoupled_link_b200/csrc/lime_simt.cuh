// Launchers of the generic CUDA-core kernels (simt_kernels.cu).
#pragma once
#include "lime_common.cuh"

namespace lime {

size_t simt_layer_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist);
size_t simt_cache_ws_bytes(const lime_dims& D);

template <class T>
void simt_context_links(const lime_dims& D, int64_t B, const void* L, const void* ctx,
                        const lime_ctx_mlp& w, void* LC, cudaStream_t st);
template <class T>
void simt_xor_layer(const lime_dims& D, int64_t B, const int64_t* off, int64_t nh,
                    const void* E_in, const void* Z_in, const lime_layer_w& w, void* E_out,
                    void* Z_out, float* ws, unsigned* status, cudaStream_t st);
template <class T>
void simt_build_qk_cache(const lime_dims& D, const void* Tm, int64_t n, const void* L,
                         const void* Wq, const void* Wk, void* cache, float* ws,
                         cudaStream_t st);
template <class T>
void simt_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
                const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
                unsigned* status, cudaStream_t st);

}  // namespace lime
