// C ABI of liblime.so: argument checks, workspace layout and kernel dispatch.
// Every numeric step runs in the kernels of the other files.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "lime_fast.cuh"
#include "lime_simt.cuh"

using namespace lime;

namespace lime {
static std::atomic<uint64_t> g_launches{0};
int check_cache_args(const lime_dims* dims, const void* T, int64_t n_items, const void* L,
                     const void* Wq_c, const void* Wk_c, const void* cache_out);
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace lime

namespace {

constexpr size_t kStatusBytes = 256;  // status word + padding at the workspace head

bool dims_ok(const lime_dims* D) {
  if (!D) return false;
  if (D->dtype != LIME_F32 && D->dtype != LIME_BF16) return false;
  if (D->phi != LIME_PHI_SOFTMAX && D->phi != LIME_PHI_SILU) return false;
  if (D->window < 0 || D->window > 64) return false;
  return true;
}

// LIME_OK, or LIME_ERR_ARG / LIME_ERR_SHAPE for unusable sizes.
int check_dims(const lime_dims* D) {
  if (!dims_ok(D)) return LIME_ERR_ARG;
  if (D->d <= 0 || D->H <= 0 || D->l <= 0 || D->f <= 0 || D->c < 0) return LIME_ERR_ARG;
  if (D->d % D->H != 0 || D->d % 8 != 0 || D->d > 256) return LIME_ERR_SHAPE;
  const int dh = D->d / D->H;
  if (dh != 16 && dh != 32 && dh != 64) return LIME_ERR_SHAPE;
  if (D->l > 128 || D->f % 8 != 0 || D->f > 1024 || D->c > 256) return LIME_ERR_SHAPE;
  return LIME_OK;
}

size_t esize(const lime_dims* D) { return D->dtype == LIME_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

int launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "liblime: %s: %s\n", what, cudaGetErrorString(e));
    return LIME_ERR_CUDA;
  }
  return LIME_OK;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t scratch_bytes(const lime_dims* D, int64_t B, int64_t total_hist) {
  size_t s = simt_cache_ws_bytes(*D);
  // the CUDA-core layer path needs fp32 row buffers; the tensor-core path does not
  size_t t = fast_layer_supported(*D) ? 0 : simt_layer_ws_bytes(*D, B, total_hist);
  if (t > s) s = t;
  size_t u = fast_ws_bytes(*D, B, total_hist);
  if (u > s) s = u;
  return round256(s);
}

int check_ws(void* ws, size_t ws_bytes, const lime_dims* D, int64_t B, int64_t total_hist) {
  if (!ws || ((uintptr_t)ws & 255)) return LIME_ERR_ARG;
  if (ws_bytes < kStatusBytes + scratch_bytes(D, B, total_hist)) return LIME_ERR_ARG;
  return LIME_OK;
}

unsigned* status_of(void* ws) { return (unsigned*)ws; }
float* scratch_of(void* ws) { return (float*)((char*)ws + kStatusBytes); }

}  // namespace

namespace lime {
// Argument checks of the QK-cache build, apart from the workspace: dims,
// sizes, null pointers, 16-byte alignment and output/input aliasing.
int check_cache_args(const lime_dims* dims, const void* T, int64_t n_items, const void* L,
                     const void* Wq_c, const void* Wk_c, const void* cache_out) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n_items < 0 || n_items > (int64_t)INT32_MAX + 1) return LIME_ERR_ARG;
  if (!L || !Wq_c || !Wk_c || (n_items > 0 && (!T || !cache_out))) return LIME_ERR_ARG;
  if ((n_items > 0 && (!aligned16(T) || !aligned16(cache_out))) || !aligned16(L) ||
      !aligned16(Wq_c) || !aligned16(Wk_c))
    return LIME_ERR_ARG;
  const size_t es = esize(dims);
  const size_t cache_sz = (size_t)n_items * dims->H * dims->l * es;
  if (overlap(cache_out, cache_sz, T, (size_t)n_items * dims->d * es) ||
      overlap(cache_out, cache_sz, L, (size_t)dims->l * dims->d * es) ||
      overlap(cache_out, cache_sz, Wq_c, (size_t)dims->d * dims->d * es) ||
      overlap(cache_out, cache_sz, Wk_c, (size_t)dims->d * dims->d * es))
    return LIME_ERR_ALIAS;
  return LIME_OK;
}
}  // namespace lime

extern "C" {

size_t lime_workspace_bytes(const lime_dims* dims, int64_t B, int64_t total_hist) {
  if (check_dims(dims) != LIME_OK || B < 0 || total_hist < 0) return 0;
  return kStatusBytes + scratch_bytes(dims, B, total_hist);
}

int lime_workspace_init(void* workspace, size_t bytes, cudaStream_t stream) {
  if (!workspace || bytes < kStatusBytes || ((uintptr_t)workspace & 255)) return LIME_ERR_ARG;
  if (cudaMemsetAsync(workspace, 0, kStatusBytes, stream) != cudaSuccess) return LIME_ERR_CUDA;
  return LIME_OK;
}

int lime_build_qk_cache(const lime_dims* dims, const void* T, int64_t n_items, const void* L,
                        const void* Wq_c, const void* Wk_c, void* cache_out, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  int rc = lime::check_cache_args(dims, T, n_items, L, Wq_c, Wk_c, cache_out);
  if (rc) return rc;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  if (dims->dtype == LIME_BF16 && fast_cache_supported(*dims)) {
    rc = fast_build_qk_cache(*dims, T, n_items, L, Wq_c, Wk_c, cache_out,
                             scratch_of(workspace), status_of(workspace), stream);
    if (rc) return rc;
  } else if (dims->dtype == LIME_BF16) {
    simt_build_qk_cache<bf16>(*dims, T, n_items, L, Wq_c, Wk_c, cache_out, scratch_of(workspace),
                              stream);
  } else {
    simt_build_qk_cache<float>(*dims, T, n_items, L, Wq_c, Wk_c, cache_out,
                               scratch_of(workspace), stream);
  }
  return launch_status("lime_build_qk_cache");
}

int lime_context_links(const lime_dims* dims, int64_t B, const void* L, const void* ctx,
                       const lime_ctx_mlp* w, void* LC_out, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->c < 1) return LIME_ERR_SHAPE;
  if (B < 0 || B > INT32_MAX) return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  if (B == 0) return LIME_OK;
  if (!L || !ctx || !w || !LC_out || !w->Wc1 || !w->bc1 || !w->Wc2 || !w->bc2)
    return LIME_ERR_ARG;
  if (!aligned16(w->Wc1) || !aligned16(w->Wc2)) return LIME_ERR_ARG;
  const size_t es = esize(dims);
  const size_t out_sz = (size_t)B * dims->l * dims->d * es;
  if (overlap(LC_out, out_sz, L, (size_t)dims->l * dims->d * es) ||
      overlap(LC_out, out_sz, ctx, (size_t)B * dims->c * es))
    return LIME_ERR_ALIAS;
  if (fast_ctx_supported(*dims) && aligned16(L) && aligned16(ctx) && aligned16(LC_out)) {
    if ((rc = fast_context_links(*dims, B, L, ctx, *w, LC_out, status_of(workspace), stream)))
      return rc;
  } else if (dims->dtype == LIME_BF16)
    simt_context_links<bf16>(*dims, B, L, ctx, *w, LC_out, stream);
  else
    simt_context_links<float>(*dims, B, L, ctx, *w, LC_out, stream);
  return launch_status("lime_context_links");
}

int lime_xor_layer(const lime_dims* dims, int64_t B, const int64_t* hist_offsets,
                   int64_t total_hist, const void* E_in, const void* Z_in,
                   const lime_layer_w* w, void* E_out, void* Z_out, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (B < 0 || B > INT32_MAX || total_hist < 0 || total_hist > INT32_MAX) return LIME_ERR_ARG;
  if (B == 0) return total_hist == 0 ? LIME_OK : LIME_ERR_ARG;
  if (!hist_offsets || !Z_in || !Z_out || !w) return LIME_ERR_ARG;
  if (total_hist > 0 && !E_in) return LIME_ERR_ARG;
  const void* ptrs[] = {w->g1, w->b1, w->Wq, w->Wk, w->Wv, w->Wo, w->g2, w->b2, w->W1, w->W3, w->W2};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LIME_ERR_ARG;
  if (!aligned16(Z_in) || !aligned16(Z_out) || (E_in && !aligned16(E_in)) ||
      (E_out && !aligned16(E_out)) || ((uintptr_t)hist_offsets & 7))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, B, total_hist))) return rc;
  const size_t es = esize(dims);
  const size_t e_sz = (size_t)total_hist * dims->d * es, z_sz = (size_t)B * dims->l * dims->d * es;
  if (overlap(E_out, e_sz, E_in, e_sz) || overlap(E_out, e_sz, Z_in, z_sz) ||
      overlap(Z_out, z_sz, E_in, e_sz) || overlap(Z_out, z_sz, Z_in, z_sz) ||
      overlap(E_out, e_sz, Z_out, z_sz))
    return LIME_ERR_ALIAS;
  if (dims->dtype == LIME_BF16 && fast_layer_supported(*dims)) {
    rc = fast_xor_layer(*dims, B, hist_offsets, total_hist, E_in, Z_in, *w, E_out, Z_out,
                        scratch_of(workspace), status_of(workspace), stream);
    if (rc) return rc;
  } else if (dims->dtype == LIME_BF16) {
    simt_xor_layer<bf16>(*dims, B, hist_offsets, total_hist, E_in, Z_in, *w, E_out, Z_out,
                         scratch_of(workspace), status_of(workspace), stream);
  } else {
    simt_xor_layer<float>(*dims, B, hist_offsets, total_hist, E_in, Z_in, *w, E_out, Z_out,
                          scratch_of(workspace), status_of(workspace), stream);
  }
  return launch_status("lime_xor_layer");
}

int lime_score_candidates(const lime_dims* dims, int64_t B, const void* cache, int64_t n_items,
                          const int32_t* cand_ids, const int64_t* cand_offsets,
                          int64_t total_cand, const void* LP, void* O_out, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (B < 0 || B > INT32_MAX || n_items < 0 || total_cand < 0) return LIME_ERR_ARG;
  if (B == 0) return total_cand == 0 ? LIME_OK : LIME_ERR_ARG;
  if (!cand_offsets || !LP || ((uintptr_t)cand_offsets & 7)) return LIME_ERR_ARG;
  if (total_cand > 0 && (!cand_ids || !O_out || !cache)) return LIME_ERR_ARG;
  if (!aligned16(LP) || (O_out && !aligned16(O_out)) || (cache && !aligned16(cache)) ||
      ((uintptr_t)cand_ids & 3))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  const size_t es = esize(dims);
  const size_t o_sz = (size_t)total_cand * dims->d * es;
  if (overlap(O_out, o_sz, cache, (size_t)n_items * dims->H * dims->l * es) ||
      overlap(O_out, o_sz, LP, (size_t)B * dims->l * dims->d * es) ||
      overlap(O_out, o_sz, cand_ids, (size_t)total_cand * 4))
    return LIME_ERR_ALIAS;
  if (total_cand == 0) return LIME_OK;
  if (dims->dtype == LIME_BF16 && fast_score_supported(*dims)) {
    rc = fast_score(*dims, B, cache, n_items, cand_ids, cand_offsets, total_cand, LP, O_out,
                    scratch_of(workspace), status_of(workspace), stream);
    if (rc) return rc;
  } else if (dims->dtype == LIME_BF16) {
    simt_score<bf16>(*dims, B, cache, n_items, cand_ids, cand_offsets, total_cand, LP, O_out,
                     status_of(workspace), stream);
  } else {
    simt_score<float>(*dims, B, cache, n_items, cand_ids, cand_offsets, total_cand, LP, O_out,
                      status_of(workspace), stream);
  }
  return launch_status("lime_score_candidates");
}

int lime_score_candidates_uncached(const lime_dims* dims, int64_t B, const void* T,
                                   int64_t n_items, const void* image, const int32_t* cand_ids,
                                   const int64_t* cand_offsets, int64_t total_cand, const void* LP,
                                   void* O_out, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (dims->dtype != LIME_BF16 || !fast_online_supported(*dims) || !lime_qk_image_bytes(dims))
    return LIME_ERR_SHAPE;
  if (B < 0 || B > INT32_MAX || n_items < 0 || total_cand < 0) return LIME_ERR_ARG;
  if (B == 0) return total_cand == 0 ? LIME_OK : LIME_ERR_ARG;
  if (!cand_offsets || !LP || !image || ((uintptr_t)cand_offsets & 7)) return LIME_ERR_ARG;
  if (total_cand > 0 && (!cand_ids || !O_out || !T)) return LIME_ERR_ARG;
  if (!aligned16(LP) || !aligned16(image) || (O_out && !aligned16(O_out)) ||
      (T && !aligned16(T)) || ((uintptr_t)cand_ids & 3))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  const size_t es = esize(dims);
  const size_t o_sz = (size_t)total_cand * dims->d * es;
  if (overlap(O_out, o_sz, T, (size_t)n_items * dims->d * es) ||
      overlap(O_out, o_sz, image, lime_qk_image_bytes(dims)) ||
      overlap(O_out, o_sz, LP, (size_t)B * dims->l * dims->d * es) ||
      overlap(O_out, o_sz, cand_ids, (size_t)total_cand * 4))
    return LIME_ERR_ALIAS;
  if (total_cand == 0) return LIME_OK;
  if ((rc = fast_score_online(*dims, B, T, n_items, image, cand_ids, cand_offsets, total_cand, LP,
                              O_out, status_of(workspace), stream)))
    return rc;
  return launch_status("lime_score_candidates_uncached");
}

size_t lime_qk_image_bytes(const lime_dims* dims) {
  if (!dims || check_dims(dims) || dims->dtype != LIME_BF16 || !fast_cache_supported(*dims))
    return 0;
  return (size_t)2 * dims->d * dims->H * dims->l;
}

int lime_fold_qk(const lime_dims* dims, const void* L, const void* Wq_c, const void* Wk_c,
                 void* image, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!lime_qk_image_bytes(dims)) return LIME_ERR_SHAPE;
  if (!L || !Wq_c || !Wk_c || !image) return LIME_ERR_ARG;
  if (!aligned16(L) || !aligned16(Wq_c) || !aligned16(Wk_c) || !aligned16(image))
    return LIME_ERR_ARG;
  const size_t es = esize(dims), img = lime_qk_image_bytes(dims);
  if (overlap(image, img, L, (size_t)dims->l * dims->d * es) ||
      overlap(image, img, Wq_c, (size_t)dims->d * dims->d * es) ||
      overlap(image, img, Wk_c, (size_t)dims->d * dims->d * es))
    return LIME_ERR_ALIAS;
  if ((rc = fast_fold_qk(*dims, L, Wq_c, Wk_c, image, stream))) return rc;
  return launch_status("lime_fold_qk");
}

int lime_build_qk_cache_folded(const lime_dims* dims, const void* T, int64_t n_items,
                               const void* image, void* cache_out, int32_t tiles_per_cta,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!lime_qk_image_bytes(dims)) return LIME_ERR_SHAPE;
  if (n_items < 0 || n_items > (int64_t)INT32_MAX + 1 || tiles_per_cta < 0) return LIME_ERR_ARG;
  if (!image || (n_items > 0 && (!T || !cache_out))) return LIME_ERR_ARG;
  if (!aligned16(image) || (n_items > 0 && (!aligned16(T) || !aligned16(cache_out))))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  const size_t es = esize(dims);
  const size_t cache_sz = (size_t)n_items * dims->H * dims->l * es;
  if (overlap(cache_out, cache_sz, T, (size_t)n_items * dims->d * es) ||
      overlap(cache_out, cache_sz, image, lime_qk_image_bytes(dims)) ||
      overlap(workspace, workspace_bytes, image, lime_qk_image_bytes(dims)) ||
      overlap(workspace, workspace_bytes, cache_out, cache_sz))
    return LIME_ERR_ALIAS;
  if ((rc = fast_build_qk_cache_folded(*dims, T, n_items, image, cache_out, tiles_per_cta,
                                       status_of(workspace), stream)))
    return rc;
  return launch_status("lime_build_qk_cache_folded");
}

int lime_build_qk_cache_u8(const lime_dims* dims, const void* T, int64_t n_items, const void* L,
                           const void* Wq_c, const void* Wk_c, uint8_t* cache_out,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!fast_cache_u8_supported(*dims) || dims->phi != LIME_PHI_SOFTMAX) return LIME_ERR_SHAPE;
  if (n_items < 0 || n_items > (int64_t)INT32_MAX + 1) return LIME_ERR_ARG;
  if (!L || !Wq_c || !Wk_c || (n_items > 0 && (!T || !cache_out))) return LIME_ERR_ARG;
  if ((n_items > 0 && (!aligned16(T) || !aligned16(cache_out))) || !aligned16(L) ||
      !aligned16(Wq_c) || !aligned16(Wk_c))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  const size_t es = esize(dims);
  const size_t cache_sz = (size_t)n_items * dims->H * dims->l;
  if (overlap(cache_out, cache_sz, T, (size_t)n_items * dims->d * es) ||
      overlap(cache_out, cache_sz, L, (size_t)dims->l * dims->d * es) ||
      overlap(cache_out, cache_sz, Wq_c, (size_t)dims->d * dims->d * es) ||
      overlap(cache_out, cache_sz, Wk_c, (size_t)dims->d * dims->d * es))
    return LIME_ERR_ALIAS;
  if ((rc = fast_build_qk_cache_u8(*dims, T, n_items, L, Wq_c, Wk_c, cache_out,
                                   scratch_of(workspace), status_of(workspace), stream)))
    return rc;
  return launch_status("lime_build_qk_cache_u8");
}

int lime_score_candidates_u8(const lime_dims* dims, int64_t B, const uint8_t* cache,
                             int64_t n_items, const int32_t* cand_ids,
                             const int64_t* cand_offsets, int64_t total_cand, const void* LP,
                             void* O_out, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!fast_score_u8_supported(*dims)) return LIME_ERR_SHAPE;
  if (B < 0 || B > INT32_MAX || n_items < 0 || total_cand < 0) return LIME_ERR_ARG;
  if (B == 0) return total_cand == 0 ? LIME_OK : LIME_ERR_ARG;
  if (!cand_offsets || !LP || ((uintptr_t)cand_offsets & 7)) return LIME_ERR_ARG;
  if (total_cand > 0 && (!cand_ids || !O_out || !cache)) return LIME_ERR_ARG;
  if (!aligned16(LP) || (O_out && !aligned16(O_out)) || (cache && !aligned16(cache)) ||
      ((uintptr_t)cand_ids & 3))
    return LIME_ERR_ARG;
  if ((rc = check_ws(workspace, workspace_bytes, dims, 0, 0))) return rc;
  const size_t es = esize(dims);
  const size_t o_sz = (size_t)total_cand * dims->d * es;
  if (overlap(O_out, o_sz, cache, (size_t)n_items * dims->H * dims->l) ||
      overlap(O_out, o_sz, LP, (size_t)B * dims->l * dims->d * es) ||
      overlap(O_out, o_sz, cand_ids, (size_t)total_cand * 4))
    return LIME_ERR_ALIAS;
  if (total_cand == 0) return LIME_OK;
  if ((rc = fast_score_u8(*dims, B, cache, n_items, cand_ids, cand_offsets, total_cand, LP, O_out,
                          status_of(workspace), stream)))
    return rc;
  return launch_status("lime_score_candidates_u8");
}

int lime_get_status(void* workspace, cudaStream_t stream, int* flags) {
  if (!workspace || !flags || ((uintptr_t)workspace & 255)) return LIME_ERR_ARG;
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return LIME_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LIME_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(unsigned), stream) != cudaSuccess) return LIME_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LIME_ERR_CUDA;
  *flags = (int)v;
  return LIME_OK;
}

uint64_t lime_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
