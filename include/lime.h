/*
 * lime.h — C ABI of liblime.so, the B200 (sm_100a) hot path of LIME:
 * link embeddings with decoupled XOR attention for recommendation.
 *
 * Sources, by page title and section:
 *   LIME note    = papernotes.org, "LIME: 基于解耦XOR注意力与全局链接嵌入的测试期
 *                  高效扩展推荐模型" (整体框架, 关键设计 1-3, 一个完整示例,
 *                  损失函数 / 训练策略).
 *   LIME listing = thelatestinai.com, "LIME: Link-based User-item Interaction
 *                  Modeling with Decoupled XOR Attention for Efficient Test
 *                  Time Scaling" (Figures 3-4, Tables 10, 12).
 *
 * Conventions shared by every call
 *   - Pointers marked "device" are CUDA device pointers owned by the caller.
 *     The library allocates nothing; scratch lives in the caller's workspace.
 *   - Every call is asynchronous on `stream`, except lime_get_status, which
 *     synchronises it.  Calls sharing one workspace must not overlap on the
 *     GPU (issue them on one stream).
 *   - dims->dtype applies to every floating-point tensor of a call
 *     (LIME_BF16: bf16 storage, fp32 accumulation and softmax statistics;
 *     LIME_F32: fp32 throughout).  Integer tensors are int32 (candidate IDs)
 *     and int64 (offsets).
 *   - Float tensors and the workspace start on 16- and 256-byte boundaries;
 *     offsets on 8-byte boundaries (ERR_ARG otherwise).
 *   - Matrices are row-major.  Weights are [d_in, d_out] and applied as x·W.
 *     Head h owns the d_h = d/H contiguous columns [h*d_h, (h+1)*d_h).
 *   - Jagged inputs are packed: user u owns rows [off[u], off[u+1]) of the
 *     packed tensor; off has B+1 entries, off[0] = 0, off[B] = total.
 *   - Return value: LIME_OK or a negative LIME_ERR_* code.  On an error code
 *     nothing was launched.  Errors found on the device (a candidate ID out of
 *     range, offsets that are not monotone or do not end at `total`) do not
 *     abort: the kernel keeps every access in bounds (out-of-range IDs give a
 *     zero output row; user ranges are clamped into [0, total]) and sets a
 *     sticky LIME_FLAG_* bit in the workspace, read by lime_get_status.
 */
#ifndef LIME_H
#define LIME_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LIME_F32 = 0, LIME_BF16 = 1 } lime_dtype;

/* The attention weight function phi of both XOR branches and the candidate
 * side (LIME note, 关键设计 1: "scaled Softmax or SiLU"; 损失函数 / 训练策略:
 * softmax for single-layer models, SiLU in deep stacks).  LIME_PHI_SILU uses
 * SiLU of each scaled score divided by the number of keys the query may attend
 * to: l for a history query and for a candidate, N_u for a link query (the
 * pages state no normaliser; this keeps an average's scale).  The int8 cache
 * supports softmax only (SiLU weights can be negative).                     */
typedef enum { LIME_PHI_SOFTMAX = 0, LIME_PHI_SILU = 1 } lime_phi;

/* LIME-XOR+Window (LIME note, 关键设计 3): besides the l links, each history
 * token attends to the neighbouring history tokens of its own user, window
 * rows on each side (itself excluded, fewer at the ends of the history), all
 * in one phi over the union of keys; link queries are unchanged.  The pages'
 * variant has l neighbours in all: window = l / 2.  0 <= window <= 64; a
 * nonzero window runs the CUDA-core layer kernels.                          */

enum {
  LIME_OK = 0,
  LIME_ERR_ARG = -1,    /* null pointer, negative size, workspace too small  */
  LIME_ERR_SHAPE = -2,  /* d % H != 0, d_h or l outside the supported range  */
  LIME_ERR_ALIAS = -3,  /* an output overlaps an input it is computed from   */
  LIME_ERR_CUDA = -4    /* a CUDA launch or copy failed                       */
};

enum {
  LIME_FLAG_BAD_ID = 1,       /* a candidate ID was outside [0, n_items)       */
  LIME_FLAG_BAD_OFFSETS = 2,  /* offsets not monotone / not from 0 to total    */
  LIME_FLAG_TIMEOUT = 4       /* a bounded device-side wait gave up            */
};

/* Model sizes.  Supported: 1 <= H, d % H == 0, d % 8 == 0, d <= 256,
 * d_h = d/H in {16, 32, 64}, 1 <= l <= 128, f % 8 == 0, f <= 1024, 0 <= c <= 256. */
typedef struct {
  int32_t d;      /* model dim                                               */
  int32_t H;      /* attention heads                                         */
  int32_t l;      /* number of links (ell)                                   */
  int32_t f;      /* GatedMLP hidden width                                   */
  int32_t c;      /* user context feature dim (0: no context MLP)            */
  int32_t dtype;  /* lime_dtype                                              */
  int32_t phi;    /* lime_phi: the attention weight function (0 = softmax)   */
  int32_t window; /* LIME-XOR+Window: a history query also attends to the    */
                  /* user's history rows within this distance (0: XOR only) */
} lime_dims;

/* One LIME-XOR layer's parameters (device pointers, dims->dtype):
 * g1,b1,g2,b2 [d]; Wq,Wk,Wv,Wo [d,d]; W1,W3 [d,f]; W2 [f,d]. */
typedef struct {
  const void *g1, *b1, *Wq, *Wk, *Wv, *Wo, *g2, *b2, *W1, *W3, *W2;
} lime_layer_w;

/* Context-link MLP parameters (device, dims->dtype):
 * Wc1 [d+c, d], bc1 [d], Wc2 [d, d], bc2 [d]. */
typedef struct {
  const void *Wc1, *bc1, *Wc2, *bc2;
} lime_ctx_mlp;

/* Bytes of device workspace the calls below need for a batch of B users with
 * total_hist packed history rows and an item catalogue of any size.  The
 * workspace must be 256-byte aligned, zeroed once by lime_workspace_init, and
 * may be reused by any later call with the same or smaller sizes. */
size_t lime_workspace_bytes(const lime_dims* dims, int64_t B, int64_t total_hist);

/* Clears the workspace's status word (asynchronous on stream). */
int lime_workspace_init(void* workspace, size_t bytes, cudaStream_t stream);

/* QK cache: cache[m, h, :] = softmax_k( s * (T_m Wq_c)_h · (L_k Wk_c)_h ),
 * s = 1/sqrt(d_h).  LIME note 关键设计 1 (O = phi(T L^T) L^P; the weights
 * depend only on the item and the global links, so they are precomputed for
 * the catalogue) and 整体框架 (offline item side); LIME listing Table 12 (one
 * weight per item, head and link).
 *   T       device [n_items, d]     item embeddings
 *   L       device [l, d]           global links (raw, not contextualised)
 *   Wq_c    device [d, d]           candidate-side query projection
 *   Wk_c    device [d, d]           candidate-side key projection
 *   cache_out device [n_items, H, l] softmax weights (dims->dtype)
 *   workspace, workspace_bytes: device scratch of at least
 *           lime_workspace_bytes(dims, 0, 0) bytes (ERR_ARG when smaller).  */
int lime_build_qk_cache(const lime_dims* dims, const void* T, int64_t n_items,
                        const void* L, const void* Wq_c, const void* Wk_c,
                        void* cache_out, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* Two-stage form of lime_build_qk_cache, for callers that run the small first
 * stage on another stream (it depends only on the weights):
 * lime_fold_qk writes the folded per-head matrix G_h = s Wq_c[:, h-cols]
 * (L Wk_c[:, h-cols])^T (d x H*l, the same for every item; LIME note 关键设计
 * 1: the weights depend only on the item and the global links) to `image`
 * as the 128-byte-swizzled operand image the build reads;
 * lime_build_qk_cache_folded then computes cache[m, h, :] =
 * softmax_k((T_m G_h)_k) over the catalogue.  Together they equal
 * lime_build_qk_cache.
 *   image  device, lime_qk_image_bytes(dims) bytes (2*d*H*l), 16-byte
 *          aligned; written by lime_fold_qk, read by the build.
 *   tiles_per_cta  0: one persistent CTA per SM (fastest alone); k > 0:
 *          CTAs of about k 128-item tiles each, so that a build issued on a
 *          low-priority stream yields SMs to higher-priority work (every
 *          kernel is launched with its stream's priority).  Negative:
 *          LIME_ERR_ARG.
 * Other arguments, checks and errors as lime_build_qk_cache.  Supported:
 * the bf16 tensor-core shapes (lime_qk_image_bytes returns 0 otherwise and
 * both calls return LIME_ERR_SHAPE).  lime_fold_qk uses no workspace.      */
size_t lime_qk_image_bytes(const lime_dims* dims);
int lime_fold_qk(const lime_dims* dims, const void* L, const void* Wq_c, const void* Wk_c,
                 void* image, cudaStream_t stream);
int lime_build_qk_cache_folded(const lime_dims* dims, const void* T, int64_t n_items,
                               const void* image, void* cache_out, int32_t tiles_per_cta,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Uncached (online) candidate scoring: the same O_m as
 * lime_score_candidates, with the weights computed per candidate from the item
 * table instead of read from a QK cache,
 *   O[m, h-cols] = sum_k softmax_k(s (T[id_m] Wq_c)_h . (L Wk_c)_{k,h}) LP_u[k, h-cols]
 * (LIME note 关键设计 1, O = MHA(T, L, L^P); LIME listing Table 10
 * "uncached global"; the cold-start path for items not in the cache).
 *   T        device [n_items, d] item table, 16-byte aligned.
 *   image    device, the folded G image written by lime_fold_qk for the same
 *            dims, L, Wq_c, Wk_c (lime_qk_image_bytes(dims) bytes).
 * Other arguments, checks, flags and errors as lime_score_candidates (an
 * out-of-range ID sets LIME_FLAG_BAD_ID and its row of O is zero).
 * Supported: bf16, d = 128, H = 4, l in {16, 32, 64} (else LIME_ERR_SHAPE). */
int lime_score_candidates_uncached(const lime_dims* dims, int64_t B, const void* T,
                                   int64_t n_items, const void* image, const int32_t* cand_ids,
                                   const int64_t* cand_offsets, int64_t total_cand, const void* LP,
                                   void* O_out, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/* Allocation-free variant of lime_build_qk_cache.  The paper has no
 * counterpart: it exists for callers that cannot allocate device memory, such
 * as a plug-in whose host framework owns the whole device memory pool, or a
 * latency-critical serving loop that cannot accept cudaMalloc's implicit
 * device synchronisation.  The caller still owns T, L, Wq_c, Wk_c and
 * cache_out (same meaning, layout and checks as lime_build_qk_cache); the
 * scratch lives in a static device array of LIME_NOALLOC_SCRATCH_BYTES bytes
 * that every GPU loading the library holds until the process exits.
 *   - Each call made outside a stream capture (with the device current) looks
 *     up the array's device address; a call made during a capture reuses the
 *     address found by the last such call on that device, so make the first
 *     call on a device before any stream capture.
 *   - Arguments are checked exactly as lime_build_qk_cache checks them, with
 *     the same return codes, before the array is touched.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears the status word it uses.  Calls that overlap on the GPU (on
 *     different streams, say) race on the array.
 *   - The scratch a call needs is lime_workspace_bytes(dims, 0, 0); when that
 *     exceeds LIME_NOALLOC_SCRATCH_BYTES the call returns LIME_ERR_SCRATCH
 *     (use lime_build_qk_cache with a workspace instead).
 *   - Device-side status flags of these calls (LIME_FLAG_TIMEOUT when a
 *     bounded wait gave up and the cache may be partly written) are kept in
 *     the array's status word and read by lime_noalloc_get_status.
 * Calls no cudaMalloc, cudaFree or allocating library routine.            */
#define LIME_NOALLOC_SCRATCH_BYTES (1u << 20)
enum { LIME_ERR_SCRATCH = -5 /* scratch need above LIME_NOALLOC_SCRATCH_BYTES */ };
int lime_build_qk_cache_noalloc(const lime_dims* dims, const void* T, int64_t n_items,
                                const void* L, const void* Wq_c, const void* Wk_c,
                                void* cache_out, cudaStream_t stream);

/* The status word of lime_build_qk_cache_noalloc's static array on the
 * current device: synchronises `stream`, copies the sticky LIME_FLAG_* word
 * to *flags and clears it (as lime_get_status does for a workspace).
 * Allocation-free.  ERR_ARG for a null `flags` or while `stream` is being
 * captured.                                                               */
int lime_noalloc_get_status(cudaStream_t stream, int* flags);

/* Context links: LC[u, k, :] = SiLU([L_k ; ctx_u] Wc1 + bc1) Wc2 + bc2.
 * LIME note 整体框架 (L^C = MLP(L ⊕ E^C)) and 一个完整示例 step 2.
 *   L   device [l, d];  ctx device [B, c];  LC_out device [B, l, d].
 *   workspace, workspace_bytes: only its status word is used (a timed-out
 *           device wait sets LIME_FLAG_TIMEOUT there); at least
 *           lime_workspace_bytes(dims, 0, 0) bytes.
 * Needs dims->c >= 1.                                                    */
int lime_context_links(const lime_dims* dims, int64_t B, const void* L,
                       const void* ctx, const lime_ctx_mlp* w, void* LC_out,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* One LIME-XOR layer over a batch of jagged user histories.
 * LIME note 关键设计 2: over X = [E; Z] a query attends to a key only when
 * exactly one of the two is a link (XORA(X,X,X) = MHA(E, Z, Z) ⊕ MHA(Z, E, E)),
 * with pre-LN on the projections (损失函数 / 训练策略), a residual after the
 * output projection and a residual GatedMLP:
 *   X^ = LN1(X); Q,K,V = X^Wq, X^Wk, X^Wv; Y = X + XORA(Q,K,V) Wo;
 *   X' = Y + (SiLU(LN2(Y) W1) * (LN2(Y) W3)) W2.
 *   hist_offsets device [B+1] int64; total_hist = hist_offsets[B]
 *   E_in   device [total_hist, d]  history rows
 *   Z_in   device [B, l, d]        link rows (L^C for the first layer)
 *   E_out  device [total_hist, d]  or NULL: NULL marks the last layer, whose
 *          history outputs nobody reads; only Z_out is produced then.
 *   Z_out  device [B, l, d]        after the last layer this is L^P.
 *   workspace, workspace_bytes: at least lime_workspace_bytes(dims, B,
 *          total_hist) bytes (ERR_ARG when smaller).
 * No output may overlap an input or the other output (ERR_ALIAS).
 * E_in, E_out, Z_in, Z_out and every weight pointer must be 16-byte aligned
 * and hist_offsets 8-byte aligned (ERR_ARG otherwise): the tensor-core path
 * moves them by TMA and 16-byte vector accesses.
 * A user with no history gets a zero link-branch attention output.
 * Streams: on the bf16 tensor-core path a non-final layer runs its link-row
 * tail on a library-owned side stream (the device's highest priority),
 * forked from `stream` with an event and joined back before the call
 * returns, so all of the layer's work stays ordered on `stream` (and inside a
 * graph captured from it).  The side stream is created by the first call on
 * the device that is not being captured; until then the layer runs in order
 * on `stream` alone.                                                      */
int lime_xor_layer(const lime_dims* dims, int64_t B,
                   const int64_t* hist_offsets, int64_t total_hist,
                   const void* E_in, const void* Z_in, const lime_layer_w* w,
                   void* E_out, void* Z_out, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);

/* Cached candidate scoring: O[m, h-cols] = sum_k cache[id_m, h, k] * LP[u, k, h-cols]
 * for every candidate m of user u.  LIME note 关键设计 1 and 一个完整示例
 * step 3 (O_c = sum_k w_k L^P_k).
 *   cache        device [n_items, H, l]   from lime_build_qk_cache
 *   cand_ids     device [total_cand] int32  row indices into cache
 *   cand_offsets device [B+1] int64; total_cand = cand_offsets[B]
 *   LP           device [B, l, d]
 *   O_out        device [total_cand, d]
 *   workspace, workspace_bytes: at least lime_workspace_bytes(dims, 0, 0).
 * Duplicate IDs are allowed; an ID outside [0, n_items) gives a zero row and
 * sets LIME_FLAG_BAD_ID.                                                  */
int lime_score_candidates(const lime_dims* dims, int64_t B, const void* cache,
                          int64_t n_items, const int32_t* cand_ids,
                          const int64_t* cand_offsets, int64_t total_cand,
                          const void* LP, void* O_out, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/* int8 QK cache (LIME listing Tables 9, 11, 12: one byte per cached weight,
 * "int8 lookup + dequant"; the encoding is not stated by the pages).  Byte
 * q[m, h, k] = round(255 * w[m, h, k]) with w the lime_build_qk_cache
 * weight computed in fp32 (ties to even; w lies in [0, 1]); dequantised as
 * q / 255.  Same arguments, checks and errors as lime_build_qk_cache, with
 *   cache_out device uint8 [n_items, H, l] (16-byte aligned).
 * Supported: bf16, d = 128, H = 4 with l in {16, 32, 64}, or H*l = 256     *
 * (else LIME_ERR_SHAPE).                                                  */
int lime_build_qk_cache_u8(const lime_dims* dims, const void* T, int64_t n_items,
                           const void* L, const void* Wq_c, const void* Wk_c,
                           uint8_t* cache_out, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* Cached scoring from an int8 cache: O[m, h-cols] = sum_k (q[id_m, h, k] / 255)
 * L^P_u[k, h-cols].  Same arguments, checks and errors as
 * lime_score_candidates, with cache a device uint8 [n_items, H, l] array
 * (16-byte aligned).  The product runs in fp16 (the bytes are exact; L^P is
 * converted exactly for 6.1e-5 <= |x| <= 65504, smaller magnitudes keep an
 * absolute error below 3e-8; larger ones overflow).  Supported: bf16,
 * d = 128, H = 4, l in {32, 64} (else LIME_ERR_SHAPE).                     */
int lime_score_candidates_u8(const lime_dims* dims, int64_t B, const uint8_t* cache,
                             int64_t n_items, const int32_t* cand_ids,
                             const int64_t* cand_offsets, int64_t total_cand,
                             const void* LP, void* O_out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* Test hook for the failure detection: runs one kernel whose bounded
 * device-side wait nothing completes.  After the wait's time limit (about
 * two seconds) it sets LIME_FLAG_TIMEOUT in the workspace's status word and
 * returns; the context stays usable.  workspace: initialised, 256-byte
 * aligned (ERR_ARG otherwise).                                            */
int lime_debug_wait_timeout(void* workspace, cudaStream_t stream);

/* Synchronises stream, copies the sticky LIME_FLAG_* word to *flags and
 * clears it. */
int lime_get_status(void* workspace, cudaStream_t stream, int* flags);

/* Number of CUDA kernels the library has launched in this process (a host
 * counter, for profiling and benchmarking; it never touches the device). */
uint64_t lime_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LIME_H */
