// Generic CUDA-core kernels of the LIME hot path.
//
// These run every step for any supported shape and for both storage types
// (fp32 and bf16, accumulation always fp32).  They are the fp32 path, and the
// bf16 path for shapes the tensor-core kernels do not cover.  Each follows the
// definition it implements step by step; the tensor-core kernels in the other
// files are the fast bf16 path.
#include "lime_simt.cuh"

namespace lime {

// ------------------------------------------------------------ context links
// LC[u,k,:] = SiLU([L_k ; ctx_u] Wc1 + bc1) Wc2 + bc2
// (LIME note, 整体框架: L^C = MLP(L ⊕ E^C)).  Block (u, g) computes links
// [g*kCtxLinks, (g+1)*kCtxLinks) of user u; each thread owns one output column
// for kCtxLinks link rows at a time, so every weight read is reused kCtxLinks
// times.  With `stage` the weights are first copied to shared memory (when
// they fit); otherwise they are read from global memory.
constexpr int kCtxLinks = 8;

template <class T>
__global__ void __launch_bounds__(128) k_context_links(int d, int c, int l,
                                                       const T* __restrict__ L,
                                                       const T* __restrict__ ctx,
                                                       const T* __restrict__ Wc1,
                                                       const T* __restrict__ bc1,
                                                       const T* __restrict__ Wc2,
                                                       const T* __restrict__ bc2,
                                                       T* __restrict__ LC, bool stage) {
  extern __shared__ float sm[];
  const int din = d + c;
  float* x = sm;                                     // [kCtxLinks][din]
  float* hid = x + kCtxLinks * din;                  // [kCtxLinks][d]
  // staged weights start on a 16-byte boundary
  T* ws1 = reinterpret_cast<T*>(
      (reinterpret_cast<uintptr_t>(hid + kCtxLinks * d) + 15) & ~uintptr_t(15));  // [din][d]
  T* ws2 = ws1 + (size_t)din * d;                    // [d][d] when staged
  const T* w1 = stage ? ws1 : Wc1;
  const T* w2 = stage ? ws2 : Wc2;
  const int64_t u = blockIdx.x;
  const int k0 = blockIdx.y * kCtxLinks;
  const int nk = l - k0 < kCtxLinks ? l - k0 : kCtxLinks;
  if (stage) {
    // 16-byte copies, several in flight per thread (d * sizeof(T) % 16 == 0)
    const int n1 = din * d * (int)sizeof(T) / 16, n2 = d * d * (int)sizeof(T) / 16;
    const uint4* g1 = reinterpret_cast<const uint4*>(Wc1);
    const uint4* g2 = reinterpret_cast<const uint4*>(Wc2);
    uint4* s1 = reinterpret_cast<uint4*>(ws1);
    uint4* s2 = reinterpret_cast<uint4*>(ws2);
#pragma unroll 8
    for (int e = threadIdx.x; e < n1; e += blockDim.x) s1[e] = g1[e];
#pragma unroll 8
    for (int e = threadIdx.x; e < n2; e += blockDim.x) s2[e] = g2[e];
  }
  for (int e = threadIdx.x; e < kCtxLinks * din; e += blockDim.x) {
    const int kk = e / din, i = e % din;
    float v = 0.f;
    if (kk < nk) v = i < d ? to_f(L[(int64_t)(k0 + kk) * d + i]) : to_f(ctx[u * c + (i - d)]);
    x[e] = v;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc[kCtxLinks];
    const float b = to_f(bc1[j]);
#pragma unroll
    for (int kk = 0; kk < kCtxLinks; ++kk) acc[kk] = b;
    for (int i = 0; i < din; ++i) {
      const float wv = to_f(w1[(size_t)i * d + j]);
#pragma unroll
      for (int kk = 0; kk < kCtxLinks; ++kk) acc[kk] += x[kk * din + i] * wv;
    }
#pragma unroll
    for (int kk = 0; kk < kCtxLinks; ++kk) hid[kk * d + j] = silu_f(acc[kk]);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc[kCtxLinks];
    const float b = to_f(bc2[j]);
#pragma unroll
    for (int kk = 0; kk < kCtxLinks; ++kk) acc[kk] = b;
    for (int i = 0; i < d; ++i) {
      const float wv = to_f(w2[(size_t)i * d + j]);
#pragma unroll
      for (int kk = 0; kk < kCtxLinks; ++kk) acc[kk] += hid[kk * d + i] * wv;
    }
    for (int kk = 0; kk < nk; ++kk) LC[(u * l + k0 + kk) * d + j] = from_f<T>(acc[kk]);
  }
}

// ------------------------------------------------------------------ GEMM
// C[R, N] = A[R, K] (fp32, row stride lda) x W[K, N] (T, row-major)
//           (+ resid[R, N] fp32 when resid != nullptr).  64x64 tiles.
template <class TW>
__global__ void __launch_bounds__(256) k_gemm(const float* __restrict__ A, int64_t lda,
                                              const TW* __restrict__ W, int K, int N,
                                              int64_t R, const float* __restrict__ resid,
                                              float* __restrict__ C) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64];
  const int64_t r0 = (int64_t)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      int r = e >> 4, k = e & 15;
      int64_t gr = r0 + r;
      int gk = k0 + k;
      As[k][r] = (gr < R && gk < K) ? A[gr * lda + gk] : 0.f;
    }
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      int k = e >> 6, n = e & 63;
      int gk = k0 + k, gn = n0 + n;
      Ws[k][n] = (gk < K && gn < N) ? to_f(W[(int64_t)gk * N + gn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int64_t r = r0 + ty * 4 + i;
    if (r >= R) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (resid) v += resid[r * N + n];
      C[r * N + n] = v;
    }
  }
}

// ------------------------------------------------------------- row helpers
// X[r] = E_in[r] for r < nh, X[nh + i] = Z_in[i]  (fp32 copy of [E; Z])
template <class T>
__global__ void k_pack_rows(const T* __restrict__ E, const T* __restrict__ Z, int64_t nh,
                            int64_t nz, int d, float* __restrict__ X) {
  int64_t n = (nh + nz) * d;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = e / d;
    X[e] = r < nh ? to_f(E[e]) : to_f(Z[e - nh * d]);
  }
}

// Row-wise LayerNorm, biased variance, eps 1e-5; one warp per row.
template <class T>
__global__ void k_layernorm(const float* __restrict__ X, int64_t R, int d,
                            const T* __restrict__ g, const T* __restrict__ b,
                            float* __restrict__ Y) {
  int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (r >= R) return;
  const float* x = X + r * d;
  float s = 0.f;
  for (int i = lane; i < d; i += 32) s += x[i];
  float mu = warp_sum(s) / d;
  float v = 0.f;
  for (int i = lane; i < d; i += 32) { float t = x[i] - mu; v += t * t; }
  float rstd = rsqrtf(warp_sum(v) / d + 1e-5f);
  for (int i = lane; i < d; i += 32) Y[r * d + i] = (x[i] - mu) * rstd * to_f(g[i]) + to_f(b[i]);
}

// G[r, j] = SiLU(G[r, j]) * G3[r, j]
__global__ void k_swiglu(float* __restrict__ G, const float* __restrict__ G3, int64_t n) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    G[e] = silu_f(G[e]) * G3[e];
}

// E_out[r] = X[r] (r < nh; skipped when E_out is null), Z_out[i] = X[nh + i]
template <class T>
__global__ void k_unpack_rows(const float* __restrict__ X, int64_t nh, int64_t nz, int d,
                              T* __restrict__ E, T* __restrict__ Z) {
  int64_t n = (nh + nz) * d;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = e / d;
    if (r < nh) {
      if (E) E[e] = from_f<T>(X[e]);
    } else {
      Z[e - nh * d] = from_f<T>(X[e]);
    }
  }
}

// ---------------------------------------------------------- XOR attention
// History branch, MHA(E, L^C, L^C): history row i of user u attends to the l
// link rows of u, per head (LIME note, 关键设计 2), and with LIME-XOR+Window
// (关键设计 3) also to the user's history rows j with 0 < |i - j| <= window,
// in one phi over the union of keys.  One warp per (row, head).  Q, K, V are
// fp32 [nh + B*l, d]; link row k of user u is row nh + u*l + k.
__global__ void k_attn_hist(const float* __restrict__ Q, const float* __restrict__ K,
                            const float* __restrict__ V, const int64_t* __restrict__ off,
                            int64_t B, int64_t nh, int d, int H, int l, float scale,
                            int phi, int window, float* __restrict__ A, unsigned* status) {
  extern __shared__ float sp[];  // [warps][l + 2 window]
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t task = blockIdx.x * (int64_t)(blockDim.x >> 5) + warp;
  if (task >= nh * H) return;
  int64_t i = task / H;
  int h = task % H;
  int dh = d / H;
  int64_t u = owner_of(off, B, i);
  // the window: history rows [wa, wb) of the same user, row i itself skipped
  int64_t ua = 0, ub = 0;
  if (window > 0) user_range(off, u, B, nh, &ua, &ub, status);
  const int64_t wa = i - window > ua ? i - window : ua;
  const int64_t wb = i + window + 1 < ub ? i + window + 1 : ub;
  const int nw = window > 0 ? (int)(wb - wa) : 0;   // window keys including i
  const int nk = l + nw;                             // key slots; slot l + (i - wa) is i
  const float* q = Q + i * d + h * dh;
  float* p = sp + warp * (l + 2 * window + 1);
  auto key_row = [&](int k) -> int64_t { return k < l ? nh + u * l + k : wa + (k - l); };
  float mx = -INFINITY;
  for (int k = lane; k < nk; k += 32) {
    const int64_t r = key_row(k);
    float s = -INFINITY;
    if (r != i || k < l) {
      const float* kk = K + r * d + h * dh;
      s = 0.f;
      for (int c = 0; c < dh; ++c) s += q[c] * kk[c];
      s *= scale;
    }
    p[k] = s;
    mx = fmaxf(mx, s);
  }
  mx = warp_max(mx);
  const int n_keys = l + (nw > 0 ? nw - 1 : 0);
  float sum = 0.f;
  if (phi == LIME_PHI_SILU) {
    // SiLU of each score over the visible keys
    for (int k = lane; k < nk; k += 32) p[k] = p[k] == -INFINITY ? 0.f : p[k] / (1.0f + expf(-p[k]));
    sum = (float)n_keys;
  } else {
    for (int k = lane; k < nk; k += 32) { float e = expf(p[k] - mx); p[k] = e; sum += e; }
    sum = warp_sum(sum);
  }
  __syncwarp();
  for (int c = lane; c < dh; c += 32) {
    float acc = 0.f;
    for (int k = 0; k < nk; ++k) acc += p[k] * V[key_row(k) * d + h * dh + c];
    A[i * d + h * dh + c] = acc / sum;
  }
}

// Link branch, MHA(L^C, E, E): link k of user u attends to the user's history
// rows, per head.  One warp per (user, head, link); each lane keeps an online
// softmax over a strided subset of the history, merged through shared memory.
// A user with no history gets a zero output.  With phi = SiLU a lane keeps the
// SiLU-weighted sum and its key count (max 0), and the same merge divides the
// total by N_u.
template <int DH>
__global__ void k_attn_link(const float* __restrict__ Q, const float* __restrict__ K,
                            const float* __restrict__ V, const int64_t* __restrict__ off,
                            int64_t B, int64_t nh, int d, int H, int l, float scale,
                            int phi, float* __restrict__ A, unsigned* status) {
  __shared__ float sm_m[4][32], sm_s[4][32];
  __shared__ float sm_acc[4][32][DH + 1];
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t task = blockIdx.x * 4 + warp;
  bool active = task < B * H * l;
  int64_t u = 0;
  int h = 0, k = 0;
  if (active) {
    u = task / (H * l);
    h = (task / l) % H;
    k = task % l;
  }
  float q[DH], acc[DH];
  const bool silu = phi == LIME_PHI_SILU;
  float m = silu ? 0.f : -INFINITY, s = 0.f;
#pragma unroll
  for (int c = 0; c < DH; ++c) acc[c] = 0.f;
  int64_t a = 0, b = 0;
  if (active) {
    user_range(off, u, B, nh, &a, &b, status);
    const float* qp = Q + (nh + u * l + k) * d + h * DH;
#pragma unroll
    for (int c = 0; c < DH; ++c) q[c] = qp[c];
    for (int64_t j = a + lane; j < b; j += 32) {
      const float* kp = K + j * d + h * DH;
      float sc = 0.f;
#pragma unroll
      for (int c = 0; c < DH; ++c) sc += q[c] * kp[c];
      sc *= scale;
      const float* vp = V + j * d + h * DH;
      if (silu) {
        const float e = sc / (1.0f + expf(-sc));
        s += 1.0f;
#pragma unroll
        for (int c = 0; c < DH; ++c) acc[c] += e * vp[c];
        continue;
      }
      float mn = fmaxf(m, sc);
      float corr = expf(m - mn), e = expf(sc - mn);
      s = s * corr + e;
#pragma unroll
      for (int c = 0; c < DH; ++c) acc[c] = acc[c] * corr + e * vp[c];
      m = mn;
    }
  }
  sm_m[warp][lane] = m;
  sm_s[warp][lane] = s;
#pragma unroll
  for (int c = 0; c < DH; ++c) sm_acc[warp][lane][c] = acc[c];
  __syncwarp();
  if (!active) return;
  float M = -INFINITY;
  for (int t = 0; t < 32; ++t) M = fmaxf(M, sm_m[warp][t]);
  float S = 0.f;
  for (int t = 0; t < 32; ++t)
    if (sm_s[warp][t] > 0.f) S += sm_s[warp][t] * expf(sm_m[warp][t] - M);
  for (int c = lane; c < DH; c += 32) {
    float o = 0.f;
    for (int t = 0; t < 32; ++t)
      if (sm_s[warp][t] > 0.f) o += sm_acc[warp][t][c] * expf(sm_m[warp][t] - M);
    A[(nh + u * l + k) * d + h * DH + c] = (b > a) ? o / S : 0.f;
  }
}

// ------------------------------------------------------------- cache build
// Kc[k, c] = sum_j L[k, j] Wk_c[j, c]  (fp32 out), one block per link row.
template <class T>
__global__ void k_link_keys(const T* __restrict__ L, const T* __restrict__ Wk, int d,
                            float* __restrict__ Kc) {
  int k = blockIdx.x;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < d; ++j) acc += to_f(L[(int64_t)k * d + j]) * to_f(Wk[(int64_t)j * d + c]);
    Kc[(int64_t)k * d + c] = acc;
  }
}

// Gfold[i, h*l + k] = scale * sum_{c in head h} Wq_c[i, c] Kc[k, c]   (fp32)
// so that the cache logits are T_m · Gfold[:, h*l + k].
template <class T>
__global__ void k_fold_g(const T* __restrict__ Wq, const float* __restrict__ Kc, int d,
                         int H, int l, float scale, float* __restrict__ G) {
  int i = blockIdx.x;
  int dh = d / H;
  for (int j = threadIdx.x; j < H * l; j += blockDim.x) {
    int h = j / l, k = j % l;
    float acc = 0.f;
    for (int c = h * dh; c < (h + 1) * dh; ++c) acc += to_f(Wq[(int64_t)i * d + c]) * Kc[(int64_t)k * d + c];
    G[(int64_t)i * H * l + j] = acc * scale;
  }
}

// cache[m, h, :] = phi_k(T_m · Gfold[:, h*l + k]) (softmax, or SiLU / l).
// One block of H*l threads (rounded up to a warp multiple) per group of 8 items.
template <class T>
__global__ void k_cache_simt(const T* __restrict__ Tm, int64_t n_items, int d, int H, int l,
                             const float* __restrict__ G, int phi, T* __restrict__ cache) {
  extern __shared__ float sm[];
  float* trow = sm;             // [8][d]
  float* logit = sm + 8 * d;    // [8][H*l]
  const int HL = H * l;
  const int64_t m0 = (int64_t)blockIdx.x * 8;
  for (int e = threadIdx.x; e < 8 * d; e += blockDim.x) {
    int64_t m = m0 + e / d;
    trow[e] = m < n_items ? to_f(Tm[m * d + e % d]) : 0.f;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < HL; j += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    for (int i = 0; i < d; ++i) {
      float g = G[(int64_t)i * HL + j];
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t] += trow[t * d + i] * g;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) logit[t * HL + j] = acc[t];
  }
  __syncthreads();
  // one thread per (item, head): softmax over the l links
  for (int e = threadIdx.x; e < 8 * H; e += blockDim.x) {
    int t = e / H, h = e % H;
    int64_t m = m0 + t;
    if (m >= n_items) continue;
    float* z = logit + t * HL + h * l;
    if (phi == LIME_PHI_SILU) {
      for (int k = 0; k < l; ++k)
        cache[(m * H + h) * l + k] = from_f<T>(z[k] / (1.0f + expf(-z[k])) / (float)l);
      continue;
    }
    float mx = -INFINITY;
    for (int k = 0; k < l; ++k) mx = fmaxf(mx, z[k]);
    float s = 0.f;
    for (int k = 0; k < l; ++k) s += expf(z[k] - mx);
    float inv = 1.f / s;
    for (int k = 0; k < l; ++k) cache[(m * H + h) * l + k] = from_f<T>(expf(z[k] - mx) * inv);
  }
}

// ---------------------------------------------------------------- scoring
// O[m, h*dh + c] = sum_k cache[id_m, h, k] * LP[u, k, h*dh + c]
// (LIME note, 一个完整示例 step 3).  One warp per candidate.
template <class T>
__global__ void k_score_simt(const T* __restrict__ cache, int64_t n_items,
                             const int32_t* __restrict__ ids, const int64_t* __restrict__ off,
                             int64_t B, int64_t total, const T* __restrict__ LP, int d, int H,
                             int l, T* __restrict__ O, unsigned* status) {
  extern __shared__ float sw[];  // [warps][H*l]
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t m = blockIdx.x * (int64_t)(blockDim.x >> 5) + warp;
  if (m >= total) return;
  const int HL = H * l, dh = d / H;
  int64_t u = owner_of(off, B, m);
  if (lane == 0) {
    int64_t a, b;
    user_range(off, u, B, total, &a, &b, status);
  }
  int64_t id = ids[m];
  float* w = sw + warp * HL;
  bool ok = id >= 0 && id < n_items;
  if (!ok && lane == 0) raise_flag(status, LIME_FLAG_BAD_ID);
  for (int j = lane; j < HL; j += 32) w[j] = ok ? to_f(cache[id * HL + j]) : 0.f;
  __syncwarp();
  for (int j = lane; j < d; j += 32) {
    int h = j / dh;
    float acc = 0.f;
    for (int k = 0; k < l; ++k) acc += w[h * l + k] * to_f(LP[(u * l + k) * d + j]);
    O[m * d + j] = from_f<T>(acc);
  }
}

// ------------------------------------------------------------ launchers

static inline int grid_for(int64_t n, int per_block, int cap = 148 * 32) {
  int64_t g = (n + per_block - 1) / per_block;
  if (g < 1) g = 1;
  return (int)(g > cap ? cap : g);
}

template <class T>
void simt_context_links(const lime_dims& D, int64_t B, const void* L, const void* ctx,
                        const lime_ctx_mlp& w, void* LC, cudaStream_t st) {
  const int din = D.d + D.c;
  const size_t small = (size_t)kCtxLinks * (din + D.d) * sizeof(float);
  const size_t staged = small + 16 + ((size_t)din * D.d + (size_t)D.d * D.d) * sizeof(T);
  const bool stage = staged <= 200 * 1024;
  const size_t smem = stage ? staged : small;
  cudaFuncSetAttribute(k_context_links<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((unsigned)B, (unsigned)((D.l + kCtxLinks - 1) / kCtxLinks));
  k_context_links<T><<<grid, 128, smem, st>>>(
      D.d, D.c, D.l, (const T*)L, (const T*)ctx, (const T*)w.Wc1, (const T*)w.bc1,
      (const T*)w.Wc2, (const T*)w.bc2, (T*)LC, stage);
  note_launches(1);
}

static void gemm(const float* A, int64_t lda, const void* W, bool bf, int K, int N, int64_t R,
                 const float* resid, float* C, cudaStream_t st) {
  if (R == 0) return;
  dim3 grid((N + 63) / 64, (unsigned)((R + 63) / 64));
  if (bf)
    k_gemm<bf16><<<grid, 256, 0, st>>>(A, lda, (const bf16*)W, K, N, R, resid, C);
  else
    k_gemm<float><<<grid, 256, 0, st>>>(A, lda, (const float*)W, K, N, R, resid, C);
  note_launches(1);
}

size_t simt_layer_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist) {
  int64_t R = total_hist + B * D.l;
  return (size_t)R * (7 * (size_t)D.d + 2 * (size_t)D.f) * sizeof(float);
}

template <class T>
void simt_xor_layer(const lime_dims& D, int64_t B, const int64_t* off, int64_t nh,
                    const void* E_in, const void* Z_in, const lime_layer_w& w, void* E_out,
                    void* Z_out, float* ws, unsigned* status, cudaStream_t st) {
  const int d = D.d, f = D.f, H = D.H, l = D.l, dh = d / H;
  const bool bf = sizeof(T) == 2;
  const int64_t nz = B * l, R = nh + nz;
  float* X = ws;
  float* Xh = X + R * d;
  float* Q = Xh + R * d;
  float* K = Q + R * d;
  float* V = K + R * d;
  float* A = V + R * d;
  float* Y = A + R * d;
  float* G1 = Y + R * d;
  float* G3 = G1 + R * f;
  const float scale = 1.0f / sqrtf((float)dh);
  int g = grid_for(R * d, 256);
  k_pack_rows<T><<<g, 256, 0, st>>>((const T*)E_in, (const T*)Z_in, nh, nz, d, X);
  note_launches(1);
  k_layernorm<T><<<(unsigned)((R * 32 + 255) / 256), 256, 0, st>>>(X, R, d, (const T*)w.g1,
                                                                  (const T*)w.b1, Xh);
  note_launches(1);
  gemm(Xh, d, w.Wq, bf, d, d, R, nullptr, Q, st);
  gemm(Xh, d, w.Wk, bf, d, d, R, nullptr, K, st);
  gemm(Xh, d, w.Wv, bf, d, d, R, nullptr, V, st);
  if (nh > 0) {
    int64_t tasks = nh * H;
    k_attn_hist<<<(unsigned)((tasks + 7) / 8), 256, 8 * (l + 2 * D.window + 1) * sizeof(float),
                  st>>>(Q, K, V, off, B, nh, d, H, l, scale, D.phi, D.window, A, status);
    note_launches(1);
  }
  {
    int64_t tasks = B * H * l;
    unsigned grid = (unsigned)((tasks + 3) / 4);
    if (dh == 16)
      k_attn_link<16><<<grid, 128, 0, st>>>(Q, K, V, off, B, nh, d, H, l, scale, D.phi, A, status);
    else if (dh == 32)
      k_attn_link<32><<<grid, 128, 0, st>>>(Q, K, V, off, B, nh, d, H, l, scale, D.phi, A, status);
    else
      k_attn_link<64><<<grid, 128, 0, st>>>(Q, K, V, off, B, nh, d, H, l, scale, D.phi, A, status);
    note_launches(1);
  }
  gemm(A, d, w.Wo, bf, d, d, R, X, Y, st);          // Y = X + A Wo
  k_layernorm<T><<<(unsigned)((R * 32 + 255) / 256), 256, 0, st>>>(Y, R, d, (const T*)w.g2,
                                                                  (const T*)w.b2, Xh);
  note_launches(1);
  gemm(Xh, d, w.W1, bf, d, f, R, nullptr, G1, st);
  gemm(Xh, d, w.W3, bf, d, f, R, nullptr, G3, st);
  k_swiglu<<<grid_for(R * f, 256), 256, 0, st>>>(G1, G3, R * f);
  note_launches(1);
  gemm(G1, f, w.W2, bf, f, d, R, Y, X, st);         // X' = Y + hidden W2
  k_unpack_rows<T><<<g, 256, 0, st>>>(X, nh, nz, d, (T*)E_out, (T*)Z_out);
  note_launches(1);
}

size_t simt_cache_ws_bytes(const lime_dims& D) {
  return ((size_t)D.l * D.d + (size_t)D.d * D.H * D.l) * sizeof(float);
}

template <class T>
void simt_build_qk_cache(const lime_dims& D, const void* Tm, int64_t n, const void* L,
                         const void* Wq, const void* Wk, void* cache, float* ws,
                         cudaStream_t st) {
  const int d = D.d, H = D.H, l = D.l, HL = H * l;
  float* Kc = ws;
  float* G = ws + (size_t)l * d;
  const float scale = 1.0f / sqrtf((float)(d / H));
  k_link_keys<T><<<l, 128, 0, st>>>((const T*)L, (const T*)Wk, d, Kc);
  note_launches(1);
  k_fold_g<T><<<d, 128, 0, st>>>((const T*)Wq, Kc, d, H, l, scale, G);
  note_launches(1);
  if (n == 0) return;
  int threads = ((HL + 31) / 32) * 32;
  if (threads > 1024) threads = 1024;
  size_t smem = (size_t)8 * (d + HL) * sizeof(float);
  k_cache_simt<T><<<(unsigned)((n + 7) / 8), threads, smem, st>>>((const T*)Tm, n, d, H, l, G,
                                                                 D.phi, (T*)cache);
  note_launches(1);
}

template <class T>
void simt_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
                const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
                unsigned* status, cudaStream_t st) {
  if (total == 0) return;
  size_t smem = (size_t)8 * D.H * D.l * sizeof(float);
  k_score_simt<T><<<(unsigned)((total + 7) / 8), 256, smem, st>>>(
      (const T*)cache, n_items, ids, off, B, total, (const T*)LP, D.d, D.H, D.l, (T*)O, status);
  note_launches(1);
}

template void simt_context_links<float>(const lime_dims&, int64_t, const void*, const void*,
                                        const lime_ctx_mlp&, void*, cudaStream_t);
template void simt_context_links<bf16>(const lime_dims&, int64_t, const void*, const void*,
                                       const lime_ctx_mlp&, void*, cudaStream_t);
template void simt_xor_layer<float>(const lime_dims&, int64_t, const int64_t*, int64_t,
                                    const void*, const void*, const lime_layer_w&, void*, void*,
                                    float*, unsigned*, cudaStream_t);
template void simt_xor_layer<bf16>(const lime_dims&, int64_t, const int64_t*, int64_t,
                                   const void*, const void*, const lime_layer_w&, void*, void*,
                                   float*, unsigned*, cudaStream_t);
template void simt_build_qk_cache<float>(const lime_dims&, const void*, int64_t, const void*,
                                         const void*, const void*, void*, float*, cudaStream_t);
template void simt_build_qk_cache<bf16>(const lime_dims&, const void*, int64_t, const void*,
                                        const void*, const void*, void*, float*, cudaStream_t);
template void simt_score<float>(const lime_dims&, int64_t, const void*, int64_t, const int32_t*,
                                const int64_t*, int64_t, const void*, void*, unsigned*,
                                cudaStream_t);
template void simt_score<bf16>(const lime_dims&, int64_t, const void*, int64_t, const int32_t*,
                               const int64_t*, int64_t, const void*, void*, unsigned*,
                               cudaStream_t);

}  // namespace lime
