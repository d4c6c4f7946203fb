// One LIME-XOR layer on the 5th-generation tensor cores (bf16 storage,
// d = 128, 4 heads of 32, l in {16, 32, 64}, GatedMLP width 256).
//
// LIME note, 关键设计 2: over X = [E; Z] the XOR mask keeps only history<->link
// attention, XORA(X,X,X) = MHA(E, Z, Z) ⊕ MHA(Z, E, E), at O(l·N) cost; the
// layer is pre-LN with residual connections and a gated feed-forward block.
//
// Work is split by row kind.  Link rows (B·l of them) carry L^P, so their
// projections run with split-bf16 activations (x = hi + lo, both bf16; the
// bf16 weights are exact), i.e. at close to fp32 accuracy for twice the MMA
// work on a few rows.  History rows (the O(N) part) use bf16 operands with
// fp32 accumulation, statistics and residual adds.  History rows are cut into
// per-user tiles of 128 rows (a tile never spans two users; its tail rows are
// masked).  The query/key products are folded per user through the link
// rows (Q_E K_Z^T = X^ (Wq K_Z^T), Q_Z K_E^T = (Q_Z Wk^T) X^^T, P V_Z Wo =
// P (V_Z Wo) per head), so Q_E and K_E are never formed.
//
//   k_prep_weights   layer weights -> K-major 128B-swizzled images (W^T); its
//                    block 0 turns hist_offsets into the tile list (user,
//                    first row, valid rows)
//   k_link_proj      LN1(Z) -> Q_Z, K_Z, V_Z (split precision) -> per-user
//                    folded images G = s Wq K_Z^T (transposed), Q' = s Q_Z
//                    Wk^T (hi + lo) and VO = V_Z Wo, per head; one CTA per
//                    (128 link rows, image)
//   k_hist_xattn     LN1(E) -> history scores X^ G, softmax over l, Yd = P VO
//                    (fp16 attention delta); link scores Q' X^^T (transposed:
//                    (head, link) on the TMEM lanes), V_E = X^ Wv, per tile
//                    and (head, link) the partial softmax statistics (max,
//                    sum) and the weighted V_E sum
//   k_hist_ffn       Y = E + Yd, LN2, GatedMLP in 64-wide chunks, E' = Y + ·
//                    (warp-specialized pipeline)
//   k_link_tail      per 128 link rows, a cluster of four CTAs: log-sum-exp
//                    merge of the tile partials -> b, Y_Z = Z + b·Wo, LN2,
//                    GatedMLP (one hidden chunk per CTA, split precision),
//                    Z' = Y_Z + sum of the chunks
// The last layer (E_out = NULL) skips everything only E' needs: G, VO, the
// history branch of k_hist_xattn and k_hist_ffn.
//
// Kernels use 512 threads (thread (row, part): a TMEM lane and a quarter of
// the row's columns) or warp-specialized roles; one thread issues the MMAs.
// Every kernel is launched with programmatic dependent launch (pdl_launch /
// pdl_wait).  Every wait is bounded and sets LIME_FLAG_TIMEOUT.
#include <mutex>
#include <type_traits>

#include "lime_fast.cuh"
#include "sm100.cuh"

namespace lime {

using namespace sm100;

namespace {

constexpr int kD = 128, kH = 4, kDH = 32, kF = 256, kTile = 128;
constexpr uint32_t kBlk = 128 * 128;  // bytes of one [128 rows x 64 cols] bf16 block
constexpr float kLnEps = 1e-5f;
constexpr int kRec = 36;  // floats per link-branch record: max, sum, 2 pad, 32 weighted sums

struct LayerWs {
  size_t img_q, img_k, img_v, img_o, img_13, img_2;
  size_t img_vg;   // (g1 Wv)^T as hi, lo images, then cv = colsum(g1 Wv), dv = b1 Wv (fp32)
  size_t sched, tiles, tile_start;
  size_t yd, uimg, part;
  size_t qe, ke, ve, att, kz, vz;   // window layers: history Q, K, V and A; link K, V (fp32)
  size_t total;
  int64_t max_tiles;
  uint32_t uimg_bytes;   // per user: nhalf half images
  uint32_t half_bytes;   // one half image (128 (head, link) rows)
};

__host__ __device__ constexpr size_t up1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

// per-user folded images, in halves of 128 (head, link) rows (one half for
// l <= 32, two for l = 64: half i holds heads 2i and 2i+1): G'^T, Q'g, VO
// ([128 x 128] bf16 each), then the fp32 vectors cQ, dQ, cG, dG ([128] each);
// with phi = SiLU also the low half of G' (G' = hi + lo)
constexpr uint32_t kUimgVec = 6 * kBlk;
constexpr uint32_t kUimgBytes = 6 * kBlk + 4 * 128 * 4;
constexpr uint32_t kUimgGlo = kUimgBytes;

LayerWs layer_ws(int l, int64_t B, int64_t nh, bool silu, int window) {
  LayerWs w;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = up1k(o + bytes); return r; };
  w.img_q = take(2 * kBlk);
  w.img_k = take(2 * kBlk);
  w.img_v = take(2 * kBlk);
  w.img_o = take(2 * kBlk);
  w.img_13 = take(8 * kBlk);
  w.img_2 = take(4 * kBlk);
  w.img_vg = take(4 * kBlk + 2 * kD * 4);
  w.max_tiles = nh / kTile + B + 1;
  w.sched = take(16);
  w.tiles = take((size_t)w.max_tiles * 16);
  w.tile_start = take((size_t)(B + 1) * 4);
  w.yd = take((size_t)nh * kD * 2);   // attention delta (fp16)
  w.half_bytes = kUimgBytes + (silu ? 2 * kBlk : 0);
  w.uimg_bytes = (uint32_t)((kH * l + 127) / 128) * w.half_bytes;
  w.uimg = take((size_t)B * w.uimg_bytes);
  w.part = take((size_t)w.max_tiles * kH * l * kRec * 4);
  w.qe = w.ke = w.ve = w.att = w.kz = w.vz = 0;
  if (window > 0) {
    w.qe = take((size_t)nh * kD * 4);
    w.ke = take((size_t)nh * kD * 4);
    w.ve = take((size_t)nh * kD * 4);
    w.att = take((size_t)nh * kD * 4);
    w.kz = take((size_t)B * l * kD * 4);
    w.vz = take((size_t)B * l * kD * 4);
  }
  w.total = o;
  return w;
}

// LayerNorm scratch of the 512-thread kernels: two [4][128] reduction
// buffers and the affine parameters as fp32 (g, then b).
constexpr int kLnFloats = 2 * 512 + 2 * kD;
constexpr int kLnBytes = kLnFloats * 4;

// Stages g and b (bf16 [128]) as fp32 at gb (call before the first LN; the
// LN's own barriers order these writes before the reads).
__device__ __forceinline__ void ln_stage(float* gb, const bf16* g, const bf16* b) {
  if (threadIdx.x < kD) {
    gb[threadIdx.x] = __bfloat162float(g[threadIdx.x]);
    gb[kD + threadIdx.x] = __bfloat162float(b[threadIdx.x]);
  }
}

// Statistics of one 32-value part of a row: its mean and the sum of squared
// deviations from that mean (two passes over the registers, so no
// cancellation between E[x^2] and mu^2 however large the row's mean is).
__device__ __forceinline__ void part_stats(const float* x, float& mean, float& m2) {
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) s += x[k];
  mean = s * (1.0f / 32);
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float dlt = x[k] - mean;
    q = fmaf(dlt, dlt, q);
  }
  m2 = q;
}

// Row mean and rstd from the four parts' (mean, m2): the parallel-variance
// merge for equal counts, M2 = sum m2_p + 32 sum (mean_p - mu)^2 (biased
// variance M2 / 128, eps as in LayerNorm).
__device__ __forceinline__ void merge4_stats(float m0, float m1, float m2_, float m3, float q0,
                                             float q1, float q2, float q3, float& mu,
                                             float& rstd) {
  mu = (m0 + m1 + m2_ + m3) * 0.25f;
  const float d0 = m0 - mu, d1 = m1 - mu, d2 = m2_ - mu, d3 = m3 - mu;
  const float M2 = (q0 + q1) + (q2 + q3) + 32.0f * (d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3);
  rstd = rsqrtf(M2 * (1.0f / kD) + kLnEps);
}

// LayerNorm of one row held as four 32-column parts (x = this thread's part,
// columns c0..c0+31), affine with the staged g, b.  Each part's mean and
// centred sum of squares are exchanged through `red` and merged (see
// merge4_stats).  `red` is a kLnFloats scratch (red[0..1023] for the
// reductions, g and b after them); all 512 threads take part (one block-wide
// barrier; the caller's next barrier must come before red is written again).
__device__ __forceinline__ void layer_norm_part(float* x, int c0, float* red, int part, int row) {
  float pm, pq;
  part_stats(x, pm, pq);
  red[part * 128 + row] = pm;
  red[512 + part * 128 + row] = pq;
  __syncthreads();
  float mu, rstd;
  merge4_stats(red[row], red[128 + row], red[256 + row], red[384 + row], red[512 + row],
               red[640 + row], red[768 + row], red[896 + row], mu, rstd);
  const float4* g4 = reinterpret_cast<const float4*>(red + 1024 + c0);
  const float4* b4 = reinterpret_cast<const float4*>(red + 1024 + kD + c0);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 gv = g4[q], bv = b4[q];
    x[4 * q] = (x[4 * q] - mu) * rstd * gv.x + bv.x;
    x[4 * q + 1] = (x[4 * q + 1] - mu) * rstd * gv.y + bv.y;
    x[4 * q + 2] = (x[4 * q + 2] - mu) * rstd * gv.z + bv.z;
    x[4 * q + 3] = (x[4 * q + 3] - mu) * rstd * gv.w + bv.w;
  }
}

// Writes 32 values (columns c0 .. c0+31 of row `row`) as hi = bf16(x) and
// lo = bf16(x - hi) into two [128 x 128] swizzled operands.
__device__ __forceinline__ void split_part_st(uint8_t* hi, uint8_t* lo, int row, int c0,
                                              const float* x) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float h8[8], l8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      h8[k] = __bfloat162float(__float2bfloat16_rn(x[q * 8 + k]));
      l8[k] = x[q * 8 + k] - h8[k];
    }
    sw_st16(hi, kBlk, row, c0 + q * 8, pack8(h8));
    sw_st16(lo, kBlk, row, c0 + q * 8, pack8(l8));
  }
}

// SiLU with the hardware exp2 and reciprocal approximations (a few ulp in
// fp32; the result is rounded to bf16 for the next product).  An IEEE
// division here would cost about as much as the rest of the gate's epilogue.
// For very negative x, 1 + exp(-x) overflows to inf and the result is -0.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// SiLU through the identity sigmoid(x) = (1 + tanh(x/2)) / 2 with the
// hardware tanh approximation (relative error about 2^-11): one special-
// function operation instead of two, for the history rows' GatedMLP, whose
// hidden value is rounded to bf16 (2^-9) right after.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  return fmaf(h, tanh_approx(h), h);
}

// 2^x with the hardware approximation (ex2.approx: relative error about
// 2^-22; -inf -> +0).  The softmax kernels keep their scores in log2 units
// (scaled by log2 e in the folded constants), so e^(z - m) is one ex2.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// fp32 [rows x 128] staging: row r is 512 bytes, its 16-byte chunk c sits at
// r*512 + ((c ^ (r & 31)) * 16), so row-per-thread and row-per-warp accesses
// are both free of bank conflicts.
__device__ __forceinline__ float4* f32_chunk(uint8_t* base, int r, int c) {
  return reinterpret_cast<float4*>(base + r * 512 + ((c ^ (r & 31)) << 4));
}

// Common CTA prologue: barriers, abort flag, TMEM allocation (`ncols` columns).
struct Cta {
  uint64_t* bar;      // [0] loads, [1] mma, [2..3] extra loads
  uint32_t* slot;
  int* abort_flag;
  uint32_t tmem;
  uint32_t ncols;
};

__device__ __forceinline__ void cta_setup(uint8_t* bar_area, int nbar, Cta& c,
                                          uint32_t ncols = 512) {
  c.ncols = ncols;
  c.bar = reinterpret_cast<uint64_t*>(bar_area);
  c.slot = reinterpret_cast<uint32_t*>(bar_area + 8 * nbar);
  c.abort_flag = reinterpret_cast<int*>(bar_area + 8 * nbar + 8);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nbar; ++i) mbar_init(&c.bar[i], 1);
    *c.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) tmem_alloc(c.slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = *c.slot;
  pdl_launch();
  pdl_wait();
}

__device__ __forceinline__ void cta_teardown(Cta& c) {
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(c.tmem, c.ncols);
  }
}

// 512-thread kernels: warp w serves TMEM lane quadrant w % 4.
__device__ __forceinline__ uint32_t quad_addr(const Cta& c) {
  return c.tmem + ((uint32_t)(((threadIdx.x >> 5) & 3) * 32) << 16);
}

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------ weight images
// Image of W^T (K-major B operand) for x·W, W row-major [k_in, n_out]:
//   Wq, Wk, Wv, Wo, W2: element (n, k) at (k/64)*rows*128 + sw128_offset(n, k%64)
//   W1, W3 (n in [0,256)): chunk n/64 of 16 KB, inside it (k/64)*8192 +
//   sw128_offset(n%64, k%64), so one 64-wide GatedMLP chunk is contiguous.
__device__ void schedule_tiles(const int64_t* __restrict__ off, int64_t B, int64_t nh,
                               int max_tiles, int* __restrict__ sched, int4* __restrict__ tiles,
                               int* __restrict__ tile_start, unsigned* status);

// Block 0 builds the tile schedule, block 1 the V_E vectors (cv, dv); the
// other blocks write the weight images.
__global__ void __launch_bounds__(1024) k_prep_weights(
    const bf16* __restrict__ Wq, const bf16* __restrict__ Wk, const bf16* __restrict__ Wv,
    const bf16* __restrict__ Wo, const bf16* __restrict__ W1, const bf16* __restrict__ W3,
    const bf16* __restrict__ W2, const bf16* __restrict__ g1, const bf16* __restrict__ b1,
    uint8_t* __restrict__ ws, LayerWs L, const int64_t* __restrict__ off, int64_t B, int64_t nh,
    unsigned* status) {
  pdl_launch();
  pdl_wait();
  if (blockIdx.x == 0) {
    schedule_tiles(off, B, nh, (int)L.max_tiles, reinterpret_cast<int*>(ws + L.sched),
                   reinterpret_cast<int4*>(ws + L.tiles), reinterpret_cast<int*>(ws + L.tile_start),
                   status);
    return;
  }
  if (blockIdx.x == 1) {
    // cv[n] = sum_i g1[i] Wv[i][n] (each product is exact in fp32, and equal to
    // the hi + lo image pair), dv[n] = sum_i b1[i] Wv[i][n]: thread (n, g)
    // sums rows 16g .. 16g+15, then thread n adds the eight partials
    __shared__ float part_cd[2][8][kD];
    const int n = threadIdx.x & (kD - 1), g = threadIdx.x >> 7;
    float cv = 0.f, dv = 0.f;
#pragma unroll
    for (int i = g * 16; i < g * 16 + 16; ++i) {
      const float w = __bfloat162float(Wv[i * kD + n]);
      cv = fmaf(__bfloat162float(g1[i]), w, cv);
      dv = fmaf(__bfloat162float(b1[i]), w, dv);
    }
    part_cd[0][g][n] = cv;
    part_cd[1][g][n] = dv;
    __syncthreads();
    if (threadIdx.x < kD) {
      float* vec = reinterpret_cast<float*>(ws + L.img_vg + 4 * kBlk);
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) { a += part_cd[0][j][n]; b += part_cd[1][j][n]; }
      vec[n] = a;
      vec[kD + n] = b;
    }
    return;
  }
  // Thread (matrix, n, k8) gathers W[k8*8 .. k8*8+7][n] (loads coalesced over
  // n) and writes them as one 16-byte chunk of row n of the image.
  const int64_t e = (blockIdx.x - 2) * (int64_t)blockDim.x + threadIdx.x;
  const int64_t n_sq = kD * kD / 8, n_ff = kD * kF / 8;   // chunks per matrix
  float f[8];
  if (e < 4 * n_sq) {
    const int w = (int)(e / n_sq), r = (int)(e % n_sq);
    const int k8 = r / kD, n = r % kD;
    const bf16* src = w == 0 ? Wq : w == 1 ? Wk : w == 2 ? Wv : Wo;
    const size_t base = w == 0 ? L.img_q : w == 1 ? L.img_k : w == 2 ? L.img_v : L.img_o;
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = __bfloat162float(src[(k8 * 8 + j) * kD + n]);
    sw_st16(ws + base, kBlk, n, k8 * 8, pack8(f));
  } else if (e < 4 * n_sq + 2 * n_ff) {
    const int64_t r0 = e - 4 * n_sq;
    const int w = (int)(r0 / n_ff), r = (int)(r0 % n_ff);
    const int k8 = r / kF, n = r % kF;
    // chunk n/64 of the hidden layer: K block k/64 holds W1's 64 rows, then W3's
    const bf16* src = w == 0 ? W1 : W3;
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = __bfloat162float(src[(k8 * 8 + j) * kF + n]);
    *reinterpret_cast<uint4*>(ws + L.img_13 + (n >> 6) * (2 * kBlk) + ((k8 * 8) >> 6) * kBlk +
                              w * 8192 + sw128_offset(n & 63, (k8 * 8) & 63)) = pack8(f);
  } else if (e < 4 * n_sq + 3 * n_ff) {
    const int r = (int)(e - 4 * n_sq - 2 * n_ff);
    const int k8 = r / kD, n = r % kD;   // W2 is [256, 128]
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = __bfloat162float(W2[(k8 * 8 + j) * kD + n]);
    sw_st16(ws + L.img_2, kBlk, n, k8 * 8, pack8(f));
  } else if (e < 5 * n_sq + 3 * n_ff) {
    // (g1 Wv)^T split hi + lo: LN1's scale folded into the V_E weights
    const int r = (int)(e - 4 * n_sq - 3 * n_ff);
    const int k8 = r / kD, n = r % kD;
    float lo[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = __bfloat162float(g1[k8 * 8 + j]) * __bfloat162float(Wv[(k8 * 8 + j) * kD + n]);
      f[j] = __bfloat162float(__float2bfloat16_rn(x));
      lo[j] = x - f[j];
    }
    sw_st16(ws + L.img_vg, kBlk, n, k8 * 8, pack8(f));
    sw_st16(ws + L.img_vg + 2 * kBlk, kBlk, n, k8 * 8, pack8(lo));
  }
}

// --------------------------------------------------------------- schedule
// Tiles of 128 history rows per user, in user order.  Writes n_tiles to
// sched[0], tiles[t] = (u, first row, valid rows, 0) and tile_start[u] (the
// first tile of user u; tile_start[B] = n_tiles).  Offsets are clamped into
// [0, nh]; violations set LIME_FLAG_BAD_OFFSETS.
__device__ void schedule_tiles(const int64_t* __restrict__ off, int64_t B, int64_t nh,
                               int max_tiles, int* __restrict__ sched, int4* __restrict__ tiles,
                               int* __restrict__ tile_start, unsigned* status) {
  __shared__ int warp_sums[32];
  __shared__ int s_base;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t u0 = 0; u0 < B; u0 += blockDim.x) {
    const int64_t u = u0 + threadIdx.x;
    int64_t a = 0, b = 0;
    int cnt = 0;
    if (u < B) {
      user_range(off, u, B, nh, &a, &b, status);
      cnt = (int)((b - a + kTile - 1) / kTile);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int v = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      warp_sums[lane] = v;
    }
    __syncthreads();
    const int start = s_base + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - cnt;
    if (u < B) {
      tile_start[u] = start;
      for (int i = 0; i < cnt && start + i < max_tiles; ++i) {
        const int64_t r0 = a + (int64_t)i * kTile;
        const int64_t nv = b - r0 < kTile ? b - r0 : kTile;
        tiles[start + i] = make_int4((int)u, (int)r0, (int)nv, 0);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base += warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = s_base < max_tiles ? s_base : max_tiles;
    sched[0] = n;
    tile_start[B] = n;
  }
}

// ----------------------------------------------------- link projections
// Per-user operand images, at uimg + u * uimg_bytes: three [128 rows x 128]
// bf16 K-major 128B-swizzled images of two kBlk blocks each, then fp32
// vectors.  Row p = h*L + k is (head h, link k); rows p >= H*L are never
// written and only ever reach MMA output rows that nothing reads.
//   G'   [0, 2 kBlk)   G'[p, i] = g1[i] (s K_Z[k, h] Wq[:, h]^T)[i]   (h: head h's 32 columns)
//   Q'g  [2, 4 kBlk)   Q'g[p, i] = g1[i] (s Q_Z[k, h] Wk[:, h]^T)[i]
//   VO   [4, 6 kBlk)   VO[p] = V_Z[k, h] Wo[h, :]                     (Wo's rows of head h)
//   vec  cQ, dQ, cG, dG [128] each: c[p] = sum_i of the stored row p of Q'g
//        (G'), d[p] = sum_i b1[i] of the unscaled row (times log2 e for phi =
//        softmax: the history kernel's scores are in log2 units)
// By associativity the history scores are Q_E,h (s K_Z,h)^T = X^ G_h, the
// link scores (s Q_Z,h) K_E,h^T = Q'_h X^^T and the history branch through
// Wo is (P_h V_Z,h) Wo_h = P_h VO_h.  With X^ = LN1(E) = rstd (E - mu) g1 + b1
// per history row, Q' X^^T = rstd (Q'g E^T - mu cQ) + dQ (and likewise X^ G),
// so the history kernel multiplies the raw rows E and needs only each row's
// mean and rstd; it never forms Q_E, K_E or X^.
//
// CTA (128 link rows, which, z): which = 0 -> Q'g, 1 -> G', 2 -> VO, for heads
// z*hpc .. z*hpc + hpc - 1 (hpc = H / gridDim.z; more CTAs spread the image
// writes, which dominate, over more SMs).  LN1(Z) (split) -> projection P =
// X^z Wm -> s P (which < 2) split hi + lo -> per head h of the CTA the fold
// P[:, h] B_h (K = 32, two MMAs), B_h = Wk's, Wq's or Wo's head-h slice of its
// weight image -> rows h*L + k of the users' images, staged and written with
// bulk copies.  512 threads: thread (row, part) owns columns part*32 ..
// part*32+31.
template <int L>
__global__ void __launch_bounds__(512, 1)
    k_link_proj(const bf16* __restrict__ Z, int64_t nrows, const bf16* __restrict__ g1,
                const bf16* __restrict__ b1, uint8_t* __restrict__ ws, LayerWs Lw, float scale,
                bool silu, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1k(smem_raw);
  uint8_t* sAh = sm;
  uint8_t* sAl = sm + 2 * kBlk;
  uint8_t* sW = sm + 4 * kBlk;    // projection weight image (W^T, K-major)
  uint8_t* sF = sm + 6 * kBlk;    // fold weight image
  float* red = reinterpret_cast<float*>(sm + 8 * kBlk);
  const int which = blockIdx.y;
  const int hpc = kH / (int)gridDim.z, h0 = (int)blockIdx.z * hpc;   // this CTA's heads
  Cta c;
  cta_setup(sm + 8 * kBlk + kLnBytes, 2, c, 512);
  ln_stage(red + 1024, g1, b1);
  uint32_t mph = 0;
  if (threadIdx.x == 0) {
    const size_t img = which == 0 ? Lw.img_q : which == 1 ? Lw.img_k : Lw.img_v;
    const size_t fold = which == 0 ? Lw.img_k : which == 1 ? Lw.img_q : Lw.img_o;
    mbar_arrive_expect_tx(&c.bar[0], 4 * kBlk);
    bulk_load(sW, ws + img, 2 * kBlk, &c.bar[0]);
    bulk_load(sF, ws + fold, 2 * kBlk, &c.bar[0]);
  }
  const int warp = threadIdx.x >> 5;
  const int part = warp >> 2;
  const int r = (warp & 3) * 32 + (threadIdx.x & 31);
  const int c0 = part * 32;
  const int64_t R = (int64_t)blockIdx.x * kTile + r;
  const bool valid = R < nrows;
  {
    float x[32];
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(Z + R * kD + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) unpack8(src[q], x + q * 8);
    } else {
#pragma unroll
      for (int i2 = 0; i2 < 32; ++i2) x[i2] = 0.f;
    }
    layer_norm_part(x, c0, red, part, r);
    split_part_st(sAh, sAl, r, c0, x);
  }
  fence_proxy_async_smem();
  __syncthreads();
  mbar_wait(&c.bar[0], 0, status, c.abort_flag);
  if (threadIdx.x == 0) {
    tc_fence_after();
    mma_tile(c.tmem, smem_u32(sAh), kBlk, smem_u32(sW), kBlk, 128, 128, false);
    mma_tile(c.tmem, smem_u32(sAl), kBlk, smem_u32(sW), kBlk, 128, 128, true);
  }
  cta_mma_wait(&c.bar[1], mph, status, c.abort_flag);
  const uint32_t ta = quad_addr(c);
  {
    // the projection (scaled for the score operands) becomes the fold's A
    // operand, split hi + lo over the MMA operands it came from
    float v[32];
    tmem_ld16(ta + c0, v);
    tmem_ld16(ta + c0 + 16, v + 16);
    tmem_ld_wait();
    if (which != 2) {
#pragma unroll
      for (int i2 = 0; i2 < 32; ++i2) v[i2] *= scale;
    }
    split_part_st(sAh, sAl, r, c0, v);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_fence_after();
    for (int h = h0; h < h0 + hpc; ++h) {
      const uint32_t d = c.tmem + (h - h0) * 128;
      const uint32_t ah = smem_u32(sAh) + (h >> 1) * kBlk + (h & 1) * 64;
      const uint32_t al = smem_u32(sAl) + (h >> 1) * kBlk + (h & 1) * 64;
      if (which == 2) {
        // B[n][k'] = Wo[32h + k'][n]: Wo^T's image with a K offset of 32h
        const uint32_t b = smem_u32(sF) + (h >> 1) * kBlk + (h & 1) * 64;
        mma_tile(d, ah, kBlk, b, kBlk, 128, kDH, false);
        mma_tile(d, al, kBlk, b, kBlk, 128, kDH, true);
      } else {
        // B[n][k'] = W[n][32h + k']: rows 32h .. of W^T's image read MN-major
        const uint32_t b = smem_u32(sF) + h * kDH * 128;
        mma_tile_bmn(d, ah, kBlk, b, kBlk, 128, kDH, false);
        mma_tile_bmn(d, al, kBlk, b, kBlk, 128, kDH, true);
      }
    }
  }
  cta_mma_wait(&c.bar[1], mph, status, c.abort_flag);
  // The fold outputs are staged (the MMA operands are dead) in the images'
  // own swizzled layout: lane r = j*L + k of user j lands at row r, which has
  // the swizzle phase of its image row h*L + k, so user j's L rows of a head
  // leave as one L*128-byte bulk copy per 64-column block (up to four heads
  // per CTA, one 32 KB buffer each).  Q' and G carry LN1's affine map of the
  // history rows: they are stored scaled by g1 along d (Q'g, G'), with
  // c[p] = sum_i Q'g[p, i] (of the stored bf16 values) and d[p] = sum_i
  // Q'[p, i] b1[i] (likewise for G) in the user's vector area, so that
  // Q' X^^T = rstd (Q'g E^T - mu c) + d for the raw history rows E.
  constexpr int UP = kTile / L;   // users per tile
  const int64_t u0 = (int64_t)blockIdx.x * UP;
  const int64_t left = nrows / L - u0;
  const int n_users = left < UP ? (int)left : UP;
  const float* gb = red + 1024;   // g1, b1 as fp32
  // phi = SiLU: G' is stored as hi + lo (two buffers per head): SiLU weights are
  // signed, so the history scores' operand rounding is not averaged away
  const bool split = which == 1 && silu;
  for (int i = 0; i < hpc; ++i) {
    const int h = h0 + i;
    float v[32];
    tmem_ld16(ta + i * 128 + c0, v);
    tmem_ld16(ta + i * 128 + c0 + 16, v + 16);
    tmem_ld_wait();
    uint8_t* buf = sm + (split ? 2 * i : i) * 2 * kBlk;
    if (which == 2) {
#pragma unroll
      for (int q = 0; q < 4; ++q) sw_st16(buf, kBlk, r, c0 + q * 8, pack8(v + q * 8));
    } else {
      float cs = 0.f, ds = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        ds = fmaf(v[j], gb[kD + c0 + j], ds);
        v[j] *= gb[c0 + j];
        if (!split) v[j] = __bfloat162float(__float2bfloat16_rn(v[j]));
        cs += v[j];
      }
      if (split)
        split_part_st(buf, buf + 2 * kBlk, r, c0, v);
      else {
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(buf, kBlk, r, c0 + q * 8, pack8(v + q * 8));
      }
      red[part * 128 + r] = cs;
      red[512 + part * 128 + r] = ds;
      __syncthreads();
      if (part == 0 && valid) {
        const int p = h * L + (int)(R % L);   // row p & 127 of half p >> 7
        float* vec = reinterpret_cast<float*>(ws + Lw.uimg + (size_t)(R / L) * Lw.uimg_bytes +
                                              (size_t)(p >> 7) * Lw.half_bytes + kUimgVec) +
                     (which == 0 ? 0 : 2 * 128);
        // softmax: d in log2 units (the history kernel scales rstd alike)
        vec[p & 127] = red[r] + red[128 + r] + red[256 + r] + red[384 + r];
        vec[128 + (p & 127)] = (red[512 + r] + red[640 + r] + red[768 + r] + red[896 + r]) *
                               (silu ? 1.0f : kLog2e);
      }
      __syncthreads();
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t img_off = which == 0 ? 2 * kBlk : which == 1 ? 0 : 4 * kBlk;
    for (int i = 0; i < hpc * (split ? 2 : 1); ++i) {
      const int h = h0 + (split ? i >> 1 : i);
      const uint32_t off = split && (i & 1) ? kUimgGlo : img_off;
      const int p0 = h * L;   // the head's first image row: row p0 & 127 of half p0 >> 7
      for (int j = 0; j < n_users; ++j) {
        uint8_t* dst = ws + Lw.uimg + (size_t)(u0 + j) * Lw.uimg_bytes +
                       (size_t)(p0 >> 7) * Lw.half_bytes + off + (p0 & 127) * 128;
        const uint8_t* src = sm + i * 2 * kBlk + j * L * 128;
        bulk_store(dst, src, L * 128);
        bulk_store(dst + kBlk, src + kBlk, L * 128);
      }
    }
    bulk_commit();
  }
  if (threadIdx.x == 0) bulk_wait<0>();   // the images are complete before the CTA exits
  cta_teardown(c);
}

// --------------------------------------------------------- XOR attention
// One persistent CTA per SM walks the tile list.  Per 128-row history tile
// (a tile never spans two users; rows past `nv` are masked), with mu, rstd the
// LN1 statistics of each raw history row E (the affine part of LN1 is folded
// into the images: see the link projections):
//   MMAs     S'^T = Q'g E^T (link scores, (head, link) on the TMEM lanes;
//            [128, 256) or [384, 512) by tile parity), V_E = E (g1 Wv) (hi +
//            lo, [256, 384)), S = E G' (history scores, [0, H*L)), each group
//            committed to its own barrier.  They need only the raw E tile, so
//            they start as soon as it lands, while the epilogue finishes the
//            previous tile.
//   stats    mu, rstd per row (reduced over the four column parts)
//   softmax  (phi = SiLU: pointwise SiLU weights, see the lime_phi notes)
//            P2 = exp(z - max), z = rstd (S'^T - mu cQ) + dQ per token column,
//            over the tile's valid rows (part = a quarter of the tokens; the
//            lane's max and sum reduced over the parts); V_E = rstd (. - mu
//            cv) + dv as bf16 over the G' image; P = softmax of each head's L
//            scores rstd (S - mu cG) + dG (part = head) over the E tile
//   MMAs     P2 V_E (into the link-score columns; lane (h, k) keeps head h's
//            32 columns) and Yd = P VO ([0, 128), already through Wo)
//   out      the link record (max, sum, 32 weighted V sums) of each lane;
//            Yd as fp16 by TMA tensor stores (plain stores for a partial
//            tile); fp16 keeps 11 bits of the delta, which the residual adds
//            to E (bf16 would cost E' up to 2^-9 |Yd|)
// HIST = false (the last layer: E' is not needed) keeps the link branch only.
//
// Shared memory: six 32 KB slots.  (g1 Wv)^T hi and lo (resident), G' -> V_E,
// Q'g -> VO, and two that alternate (A, B): A = E tile -> P -> Yd staging,
// B = P2 -> the next E tile.  Every load is issued as soon as its slot's last
// reader has completed: VO (and, in the last layer, the next Q'g) once the
// link scores are done, the next E tile and G' once P2 V_E is done, the next
// Q'g once Yd is done.
// Warps 0-15 (epilogue): thread (row, part), row = 32*(warp%4) + lane (a TMEM
// lane), part = warp/4; they synchronise among themselves with a named
// barrier.  Warp 16 (one lane) issues the MMAs and the loads: tcgen05.mma
// issue stalls while the tensor pipe is busy, which would otherwise hold an
// epilogue warp, and with it every barrier of the epilogue, until the last
// MMA group has started.
constexpr int kXaEpi = 512;
constexpr int kXaThreads = kXaEpi + 32;
constexpr uint32_t kXaSmem = 1024 + 12 * kBlk + 2048 /* mu, rstd x2 */ + 8192 /* red x2 */ +
                             1024 /* cv, dv */ + 2 * 2048 /* vec x2 */ +
                             kBlk /* one block of G'lo (phi = SiLU) */ + 256 /* barriers */;

template <int L, bool HIST, bool SILU>
__global__ void __launch_bounds__(kXaThreads, 1)
    k_hist_xattn(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                 uint8_t* __restrict__ ws, LayerWs Lw, unsigned* status) {
  constexpr int HL = kH * L;
  constexpr int NH = (HL + 127) / 128;        // halves of the (head, link) pairs
  constexpr int HLH = HL < 128 ? HL : 128;    // pairs per half
  constexpr bool SPLIT = NH > 1;
  // TMEM columns: one half -> [0,128) S, then Yd; S' at [128,256) / [384,512)
  // by tile parity; V_E [256,384).  Two halves -> [0,128) S, [128,256) S',
  // [256,384) V_E, [384,512) Yd, accumulated over the tile's two halves.
  constexpr uint32_t kYd = SPLIT ? 384 : 0;
  constexpr uint32_t kSlot = 2 * kBlk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1k(smem_raw);
  uint8_t* sWh = sm;                // (g1 Wv)^T hi
  uint8_t* sWl = sm + kSlot;        // (g1 Wv)^T lo
  uint8_t* sG = sm + 2 * kSlot;     // G' -> V_E
  uint8_t* sQ = sm + 3 * kSlot;     // Q'g -> VO
  uint8_t* rot = sm + 4 * kSlot;    // two alternating slots
  // [128] mu, then [128] rstd, by tile parity
  float* smu2 = reinterpret_cast<float*>(sm + 6 * kSlot);
  float* redS = smu2 + 512;                                 // [1024] LN1 statistics
  float* redX = redS + 1024;                                // [1024] softmax max / sum
  float* cvd = redX + 1024;                                 // cv [128], dv [128]
  float* vecs = cvd + 256;                                  // 2 x (cQ, dQ, cG, dG)
  uint8_t* sGl = reinterpret_cast<uint8_t*>(vecs + 1024);   // a 64-column block of G'lo
  Cta c;
  // bar: 0 weights, 1 S' done, 2 E tile, 3 G', 4 Q'g + vec, 5 records read
  //      out (two halves), 6 VO, 7 V_E done, 8 S done, 9 P2 V_E done, 10 Yd
  //      done, 11 Yd read out, 12 P2 and V_E written, 13 P written, 14 G'lo
  //      block landed, 15 its product done
  cta_setup(sGl + kBlk, 16, c);
  uint64_t* bar = c.bar;
  // the epilogue's hand-offs to the issuer: one arrival per epilogue warp
  if (threadIdx.x == 0) {
    for (int i : {5, 11, 12, 13}) mbar_init(&bar[i], kXaEpi / 32);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_tiles = *reinterpret_cast<const int*>(ws + Lw.sched);
  const int4* tiles = reinterpret_cast<const int4*>(ws + Lw.tiles);
  const int warp = threadIdx.x >> 5;
  if (warp == kXaEpi / 32) {
    if ((threadIdx.x & 31) == 0) {
      // ---- the issuer: loads and MMAs
      auto uimg = [&](int u, int hf) {   // half hf of user u's images
        return ws + Lw.uimg + (size_t)u * Lw.uimg_bytes + (size_t)hf * Lw.half_bytes;
      };
      auto load = [&](uint64_t* b, uint8_t* dst, const uint8_t* src) {
        mbar_arrive_expect_tx(b, kSlot);
        bulk_load(dst, src, kSlot, b);
      };
      auto load_q = [&](int u, int hf, int it) {   // Q'g and the half's vectors
        mbar_arrive_expect_tx(&bar[4], kSlot + 2048);
        bulk_load(sQ, uimg(u, hf) + 2 * kBlk, kSlot, &bar[4]);
        bulk_load(vecs + (it & 1) * 512, uimg(u, hf) + kUimgVec, 2048, &bar[4]);
      };
      auto load_e = [&](uint8_t* dst, int r0) {
        mbar_arrive_expect_tx(&bar[2], kSlot);
        tma_load_2d(dst, &tmE, 0, r0, &bar[2]);
        tma_load_2d(dst + kBlk, &tmE, 64, r0, &bar[2]);
      };
      prefetch_tmap(&tmE);
      mbar_arrive_expect_tx(&bar[0], 2 * kSlot + 1024);
      bulk_load(sWh, ws + Lw.img_vg, 2 * kSlot, &bar[0]);
      bulk_load(cvd, ws + Lw.img_vg + 4 * kBlk, 1024, &bar[0]);
      if ((int)blockIdx.x < n_tiles) {
        const int4 tl = tiles[blockIdx.x];
        load_e(rot, tl.y);
        if (HIST) load(&bar[3], sG, uimg(tl.x, 0));
        load_q(tl.x, 0, 0);
      } else {
        mbar_wait(&bar[0], 0, status, c.abort_flag);   // lands before the CTA exits
      }
      // virtual tiles (tile t, half hf), the halves of a tile back to back;
      // kt counts this CTA's tiles
      int ab = 0, t = blockIdx.x, hf = 0, kt = 0;
      for (int it = 0; t < n_tiles; ++it) {
        const int u = tiles[t].x;
        const int tn = hf + 1 < NH ? t : t + (int)gridDim.x;   // the next virtual tile
        const int hn = hf + 1 < NH ? hf + 1 : 0;
        const int un = tn < n_tiles ? tiles[tn].x : 0;
        const uint32_t ph = (uint32_t)it & 1u;
        uint8_t* sA = rot + ab * kSlot;
        uint8_t* sB = rot + (ab ^ 1) * kSlot;
        const uint32_t tS2 = c.tmem + 128 + (SPLIT ? 0u : (uint32_t)(it & 1) * 256);
        mbar_wait(&bar[2], ph, status, c.abort_flag);
        if (it == 0) mbar_wait(&bar[0], 0, status, c.abort_flag);
        mbar_wait(&bar[4], ph, status, c.abort_flag);
        // one S' buffer: the previous records must have been read out
        if (SPLIT && it > 0) mbar_wait(&bar[5], ph ^ 1u, status, c.abort_flag);
        tc_fence_after();
        mma_tile(tS2, smem_u32(sQ), kBlk, smem_u32(sA), kBlk, 128, 128, false);
        mma_commit(&bar[1]);
        mma_tile(c.tmem + 256, smem_u32(sA), kBlk, smem_u32(sWh), kBlk, 128, 128, false);
        mma_tile(c.tmem + 256, smem_u32(sA), kBlk, smem_u32(sWl), kBlk, 128, 128, true);
        mma_commit(&bar[7]);
        if (HIST) {
          // S overwrites the previous tile's Yd columns: wait for their readout
          if (!SPLIT && it > 0) mbar_wait(&bar[11], ph ^ 1u, status, c.abort_flag);
          mbar_wait(&bar[3], ph, status, c.abort_flag);
          tc_fence_after();
          mma_tile(c.tmem, smem_u32(sA), kBlk, smem_u32(sG), kBlk, HLH, 128, false);
          if constexpr (SILU) {
            // + E G'lo, one 64-column block at a time through sGl
            for (int j = 0; j < 2; ++j) {
              const uint32_t pj = (uint32_t)(2 * it + j) & 1u;
              if (j > 0) mbar_wait(&bar[15], pj ^ 1u, status, c.abort_flag);
              mbar_arrive_expect_tx(&bar[14], kBlk);
              bulk_load(sGl, uimg(u, hf) + kUimgGlo + j * kBlk, kBlk, &bar[14]);
              mbar_wait(&bar[14], pj, status, c.abort_flag);
              tc_fence_after();
              mma_tile(c.tmem, smem_u32(sA + j * kBlk), kBlk, smem_u32(sGl), kBlk, HLH, 64, true);
              mma_commit(&bar[15]);
            }
            mbar_wait(&bar[15], 1u, status, c.abort_flag);   // the block's buffer is free
          }
          mma_commit(&bar[8]);
        }
        // the link scores have read Q'g
        mbar_wait(&bar[1], ph, status, c.abort_flag);
        if (HIST) load(&bar[6], sQ, uimg(u, hf) + 4 * kBlk);
        else if (tn < n_tiles) load_q(un, hn, it + 1);
        mbar_wait(&bar[12], ph, status, c.abort_flag);
        tc_fence_after();
        mma_tile_bmn(tS2, smem_u32(sB), kBlk, smem_u32(sG), kBlk, 128, 128, false);
        mma_commit(&bar[9]);
        // P2 V_E has read P2 and V_E: the next E tile, and the next G'
        mbar_wait(&bar[9], ph, status, c.abort_flag);
        if (tn < n_tiles) {
          load_e(sB, tiles[tn].y);
          if (HIST) load(&bar[3], sG, uimg(un, hn));
          // the E tile after that into L2: its load is issued only once this
          // slot frees again, and would otherwise come from DRAM
          const int tp = tn + (int)gridDim.x;
          if (hf + 1 == NH && tp < n_tiles) {
            tma_prefetch_2d(&tmE, 0, tiles[tp].y);
            tma_prefetch_2d(&tmE, 64, tiles[tp].y);
          }
        }
        if (HIST) {
          mbar_wait(&bar[13], ph, status, c.abort_flag);
          mbar_wait(&bar[6], ph, status, c.abort_flag);
          // two halves: the first half's product starts the tile's Yd, so the
          // previous tile's Yd must have been read out
          if (SPLIT && hf == 0 && kt > 0)
            mbar_wait(&bar[11], (uint32_t)(kt - 1) & 1u, status, c.abort_flag);
          tc_fence_after();
          mma_tile_bmn(c.tmem + kYd, smem_u32(sA), kBlk, smem_u32(sQ), kBlk, 128, HLH, hf > 0);
          mma_commit(&bar[10]);
          // Yd has read P and VO: the next Q'g
          mbar_wait(&bar[10], ph, status, c.abort_flag);
          if (tn < n_tiles) load_q(un, hn, it + 1);
        }
        ab ^= 1;
        if (++hf == NH) {
          hf = 0;
          t += gridDim.x;
          ++kt;
        }
      }
    }
  } else {
    // ---- the epilogue (512 threads)
    const int part = warp >> 2;
    const int row = (warp & 3) * 32 + (threadIdx.x & 31);
    const int c0 = part * 32;
    const uint32_t ta = quad_addr(c);
    bf16* yd = reinterpret_cast<bf16*>(ws + Lw.yd);   // fp16 bits; rows copied as bytes
    float* part_rec = reinterpret_cast<float*>(ws + Lw.part);
    // The four warps of a TMEM lane quadrant hold the same 32 rows (one part
    // each): reductions over a row's parts synchronise the quadrant only, the
    // hand-offs to the issuer are one arrival per warp, and each quadrant
    // stores its own rows of Yd (its leader's bulk group).
    const int quad = warp & 3;
    const bool qlead = part == 0 && (threadIdx.x & 31) == 0;
    auto qbar = [&]() { named_bar_sync(2 + quad, 128); };
    auto warp_arrive = [&](uint64_t* b) {
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(b);
    };
    if (HIST && qlead) prefetch_tmap(&tmY);
    // LN1 statistics of this thread's row of an E tile (biased variance; see
    // layer_norm_part): mean and rstd into mu, rs, and every row's pair into
    // smu (rstd in log2 units for phi = softmax).  A quadrant barrier, then an
    // epilogue barrier (the link softmax reads every row's pair).
    auto ln1_stats = [&](const uint8_t* tileE, float* smu, float& mu, float& rs) {
      // the part's mean, then its centred sum of squares (a second read of
      // the tile's 32 values; see part_stats)
      float pm = 0.f, pq = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float x[8];
        unpack8(sw_ld16(tileE, kBlk, row, c0 + q * 8), x);
#pragma unroll
        for (int k = 0; k < 8; ++k) pm += x[k];
      }
      pm *= 1.0f / 32;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float x[8];
        unpack8(sw_ld16(tileE, kBlk, row, c0 + q * 8), x);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float dlt = x[k] - pm;
          pq = fmaf(dlt, dlt, pq);
        }
      }
      redS[part * 128 + row] = pm;
      redS[512 + part * 128 + row] = pq;
      qbar();
      merge4_stats(redS[row], redS[128 + row], redS[256 + row], redS[384 + row], redS[512 + row],
                   redS[640 + row], redS[768 + row], redS[896 + row], mu, rs);
      if (part == 0) {
        smu[row] = mu;
        smu[128 + row] = SILU ? rs : rs * kLog2e;   // softmax: log2 units
      }
      named_bar_sync(1, kXaEpi);
    };
    // History layers with l <= 32 compute the next tile's statistics while
    // this tile's Yd product runs (after its link records), instead of at
    // the head of the next tile's chain.
    constexpr bool kPre = HIST && !SPLIT;
    float mu_n = 0.f, rs_n = 0.f;
    bool pre = false;
    int ab = 0, t = blockIdx.x, hf = 0;
    for (int it = 0; t < n_tiles; ++it) {
      const int4 tl = tiles[t];
      const int r0 = tl.y, nv = tl.z;
      const uint32_t ph = (uint32_t)it & 1u;
      uint8_t* sA = rot + ab * kSlot;
      uint8_t* sB = rot + (ab ^ 1) * kSlot;
      const uint32_t tS2 = ta + 128 + (SPLIT ? 0u : (uint32_t)(it & 1) * 256);
      const int pr = hf * 128 + row;   // this lane's (head, link) pair in the link branch
      const float* vec = vecs + (it & 1) * 512;   // cQ, dQ, cG, dG
      float* smu = smu2 + (it & 1) * 256;
      mbar_wait(&bar[2], ph, status, c.abort_flag);
      if (it == 0) mbar_wait(&bar[0], 0, status, c.abort_flag);
      mbar_wait(&bar[4], ph, status, c.abort_flag);
      // LN1 statistics of this thread's row (computed ahead, or now)
      float mu_r, rs_r;
      if (pre) {
        mu_r = mu_n;
        rs_r = rs_n;
      } else {
        ln1_stats(sA, smu, mu_r, rs_r);
      }
      mbar_wait(&bar[1], ph, status, c.abort_flag);
      tc_fence_after();
      // link softmax over the tile's valid rows: row = (head, link) lane of
      // the half, part = a quarter of the tokens.  Pairs >= H*L carry no link.
      float lm, ls;
      {
        float z[32];
        tmem_ld16(tS2 + c0, z);
        tmem_ld16(tS2 + c0 + 16, z + 16);
        tmem_ld_wait();
        // all pairs of a half are links once H*L fills it; masking is only
        // needed for a tile's invalid rows (a partial tile) or missing links
        constexpr bool kAllLinks = HL % 128 == 0;
        const bool link = kAllLinks || pr < HL;
        const bool full = nv == kTile && kAllLinks;
        const float cq = link ? vec[row] : 0.f, dq = link ? vec[128 + row] : 0.f;
        const float4* mu4 = reinterpret_cast<const float4*>(smu + c0);
        const float4* rs4 = reinterpret_cast<const float4*>(smu + 128 + c0);
        float m = -INFINITY;
        auto scores = [&](auto masked) {
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 mv = mu4[j4], rv = rs4[j4];
            const float mj[4] = {mv.x, mv.y, mv.z, mv.w}, rj[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = j4 * 4 + e;
              z[j] = fmaf(rj[e], fmaf(-mj[e], cq, z[j]), dq);
              if constexpr (decltype(masked)::value) {
                if (c0 + j >= nv || !link) z[j] = -INFINITY;
              }
              m = fmaxf(m, z[j]);
            }
          }
        };
        if (full)
          scores(std::false_type{});
        else
          scores(std::true_type{});
        if constexpr (SILU) {
          // pointwise weights: SiLU of each valid score; the record's (max,
          // sum) = (0, valid tokens) makes the merge's total divide by N_u
#pragma unroll
          for (int j = 0; j < 32; ++j) z[j] = c0 + j < nv && link ? silu_fast(z[j]) : 0.f;
          if (HIST && it > 0 && qlead) bulk_wait_read<0>();
          qbar();
          lm = 0.f;
          ls = (float)nv;
        } else {
          redX[part * 128 + row] = m;
          // B held the previous tile's Yd staging: the quadrant's store must
          // have read its rows
          if (HIST && it > 0 && qlead) bulk_wait_read<0>();
          qbar();
          m = fmaxf(fmaxf(redX[row], redX[128 + row]), fmaxf(redX[256 + row], redX[384 + row]));
          // masked scores are -inf and give 0; a lane with no link at all
          // has m = -inf and takes m = 0 instead
          if (m == -INFINITY) m = 0.f;
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            z[j] = ex2_approx(z[j] - m);
            s += z[j];
          }
          redX[512 + part * 128 + row] = s;
          qbar();
          lm = m * kLn2;   // the record's max in natural-log units
          ls = redX[512 + row] + redX[640 + row] + redX[768 + row] + redX[896 + row];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sB, kBlk, row, c0 + q * 8, pack8(z + q * 8));
      }
      {
        // V_E (bf16) over the G' image (read by S): the MN-major B of P2 V_E
        mbar_wait(&bar[7], ph, status, c.abort_flag);
        if (HIST) mbar_wait(&bar[8], ph, status, c.abort_flag);
        tc_fence_after();
        float v[32];
        tmem_ld16(ta + 256 + c0, v);
        tmem_ld16(ta + 256 + c0 + 16, v + 16);
        tmem_ld_wait();
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          // cv, dv of this part's columns as float4 (shared by the warp: broadcast)
          const float4 cv4 = reinterpret_cast<const float4*>(cvd + c0)[j4];
          const float4 dv4 = reinterpret_cast<const float4*>(cvd + kD + c0)[j4];
          const float cvj[4] = {cv4.x, cv4.y, cv4.z, cv4.w}, dvj[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * j4 + e;
            v[j] = fmaf(rs_r, fmaf(-mu_r, cvj[e], v[j]), dvj[e]);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sG, kBlk, row, c0 + q * 8, pack8(v + q * 8));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bar[12]);   // P2 V_E starts once every warp has arrived
      if constexpr (HIST && !SPLIT) {
        // history softmax over the user's L links: part = head, P over the E tile
        const int h = part;
        float z[L];
#pragma unroll
        for (int q = 0; q < L / 16; ++q) tmem_ld16(ta + h * L + q * 16, z + q * 16);
        tmem_ld_wait();
        const float rsl = SILU ? rs_r : rs_r * kLog2e;   // softmax: log2 units
        {
          // cG, dG of head h's links as float4 (shared by the warp: broadcast)
          const float4* cg4 = reinterpret_cast<const float4*>(vec + 256 + h * L);
          const float4* dg4 = reinterpret_cast<const float4*>(vec + 384 + h * L);
#pragma unroll
          for (int q = 0; q < L / 4; ++q) {
            const float4 a = cg4[q], b = dg4[q];
            z[4 * q] = fmaf(rsl, fmaf(-mu_r, a.x, z[4 * q]), b.x);
            z[4 * q + 1] = fmaf(rsl, fmaf(-mu_r, a.y, z[4 * q + 1]), b.y);
            z[4 * q + 2] = fmaf(rsl, fmaf(-mu_r, a.z, z[4 * q + 2]), b.z);
            z[4 * q + 3] = fmaf(rsl, fmaf(-mu_r, a.w, z[4 * q + 3]), b.w);
          }
        }
        if constexpr (SILU) {
#pragma unroll
          for (int k = 0; k < L; ++k) z[k] = silu_fast(z[k]) * (1.0f / L);
        } else {
          float m = z[0];
#pragma unroll
          for (int k = 1; k < L; ++k) m = fmaxf(m, z[k]);
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < L; ++k) { z[k] = ex2_approx(z[k] - m); s += z[k]; }
          const float inv = 1.0f / s;
#pragma unroll
          for (int k = 0; k < L; ++k) z[k] *= inv;
        }
#pragma unroll
        for (int q = 0; q < L / 8; ++q) sw_st16(sA, kBlk, row, h * L + q * 8, pack8(z + q * 8));
      }
      if constexpr (HIST && SPLIT) {
        // two halves: the half's 128 score columns are heads 2hf and 2hf+1
        // with L = 64 links each; part p holds 32 links of head 2hf + p/2, and
        // the parts p, p^1 of a head combine their max and sum
        float z[32];
        tmem_ld16(ta + c0, z);
        tmem_ld16(ta + c0 + 16, z + 16);
        tmem_ld_wait();
        const float rsl = SILU ? rs_r : rs_r * kLog2e;   // softmax: log2 units
        {
          const float4* cg4 = reinterpret_cast<const float4*>(vec + 256 + c0);
          const float4* dg4 = reinterpret_cast<const float4*>(vec + 384 + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 a = cg4[q], b = dg4[q];
            z[4 * q] = fmaf(rsl, fmaf(-mu_r, a.x, z[4 * q]), b.x);
            z[4 * q + 1] = fmaf(rsl, fmaf(-mu_r, a.y, z[4 * q + 1]), b.y);
            z[4 * q + 2] = fmaf(rsl, fmaf(-mu_r, a.z, z[4 * q + 2]), b.z);
            z[4 * q + 3] = fmaf(rsl, fmaf(-mu_r, a.w, z[4 * q + 3]), b.w);
          }
        }
        if constexpr (SILU) {
#pragma unroll
          for (int k = 0; k < 32; ++k) z[k] = silu_fast(z[k]) * (1.0f / L);
        } else {
          float m = z[0];
#pragma unroll
          for (int k = 1; k < 32; ++k) m = fmaxf(m, z[k]);
          redX[part * 128 + row] = m;
          qbar();
          m = fmaxf(m, redX[(part ^ 1) * 128 + row]);
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k) { z[k] = ex2_approx(z[k] - m); s += z[k]; }
          redX[512 + part * 128 + row] = s;
          qbar();
          const float inv = 1.0f / (s + redX[512 + (part ^ 1) * 128 + row]);
#pragma unroll
          for (int k = 0; k < 32; ++k) z[k] *= inv;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sA, kBlk, row, c0 + q * 8, pack8(z + q * 8));
      }
      if (HIST) {
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(&bar[13]);   // Yd = P VO starts once every warp has arrived
      }
      mbar_wait(&bar[9], ph, status, c.abort_flag);
      tc_fence_after();
      {
        // link record of row p = (h, k): part h reads head h's 32 columns
        // (warp-uniform TMEM address); rows of other heads skip the store
        float acc[kDH];
        tmem_ld16(tS2 + part * kDH, acc);
        tmem_ld16(tS2 + part * kDH + 16, acc + 16);
        tmem_ld_wait();
        if (pr < HL && pr / L == part) {
          float4* rec = reinterpret_cast<float4*>(part_rec + ((size_t)t * HL + pr) * kRec);
          rec[0] = make_float4(lm, ls, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            rec[1 + q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
        if constexpr (SPLIT) {
          // the next half's link scores reuse these columns
          tc_fence_before();
          warp_arrive(&bar[5]);
        }
      }
      if constexpr (kPre) {
        // the next tile's E rows land in B once P2 V_E is done (above):
        // their statistics now, while this tile's Yd product runs
        pre = t + (int)gridDim.x < n_tiles;
        if (pre) {
          mbar_wait(&bar[2], ph ^ 1u, status, c.abort_flag);
          ln1_stats(sB, smu2 + ((it + 1) & 1) * 256, mu_n, rs_n);
        }
      }
      if (HIST) mbar_wait(&bar[10], ph, status, c.abort_flag);   // P has been read
      if (HIST && hf == NH - 1) {
        // the tile's Yd (two halves: accumulated over both)
        tc_fence_after();
        float y[32];
        tmem_ld16(ta + kYd + c0, y);
        tmem_ld16(ta + kYd + c0 + 16, y + 16);
        tmem_ld_wait();
        tc_fence_before();
        warp_arrive(&bar[11]);   // this warp has read its Yd columns (P: the MMA is done)
        // the staging rows are the quadrant's own: P's rows, which Yd has read
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sA, kBlk, row, c0 + q * 8, pack8_f16(y + q * 8));
        fence_proxy_async_smem();
        qbar();
        if (nv == kTile) {
          if (qlead) {
            tma_store_2d(&tmY, sA + quad * 4096, 0, r0 + 32 * quad);
            tma_store_2d(&tmY, sA + kBlk + quad * 4096, 64, r0 + 32 * quad);
            bulk_commit();
          }
        } else {
          for (int idx = part * 32 + (threadIdx.x & 31); idx < 512; idx += 128) {
            const int r = quad * 32 + (idx >> 4), cc = idx & 15;
            if (r < nv) reinterpret_cast<uint4*>(yd + (int64_t)(r0 + r) * kD)[cc] = sw_ld16(sA, kBlk, r, cc * 8);
          }
        }
      }
      ab ^= 1;
      if (++hf == NH) {
        hf = 0;
        t += gridDim.x;
      }
    }
    if (qlead) bulk_wait<0>();
  }
  cta_teardown(c);
}

// ------------------------------------------------------- history GatedMLP
// E' = Y + GatedMLP(LN2(Y)), Y = E + Yd, for one 128-row history tile at a
// time, as a warp-specialized pipeline (persistent, one CTA per SM):
//   warps 0-15 (epilogue): warp w serves TMEM lane quadrant w % 4 (tile rows
//     32*(w%4) ...) and column part p = w / 4 (a quarter of every row).  Per
//     tile they form Y = E (TMA tile) + Yd (fp16 rows, prefetched into L2
//     with the E tile) and store it into the tile's output accumulator OUT,
//     so that the W2 products add the GatedMLP onto the residual in place;
//     write h2 = LN2(Y) (statistics reduced over the four parts through
//     shared memory) over the E tile; compute hid = SiLU(G1) * G3 per 64-wide
//     hidden chunk from TMEM GB[g%2] into smem HB[g%2]; and store E' = OUT.
//     The next tile's Y and LN2 run before this tile's E' is read out, so the
//     tensor cores start the next tile while the epilogue finishes this one.
//   warp 16 (one lane) issues the MMAs: G(g) = h2 [W1c | W3c] (one N = 128
//     product) into GB[g%2] and OUT += hid(g) W2c with W2 resident in shared
//     memory.
//   warp 17 (one lane) loads: the E tiles (one tile ahead) and the [W1c | W3c]
//     chunk images through a two-slot ring (chunk g+1 is fetched as soon as
//     G(g-1) has consumed its slot).
// Chunks are counted over the CTA's whole tile sequence (g = 4*k + c for its
// k-th tile), so every ring barrier's parity is (g / 2) % 2.
// TMEM: GB[0] [0,128), GB[1] [128,256), OUT[k%2] [256 + 128*(k%2), +128).
constexpr int kFfnEpi = 512;   // epilogue threads (two groups of 256)
constexpr int kFfnGrp = 256;
constexpr int kFfnTiles = 32;  // tile descriptors of a CTA kept in shared memory
constexpr int kFfnSmem = 1024 + 14 * kBlk + 1024 + kFfnTiles * 16 + 256;

__global__ void __launch_bounds__(kFfnEpi + 96, 1)
    k_hist_ffn(const __grid_constant__ CUtensorMap tmE, const bf16* __restrict__ g2,
               const bf16* __restrict__ b2, const uint8_t* __restrict__ ws, LayerWs Lw,
               bf16* __restrict__ E_out, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1k(smem_raw);
  uint8_t* sE0 = sm;                   // 2 x [128 x 128] bf16: E tile -> h2 (-> LN2 scratch)
  uint8_t* sH0 = sm + 4 * kBlk;        // 2 x [128 x 64]  bf16: hid chunk
  uint8_t* sW13 = sm + 6 * kBlk;       // 2 x [W1c | W3c] ring
  uint8_t* sW2 = sm + 10 * kBlk;       // W2 image, 4 chunks
  float* sg = reinterpret_cast<float*>(sm + 14 * kBlk);   // g2, b2 as fp32 [2][128]
  int4* s_tiles = reinterpret_cast<int4*>(sm + 14 * kBlk + 1024);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 14 * kBlk + 1024 + kFfnTiles * 16);
  uint64_t* barE = bar;        // [2] E tile landed (TMA)
  uint64_t* barWt = bar + 2;   // [2] [W1c | W3c] ring slot landed
  uint64_t* barG = bar + 4;    // [2] G(g) in TMEM (MMA commit)
  uint64_t* barHid = bar + 6;  // [2] hid(g) written, GB read (epilogue arrivals)
  uint64_t* barW2 = bar + 8;   // [2] OUT += hid(g) W2c done (MMA commit)
  uint64_t* barH2 = bar + 10;  // Y in OUT and h2 written (epilogue arrivals)
  uint64_t* barOut = bar + 11; // all of the tile's MMAs done (MMA commit)
  uint64_t* barW2in = bar + 12;  // W2 image landed
  uint64_t* barDrain = bar + 13; // every MMA issued by the control lane is done
  uint64_t* barSE = bar + 14;    // E'(j) staging read out of E buffer j%2 (row-group arrivals)
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 15);
  int* abort_flag = reinterpret_cast<int*>(bar + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&barE[q], 1);
      mbar_init(&barWt[q], 1);
      mbar_init(&barG[q], 1);
      mbar_init(&barHid[q], kFfnGrp);
      mbar_init(&barW2[q], 1);
    }
    mbar_init(barH2, kFfnGrp);
    mbar_init(barSE, kFfnGrp);
    mbar_init(barOut, 1);
    mbar_init(barW2in, 1);
    mbar_init(barDrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  pdl_launch();
  pdl_wait();
  const int n_tiles = *reinterpret_cast<const int*>(ws + Lw.sched);
  const int4* tiles = reinterpret_cast<const int4*>(ws + Lw.tiles);
  const int my_tiles =
      (int)blockIdx.x < n_tiles ? (n_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  if (threadIdx.x < kD) {
    sg[threadIdx.x] = __bfloat162float(g2[threadIdx.x]);
    sg[kD + threadIdx.x] = __bfloat162float(b2[threadIdx.x]);
  }
  if ((int)threadIdx.x < my_tiles && threadIdx.x < kFfnTiles)
    s_tiles[threadIdx.x] = tiles[blockIdx.x + threadIdx.x * gridDim.x];
  __syncthreads();
  constexpr uint32_t T_OUT = 256;
  auto tile_of = [&](int k) -> int4 {
    return k < kFfnTiles ? s_tiles[k] : tiles[blockIdx.x + k * gridDim.x];
  };
  const int n_chunks = my_tiles * (kF / 64);

  if (warp == kFfnEpi / 32 + 2) {
    // E-tile loader: E(0), E(1), then E(k+2) into buffer k%2 once the row
    // group has read tile k's E' staging out of it.  Apart from the weight
    // loader, so the W1|W3 ring never waits on the readout.
    if (lane == 0 && my_tiles > 0) {
      auto load_e = [&](int k) {
        const int4 tl = tile_of(k);
        uint8_t* dst = sE0 + (k & 1) * 2 * kBlk;
        mbar_arrive_expect_tx(&barE[k & 1], 2 * kBlk);
        tma_load_2d(dst, &tmE, 0, tl.y, &barE[k & 1]);
        tma_load_2d(dst + kBlk, &tmE, 64, tl.y, &barE[k & 1]);
        // the tile's Yd rows into L2, for the epilogue's plain loads
        bulk_prefetch_l2(reinterpret_cast<const __half*>(ws + Lw.yd) + (int64_t)tl.y * kD,
                         (uint32_t)tl.z * kD * 2);
      };
      prefetch_tmap(&tmE);
      load_e(0);
      if (my_tiles > 1) load_e(1);
      for (int k = 0; k + 2 < my_tiles; ++k) {
        // buffer k%2 held h2(k) and then tile k's E' staging
        if (!mbar_wait(barSE, k & 1, status, abort_flag)) break;
        load_e(k + 2);
        // E(k+3) into L2: its load waits for the next readout
        if (k + 3 < my_tiles) {
          const int4 tp = tile_of(k + 3);
          tma_prefetch_2d(&tmE, 0, tp.y);
          tma_prefetch_2d(&tmE, 64, tp.y);
        }
      }
    }
  } else if (warp == kFfnEpi / 32 + 1) {
    // weight loader: the W1|W3 ring and W2.  It runs apart from the MMA
    // issuer because tcgen05.mma issue stalls while the tensor pipe is busy,
    // which would hold back the next loads.
    if (lane == 0 && my_tiles > 0) {
      auto load_w13 = [&](int g) {
        const int s = g & 1, ch = g & 3;
        mbar_arrive_expect_tx(&barWt[s], 2 * kBlk);
        bulk_load(sW13 + s * 2 * kBlk, ws + Lw.img_13 + ch * 2 * kBlk, 2 * kBlk, &barWt[s]);
      };
      load_w13(0);
      if (n_chunks > 1) load_w13(1);
      mbar_arrive_expect_tx(barW2in, 4 * kBlk);
      bulk_load(sW2, ws + Lw.img_2, 4 * kBlk, barW2in);
      for (int g = 1; g + 1 < n_chunks; ++g) {
        // G(g-1) done: its ring slot takes chunk g+1
        if (!mbar_wait(&barG[(g - 1) & 1], (uint32_t)(((g - 1) >> 1) & 1), status, abort_flag))
          break;
        load_w13(g + 1);
      }
    }
  } else if (warp == kFfnEpi / 32) {
    // MMA issuer
    if (lane == 0 && my_tiles > 0) {
      // G(k, c) = h2(k) [W1c | W3c] into gate buffer g%2 (g = 4k + c)
      auto gate = [&](int k, int c) {
        const int g = k * (kF / 64) + c, s = g & 1;
        if (!mbar_wait(&barWt[s], (uint32_t)((g >> 1) & 1), status, abort_flag)) return false;
        tc_fence_after();
        mma_tile(tmem + s * 128, smem_u32(sE0 + (k & 1) * 2 * kBlk), kBlk,
                 smem_u32(sW13 + s * 2 * kBlk), kBlk, 128, 128, false);
        mma_commit(&barG[s]);
        return true;
      };
      bool ok = mbar_wait(barW2in, 0, status, abort_flag);
      bool g0 = false;   // G(k, 0) already issued (ahead of tile k-1's last W2 product)
      for (int k = 0; k < my_tiles && ok; ++k) {
        const uint32_t t_out = tmem + T_OUT + (k & 1) * 128;
        if (!g0) {
          if (!(ok = mbar_wait(barH2, k & 1, status, abort_flag))) break;
          tc_fence_after();
          if (!(ok = gate(k, 0))) break;
        }
        g0 = false;
        for (int c = 0; c < kF / 64; ++c) {
          const int g = k * (kF / 64) + c;
          if (c >= 1 && !(ok = gate(k, c))) break;
          if (c >= 1) {
            const int pg = g - 1, pb = pg & 1;
            if (!(ok = mbar_wait(&barHid[pb], (uint32_t)((pg >> 1) & 1), status, abort_flag))) break;
            tc_fence_after();
            mma_tile(t_out, smem_u32(sH0 + pb * kBlk), kBlk, smem_u32(sW2 + (c - 1) * kBlk), kBlk,
                     128, 64, true);
            mma_commit(&barW2[pb]);
          }
        }
        if (!ok) break;
        const int lg = k * (kF / 64) + kF / 64 - 1, lb = lg & 1;
        // Whichever is ready first: the next tile's first gate product (its
        // gate buffer is the other one) or this tile's last W2 product.
        if (k + 1 < my_tiles) {
          const uint64_t t0 = global_ns();
          for (;;) {
            if (mbar_try_wait_ns(barH2, (k + 1) & 1, 20)) {
              tc_fence_after();
              if (!(ok = gate(k + 1, 0))) break;
              g0 = true;
              break;
            }
            if (mbar_try_wait_ns(&barHid[lb], (uint32_t)((lg >> 1) & 1), 20)) break;
            if (*abort_flag) { ok = false; break; }
            if (global_ns() - t0 > 2000000000ull) {
              raise_flag(status, LIME_FLAG_TIMEOUT);
              *abort_flag = 1;
              ok = false;
              break;
            }
          }
          if (!ok) break;
        }
        if (!(ok = mbar_wait(&barHid[lb], (uint32_t)((lg >> 1) & 1), status, abort_flag))) break;
        tc_fence_after();
        mma_tile(t_out, smem_u32(sH0 + lb * kBlk), kBlk, smem_u32(sW2 + (kF / 64 - 1) * kBlk), kBlk,
                 128, 64, true);
        mma_commit(&barW2[lb]);
        mma_commit(barOut);
      }
      // drain: no MMA of ours may be in flight when TMEM is freed
      mma_commit(barDrain);
      mbar_wait(barDrain, 0, status, abort_flag);
    }
  } else if (warp < kFfnGrp / 32) {
    // ---- row group (warps 0-7): thread (row, half), 64 columns of the row
    const int q4 = warp & 3, half = warp >> 2;
    const int row = q4 * 32 + lane;
    const int tid = (int)threadIdx.x;
    const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16);
    const int c0 = half * 64;
    const __half* yd = reinterpret_cast<const __half*>(ws + Lw.yd);
    // this thread's 64 fp16 Yd values of tile j (zeros past the tile's rows)
    auto load_yd = [&](int j, uint4* v) {
      const int4 tl = tile_of(j);
      if (row < tl.z) {
        const uint4* src = reinterpret_cast<const uint4*>(yd + (int64_t)(tl.y + row) * kD + c0);
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = src[q];
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = make_uint4(0, 0, 0, 0);
      }
    };
    // Y(j) = E + Yd into OUT[j%2]; h2(j) = LN2(Y(j)) over E buffer j%2.  Once
    // both halves have stored their Y, each thread reads the whole row back
    // from TMEM in column order for the statistics (so both halves normalise
    // with identical mu and rstd; shifted one-pass sums, shift = the row's
    // first value), then its own 64 columns again for h2.
    auto y_ln2 = [&](int j, const uint4* ydv) {
      uint8_t* sE = sE0 + (j & 1) * 2 * kBlk;
      const uint32_t t_out = ta + T_OUT + (j & 1) * 128;
      mbar_wait(&barE[j & 1], (uint32_t)((j >> 1) & 1), status, abort_flag);
      // LN2 statistics per half of the row: shifted sums (shift = the half's
      // first value) of 64 values, accumulated in column order.  This half's
      // come from the registers that form Y; the other half's are read back
      // from TMEM below, in the same order, so both threads of a row compute
      // bitwise the same two halves and the same merge.
      float K = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
      for (int p2 = 0; p2 < 2; ++p2) {
        float y[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float e[8];
          unpack8_f16(ydv[p2 * 4 + q], y + q * 8);
          unpack8(sw_ld16(sE, kBlk, row, c0 + p2 * 32 + q * 8), e);
#pragma unroll
          for (int i = 0; i < 8; ++i) y[q * 8 + i] += e[i];
        }
        if (p2 == 0) K = y[0];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float t = y[i] - K;
          s1 += t;
          s2 = fmaf(t, t, s2);
        }
        tmem_st16(t_out + c0 + p2 * 32, y);
        tmem_st16(t_out + c0 + p2 * 32 + 16, y + 16);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar_sync(1, kFfnGrp);   // both halves of every row are in OUT (and E is read)
      tc_fence_after();
      float Ko = 0.f, o1 = 0.f, o2 = 0.f;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        float o[32];
        tmem_ld16(t_out + (c0 ^ 64) + q * 32, o);
        tmem_ld16(t_out + (c0 ^ 64) + q * 32 + 16, o + 16);
        tmem_ld_wait();
        if (q == 0) Ko = o[0];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float t = o[i] - Ko;
          o1 += t;
          o2 = fmaf(t, t, o2);
        }
      }
      // each half's mean and centred sum of squares, merged for equal counts
      // (M2 = M2a + M2b + 128 ((ma - mb) / 2)^2; symmetric in the halves)
      const float ma = K + s1 * (1.0f / 64), mb = Ko + o1 * (1.0f / 64);
      const float qa = fmaxf(s2 - s1 * s1 * (1.0f / 64), 0.f);
      const float qb = fmaxf(o2 - o1 * o1 * (1.0f / 64), 0.f);
      const float mu = 0.5f * (ma + mb);
      const float dh = 0.5f * (ma - mb);
      const float rstd = rsqrtf((qa + qb + 128.0f * dh * dh) * (1.0f / kD) + kLnEps);
      // h2 of this thread's 64 columns, 16 at a time from TMEM
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float o[16];
        tmem_ld16(t_out + c0 + q * 16, o);
        tmem_ld_wait();
        const int cc = c0 + q * 16;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 gv = reinterpret_cast<const float4*>(sg + cc)[i4];
          const float4 bv = reinterpret_cast<const float4*>(sg + kD + cc)[i4];
          o[4 * i4] = (o[4 * i4] - mu) * rstd * gv.x + bv.x;
          o[4 * i4 + 1] = (o[4 * i4 + 1] - mu) * rstd * gv.y + bv.y;
          o[4 * i4 + 2] = (o[4 * i4 + 2] - mu) * rstd * gv.z + bv.z;
          o[4 * i4 + 3] = (o[4 * i4 + 3] - mu) * rstd * gv.w + bv.w;
        }
        sw_st16(sE, kBlk, row, cc, pack8(o));
        sw_st16(sE, kBlk, row, cc + 8, pack8(o + 8));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(barH2);
    };
    // E'(j) = OUT[j%2] -> bf16, staged over E buffer j%2 (h2(j) is dead once
    // every product of the tile is done) and written with coalesced stores
    auto out = [&](int j) {
      mbar_wait(barOut, (uint32_t)(j & 1), status, abort_flag);
      tc_fence_after();
      uint8_t* sE = sE0 + (j & 1) * 2 * kBlk;
#pragma unroll
      for (int p2 = 0; p2 < 2; ++p2) {
        float o[32];
        tmem_ld16(ta + T_OUT + (j & 1) * 128 + c0 + p2 * 32, o);
        tmem_ld16(ta + T_OUT + (j & 1) * 128 + c0 + p2 * 32 + 16, o + 16);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sE, kBlk, row, c0 + p2 * 32 + q * 8, pack8(o + q * 8));
      }
      tc_fence_before();
      named_bar_sync(1, kFfnGrp);   // the staging tile is complete
      const int4 tl = tile_of(j);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int idx = q * kFfnGrp + tid, r = idx >> 4, cc = idx & 15;
        if (r < tl.z)
          reinterpret_cast<uint4*>(E_out + (int64_t)(tl.y + r) * kD)[cc] = sw_ld16(sE, kBlk, r, cc * 8);
      }
      mbar_arrive(barSE);   // this thread has read its part of the staging
    };
    uint4 ydv[8];
    if (my_tiles > 0) load_yd(0, ydv);
    for (int j = 0; j <= my_tiles; ++j) {
      if (j < my_tiles) {
        y_ln2(j, ydv);
        // the next tile's Yd rows, in flight while this group reads out E'(j-1)
        if (j + 1 < my_tiles) load_yd(j + 1, ydv);
      }
      if (j >= 1) out(j - 1);
    }
  } else {
    // ---- chunk group (warps 8-15): thread (row, half): hidden units
    //      32 half .. 32 half + 31 of every 64-wide chunk
    const int q4 = warp & 3, half = (warp >> 2) & 1;
    const int row = q4 * 32 + lane;
    const uint32_t ta = tmem + ((uint32_t)(q4 * 32) << 16);
    for (int k = 0; k < my_tiles; ++k) {
      for (int c = 0; c < kF / 64; ++c) {
        const int g = k * (kF / 64) + c, sb = g & 1;
        mbar_wait(&barG[sb], (uint32_t)((g >> 1) & 1), status, abort_flag);
        tc_fence_after();
        float h[32];
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
          float gt[16], gu[16];
          tmem_ld16(ta + sb * 128 + half * 32 + p2 * 16, gt);
          tmem_ld16(ta + sb * 128 + 64 + half * 32 + p2 * 16, gu);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) h[p2 * 16 + i] = silu_tanh(gt[i]) * gu[i];
        }
        // hid(g) reuses the buffer of hid(g-2): wait until its W2 MMA is done
        if (g >= 2) mbar_wait(&barW2[sb], (uint32_t)(((g - 2) >> 1) & 1), status, abort_flag);
        uint8_t* sH = sH0 + sb * kBlk;
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(sH, kBlk, row, half * 32 + q * 8, pack8(h + q * 8));
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&barHid[sb]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------ LIME-XOR+Window history
// With a window (LIME note, 关键设计 3: a history token also attends to its
// neighbouring history tokens), a history query's keys are the user's l links
// and the history rows j with 0 < |i - j| <= window, under one phi.  The link
// branch is unchanged (k_hist_xattn without its history branch); the history
// branch runs as
//   k_rows_proj  LN1 and the Q, K, V projections of the history rows, and K, V
//                of the link rows (tensor cores; bf16 outputs)
//   k_win_attn   per (history row, head): phi over the l link keys and the
//                window keys (CUDA cores: 2 * window + l keys of 32 dims each,
//                far too little work per query for a tensor-core tile)
//   k_rows_proj  Yd = A Wo (fp16), which the GatedMLP kernel reads as usual.

// out_w[r, :] = x_r W_w, x_r = LN1(X[r, :]) (LN) or X[r, :] (X bf16, or fp32
// for IN_F32), with W_w^T's K-major image at ws + img[w].  x_r enters the
// products split into bf16 hi + lo (two MMAs each), so the fp32 outputs carry
// no bf16 rounding of the operand.  Two jobs share one persistent launch: job
// 0 (n0 rows of x[0], outputs o[0 .. NW)) and job 1 (n1 rows of x[1], the
// products with images 1 and 2 into o[3], o[4]; the link rows' K and V beside
// the history rows' Q, K, V).  Persistent CTAs of 512 threads walk the 128-row
// tiles of both jobs; the weight images are loaded once per CTA.  A tile's
// rows arrive by TMA (the next tile's load is issued as soon as this one has
// been read), thread (row, part) normalises and splits its 32 columns, one
// thread issues the products, and each output leaves by TMA tensor stores from
// a staging buffer over the dead operands (128-byte swizzled boxes: four
// fp32 boxes of 32 columns, or two fp16 boxes of 64; rows past the end are
// clipped by the stores and zero-filled by the loads).
struct RowsMaps {
  CUtensorMap x[2];
  CUtensorMap o[5];
};
struct RowsImgs {
  uint32_t img[3];
};

template <int NW, bool LN, bool IN_F32, bool F16>
__global__ void __launch_bounds__(512, 1)
    k_rows_proj(const __grid_constant__ RowsMaps tm, int64_t n0, int64_t n1,
                const bf16* __restrict__ g, const bf16* __restrict__ b,
                const uint8_t* __restrict__ ws, RowsImgs im, unsigned* status) {
  constexpr uint32_t kCols = NW == 1 ? 128 : (NW == 2 ? 256 : 512);
  constexpr uint32_t kXBytes = IN_F32 ? 4 * kBlk : 2 * kBlk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1k(smem_raw);
  uint8_t* sAh = sm;
  uint8_t* sAl = sm + 2 * kBlk;
  uint8_t* stage = sm;   // 64 KB over sAh and sAl once a tile's products are done
  uint8_t* sW = sm + 4 * kBlk;
  uint8_t* sX = sW + NW * 2 * kBlk;
  float* red = reinterpret_cast<float*>(sX + kXBytes);
  Cta c;
  // bar: 0 weights, 1 products, 2 row tile
  cta_setup(sX + kXBytes + kLnBytes, 3, c, kCols);
  if (LN) ln_stage(red + 1024, g, b);
  const int64_t T0 = (n0 + kTile - 1) / kTile, T = T0 + (n1 + kTile - 1) / kTile;
  auto load_x = [&](int64_t tile) {
    const bool j1 = tile >= T0;
    const int row0 = (int)((j1 ? tile - T0 : tile) * kTile);
    mbar_arrive_expect_tx(&c.bar[2], kXBytes);
#pragma unroll
    for (int p = 0; p < (IN_F32 ? 4 : 2); ++p)
      tma_load_2d(sX + p * kBlk, &tm.x[j1 ? 1 : 0], p * (IN_F32 ? 32 : 64), row0, &c.bar[2]);
  };
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&c.bar[0], NW * 2 * kBlk);
#pragma unroll
    for (int w = 0; w < NW; ++w) bulk_load(sW + w * 2 * kBlk, ws + im.img[w], 2 * kBlk, &c.bar[0]);
    if ((int64_t)blockIdx.x < T) load_x(blockIdx.x);
  }
  const int warp = threadIdx.x >> 5;
  const int part = warp >> 2;
  const int r = (warp & 3) * 32 + (threadIdx.x & 31);
  const int c0 = part * 32;
  const uint32_t ta = quad_addr(c);
  uint32_t mph = 0;
  int k = 0;
  for (int64_t tile = blockIdx.x; tile < T; tile += gridDim.x, ++k) {
    const bool j1 = tile >= T0;
    const int row0 = (int)((j1 ? tile - T0 : tile) * kTile);
    mbar_wait(&c.bar[2], (uint32_t)k & 1u, status, c.abort_flag);
    float x[32];
    if constexpr (IN_F32) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(sX + part * kBlk + r * 128 + ((j ^ (r & 7)) << 4));
        x[4 * j] = v.x; x[4 * j + 1] = v.y; x[4 * j + 2] = v.z; x[4 * j + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) unpack8(sw_ld16(sX, kBlk, r, c0 + q * 8), x + q * 8);
    }
    if (LN) layer_norm_part(x, c0, red, part, r);
    // the previous tile's stores have read the staging (= this tile's operands)
    if (threadIdx.x == 0) bulk_wait_read<0>();
    __syncthreads();   // every thread has read the row tile
    if (threadIdx.x == 0 && tile + gridDim.x < T) load_x(tile + gridDim.x);
    split_part_st(sAh, sAl, r, c0, x);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (k == 0) mbar_wait(&c.bar[0], 0, status, c.abort_flag);
    const int nout = j1 ? 2 : NW;
    if (threadIdx.x == 0) {
      tc_fence_after();
      for (int w = 0; w < nout; ++w) {
        const uint8_t* wimg = sW + (j1 ? w + 1 : w) * 2 * kBlk;
        mma_tile(c.tmem + w * 128, smem_u32(sAh), kBlk, smem_u32(wimg), kBlk, 128, 128, false);
        mma_tile(c.tmem + w * 128, smem_u32(sAl), kBlk, smem_u32(wimg), kBlk, 128, 128, true);
      }
    }
    cta_mma_wait(&c.bar[1], mph, status, c.abort_flag);
#pragma unroll 1
    for (int w = 0; w < nout; ++w) {
      float v[32];
      tmem_ld16(ta + w * 128 + c0, v);
      tmem_ld16(ta + w * 128 + c0 + 16, v + 16);
      tmem_ld_wait();
      if (w > 0) {
        if (threadIdx.x == 0) bulk_wait_read<0>();   // the previous output's stores
        __syncthreads();
      }
      if constexpr (F16) {
#pragma unroll
        for (int q = 0; q < 4; ++q) sw_st16(stage, kBlk, r, c0 + q * 8, pack8_f16(v + q * 8));
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(stage + part * kBlk + r * 128 + ((j ^ (r & 7)) << 4)) =
              make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (threadIdx.x == 0) {
        const CUtensorMap* om = &tm.o[j1 ? 3 + w : w];
#pragma unroll
        for (int p = 0; p < (F16 ? 2 : 4); ++p)
          tma_store_2d(om, stage + p * kBlk, p * (F16 ? 64 : 32), row0);
        bulk_commit();
      }
    }
  }
  if (threadIdx.x == 0) bulk_wait<0>();
  cta_teardown(c);
}

// A[i, head h] = sum over keys phi(s q_i . k) v for history row i of user u
// (fp32 throughout): the keys are u's l link rows (Kz, Vz) and its history
// rows j with 0 < |i - j| <= win (Ke, Ve); phi = softmax or SiLU / (number of
// keys).  A block takes kWinRows consecutive history rows, warp w the eight
// rows r0 + 8 w .. r0 + 8 w + 7.  Lane = (row group g, head h, quarter c):
// it holds dims 8c .. 8c + 7 of head h of the four rows 4g .. 4g + 3 of the
// warp, so every key value it loads feeds four rows.  Key rows are staged in
// shared memory, kWinBuf at a time (first each user's link rows, then the
// block's window range), and a warp walks its keys in lockstep: at a step the
// lanes read one key row (the heads padded to 36 floats so that the eight
// 16-byte slices of a load sit in distinct banks).  The four quarter sums of
// a row are combined by a reduce-scatter over the lane's quad, after which
// lane c owns row 4g + c: it applies the row's mask, keeps the row's softmax
// state and hands its weight to the quad (four shuffles).  The softmax keeps
// a reference value m per row and rescales only when a score passes
// m + 8 (in log2 units; weights stay below 2^8), the warp then broadcasting
// each row's factor; the result acc / sum is the same quotient as with the
// running maximum.
constexpr int kWinRows = 64;
constexpr int kWinBuf = 96;
constexpr int kWinPitch = 4 * (kDH + 4);
constexpr int kWinSmem = 2 * kWinBuf * kWinPitch * 4;
static_assert(kWinRows == 8 * 8, "eight warps of eight rows");

__device__ __forceinline__ void win_stage(float* sK, float* sV, const float* __restrict__ K,
                                          const float* __restrict__ V, int64_t row0, int nrows) {
  for (int t = threadIdx.x; t < nrows * 32; t += blockDim.x) {
    const int r = t >> 5, c4 = t & 31;
    const int dst = r * kWinPitch + (c4 >> 3) * (kDH + 4) + (c4 & 7) * 4;
    const int64_t src = (row0 + r) * kD + c4 * 4;
    cp_async16(sK + dst, K + src, true);
    cp_async16(sV + dst, V + src, true);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
}

__global__ void __launch_bounds__(256, 2)
    k_win_attn(const float* __restrict__ Qe, const float* __restrict__ Ke, const float* __restrict__ Ve,
               const float* __restrict__ Kz, const float* __restrict__ Vz,
               const int64_t* __restrict__ off, int64_t B, int64_t nh, int L, int win, float scale,
               int silu, float* __restrict__ att) {
  constexpr unsigned kAll = 0xffffffffu;
  extern __shared__ float4 win_smem[];
  float* sK = reinterpret_cast<float*>(win_smem);
  float* sV = sK + kWinBuf * kWinPitch;
  pdl_launch();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane & 3, h = (lane >> 2) & 3, g = lane >> 4;
  const bool b0 = c & 1, b1 = c & 2;
  const int quad = lane & ~3;
  const int64_t r0 = (int64_t)blockIdx.x * kWinRows;
  const int64_t w0 = r0 + warp * 8;      // the warp's first row
  const int64_t rg = w0 + 4 * g;         // the lane's first row
  const int64_t i = rg + c;              // the row this lane keeps the state of
  const int64_t rlast = (r0 + kWinRows < nh ? r0 + kWinRows : nh) - 1;
  // softmax scores in log2 units (exp(x) = 2^(x log2 e))
  const float qs = silu ? scale : scale * kLog2e;
  float q[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t ir = rg + r;
    if (ir < nh) {
      const float4* src = reinterpret_cast<const float4*>(Qe + ir * kD + h * kDH + 8 * c);
      const float4 v0 = src[0], v1 = src[1];
      q[r][0] = v0.x * qs; q[r][1] = v0.y * qs; q[r][2] = v0.z * qs; q[r][3] = v0.w * qs;
      q[r][4] = v1.x * qs; q[r][5] = v1.y * qs; q[r][6] = v1.z * qs; q[r][7] = v1.w * qs;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) q[r][k] = 0.f;
    }
  }
  int64_t u = -1, j0 = 0, j1 = -1;
  if (i < nh) {
    u = owner_of(off, B, i);
    int64_t a = off[u], b = off[u + 1];
    a = a < 0 ? 0 : a;
    b = b > nh ? nh : b;
    if (!(a <= i && i < b)) {
      a = i;   // offsets that give no owner (flagged by the layer's schedule)
      b = i + 1;
    }
    j0 = i - win > a ? i - win : a;
    j1 = i + win < b - 1 ? i + win : b - 1;
  }
  const float inv_n = 1.0f / (float)(L + (j1 - j0 > 0 ? j1 - j0 : 0));   // row i itself excluded
  const int loff = h * (kDH + 4) + 8 * c;   // the lane's floats in a staged row
  float m = -INFINITY, mthr = -INFINITY, ssum = 0.f, acc[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[r][k] = 0.f;
  // The lane's four quarter dots of one key, reduced over the quad: lane c
  // ends with the whole dot of row c.
  auto dot = [&](const float* krow) {
    const float4 k0 = reinterpret_cast<const float4*>(krow)[0];
    const float4 k1 = reinterpret_cast<const float4*>(krow)[1];
    float P[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float x = q[r][0] * k0.x;
      float y = q[r][1] * k0.y;
      x = fmaf(q[r][2], k0.z, x);
      y = fmaf(q[r][3], k0.w, y);
      x = fmaf(q[r][4], k1.x, x);
      y = fmaf(q[r][5], k1.y, y);
      x = fmaf(q[r][6], k1.z, x);
      y = fmaf(q[r][7], k1.w, y);
      P[r] = x + y;
    }
    float s0 = b1 ? P[2] : P[0], s1 = b1 ? P[3] : P[1];
    const float t0 = b1 ? P[0] : P[2], t1 = b1 ? P[1] : P[3];
    s0 += __shfl_xor_sync(kAll, t0, 2);
    s1 += __shfl_xor_sync(kAll, t1, 2);
    return (b0 ? s1 : s0) + __shfl_xor_sync(kAll, b0 ? s0 : s1, 1);
  };
  auto accumulate = [&](const float* vrow, float p) {
    const float4 v0 = reinterpret_cast<const float4*>(vrow)[0];
    const float4 v1 = reinterpret_cast<const float4*>(vrow)[1];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float pr = __shfl_sync(kAll, p, quad | r);
      acc[r][0] = fmaf(pr, v0.x, acc[r][0]);
      acc[r][1] = fmaf(pr, v0.y, acc[r][1]);
      acc[r][2] = fmaf(pr, v0.z, acc[r][2]);
      acc[r][3] = fmaf(pr, v0.w, acc[r][3]);
      acc[r][4] = fmaf(pr, v1.x, acc[r][4]);
      acc[r][5] = fmaf(pr, v1.y, acc[r][5]);
      acc[r][6] = fmaf(pr, v1.z, acc[r][6]);
      acc[r][7] = fmaf(pr, v1.w, acc[r][7]);
    }
  };
  // two keys per step (independent dots, one rescale vote): staged rows ra, rb
  auto visit2 = [&](int ra, bool va, int rb, bool vb) {
    const float sa = dot(sK + ra * kWinPitch + loff);
    const float sb = dot(sK + rb * kWinPitch + loff);
    float pa, pb;
    if (silu) {
      pa = va ? sa * __frcp_rn(1.0f + __expf(-sa)) * inv_n : 0.f;
      pb = vb ? sb * __frcp_rn(1.0f + __expf(-sb)) * inv_n : 0.f;
    } else {
      const float smax = fmaxf(va ? sa : -INFINITY, vb ? sb : -INFINITY);
      const bool need = smax > mthr;
      if (__any_sync(kAll, need)) {   // a new reference value in some row
        float corr = 1.f;
        if (need) {
          corr = ex2_approx(m - smax);   // 0 while m is -inf
          ssum *= corr;
          m = smax;
          mthr = smax + 8.0f;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float cr = __shfl_sync(kAll, corr, quad | r);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[r][k] *= cr;
        }
      }
      pa = va ? ex2_approx(sa - m) : 0.f;
      pb = vb ? ex2_approx(sb - m) : 0.f;
      ssum += pa + pb;
    }
    accumulate(sV + ra * kWinPitch + loff, pa);
    accumulate(sV + rb * kWinPitch + loff, pb);
  };
  // link keys, one pass per user owning rows of the block
  const int64_t u_lo = owner_of(off, B, r0), u_hi = owner_of(off, B, rlast);
  for (int64_t uu = u_lo; uu <= u_hi; ++uu) {
    if (off[uu + 1] <= off[uu]) continue;   // no history rows
    __syncthreads();
    win_stage(sK, sV, Kz, Vz, uu * L, L);
    if (!__any_sync(kAll, u == uu)) continue;
    const bool mine = u == uu;
#pragma unroll 1
    for (int k = 0; k < L; k += 2) {
      const bool second = k + 1 < L;
      visit2(k, mine, second ? k + 1 : k, mine && second);
    }
  }
  // window keys: rows [r0 - win, rlast + win] clipped to the history rows
  const int64_t lo = r0 - win > 0 ? r0 - win : 0;
  const int64_t hi = rlast + win < nh - 1 ? rlast + win : nh - 1;
  const int64_t wlo = w0 - win, whi = w0 + 7 + win;   // the warp's key range
  for (int64_t c0 = lo; c0 <= hi; c0 += kWinBuf) {
    const int n = (int)(hi - c0 + 1 < kWinBuf ? hi - c0 + 1 : kWinBuf);
    __syncthreads();
    win_stage(sK, sV, Ke, Ve, c0, n);
    // the lane's row's keys and the row itself, relative to c0 (clamped)
    auto rel = [&](int64_t x) { return (int)(x < c0 - 1 ? -1 : (x > c0 + kWinBuf ? kWinBuf : x - c0)); };
    const int klo = rel(j0), khi = rel(j1), kme = rel(i);
    const int a = (int)((wlo > c0 ? wlo : c0) - c0);
    const int b = (int)((whi < c0 + n - 1 ? whi : c0 + n - 1) - c0);
#pragma unroll 1
    for (int k = a; k <= b; k += 2) {
      const int k2 = k + 1 <= b ? k + 1 : k;
      visit2(k, klo <= k && k <= khi && k != kme, k2, k2 != k && klo <= k2 && k2 <= khi && k2 != kme);
    }
  }
  const float den = silu ? 1.0f : ssum;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float inv = 1.0f / __shfl_sync(kAll, den, quad | r);
    const int64_t ir = rg + r;
    if (ir < nh) {
      float4* dst = reinterpret_cast<float4*>(att + ir * kD + h * kDH + 8 * c);
      dst[0] = make_float4(acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv, acc[r][3] * inv);
      dst[1] = make_float4(acc[r][4] * inv, acc[r][5] * inv, acc[r][6] * inv, acc[r][7] * inv);
    }
  }
}

// ------------------------------------------------------- record pre-merge
// The link-branch records of a user's tiles (max, sum, 32 weighted sums per
// (tile, head, link)) are merged in runs of consecutive tiles: block b takes
// tiles [kRun b, kRun b + kRun) of the tile list, splits them at user
// boundaries and merges each run into the record slot of its first tile (in
// place, log-sum-exp, the tail's formula).  Runs therefore start at every
// user's first tile and at every multiple of kRun inside a user's tiles, and
// the link tail merges only those slots: a user with n tiles leaves it about
// n / kRun records, which keeps the tail's merge short for long histories.
// Thread (pair, q): the pair's max and sum and its weighted sums 8q .. 8q+7.
constexpr int kRun = 8;

template <int L>
__global__ void __launch_bounds__(kH * L * 4 < 512 ? kH * L * 4 : 512)
    k_rec_merge(uint8_t* __restrict__ ws, LayerWs Lw) {
  constexpr int HL = kH * L;
  pdl_launch();
  pdl_wait();
  const int n_tiles = *reinterpret_cast<const int*>(ws + Lw.sched);
  const int4* tiles = reinterpret_cast<const int4*>(ws + Lw.tiles);
  const int t0 = (int)blockIdx.x * kRun;
  if (t0 >= n_tiles) return;
  const int t1 = t0 + kRun < n_tiles ? t0 + kRun : n_tiles;
  const int q = threadIdx.x & 3;
  float* recs = reinterpret_cast<float*>(ws + Lw.part);
  // pairs in groups of blockDim / 4 (two groups for l = 64)
  for (int pr = threadIdx.x >> 2; pr < HL; pr += (int)blockDim.x >> 2) {
    int s0 = t0;
    while (s0 < t1) {
      const int u = tiles[s0].x;
      int e = s0 + 1;
      while (e < t1 && tiles[e].x == u) ++e;
      if (e - s0 > 1) {
        float2 ms[kRun];
        float4 a[kRun][2];
#pragma unroll
        for (int i = 0; i < kRun; ++i) {
          if (s0 + i < e) {
            const float4* rec = reinterpret_cast<const float4*>(recs + ((size_t)(s0 + i) * HL + pr) * kRec);
            ms[i] = *reinterpret_cast<const float2*>(rec);
            a[i][0] = rec[1 + 2 * q];
            a[i][1] = rec[2 + 2 * q];
          }
        }
        float M = -INFINITY, S = 0.f, acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
        for (int i = 0; i < kRun; ++i) {
          if (s0 + i < e) {
            const float Mn = fmaxf(M, ms[i].x);
            const float so = M == -INFINITY ? 0.f : __expf(M - Mn);
            const float sn = __expf(ms[i].x - Mn);
            S = S * so + ms[i].y * sn;
            acc[0] = acc[0] * so + a[i][0].x * sn;
            acc[1] = acc[1] * so + a[i][0].y * sn;
            acc[2] = acc[2] * so + a[i][0].z * sn;
            acc[3] = acc[3] * so + a[i][0].w * sn;
            acc[4] = acc[4] * so + a[i][1].x * sn;
            acc[5] = acc[5] * so + a[i][1].y * sn;
            acc[6] = acc[6] * so + a[i][1].z * sn;
            acc[7] = acc[7] * so + a[i][1].w * sn;
            M = Mn;
          }
        }
        __syncwarp();   // the pair's four threads have read the run's first record
        float4* dst = reinterpret_cast<float4*>(recs + ((size_t)s0 * HL + pr) * kRec);
        if (q == 0) *reinterpret_cast<float2*>(dst) = make_float2(M, S);
        dst[1 + 2 * q] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[2 + 2 * q] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
      s0 = e;
    }
  }
}

// ------------------------------------------------------------- link tail
// Everything the link rows need after the attention records, in one kernel:
//   b    = merge over the user's tiles of the link-branch records (max, sum,
//          weighted V sum) — the softmax of link k (head h) over all of the
//          user's history, as a log-sum-exp merge;
//   Y_Z  = Z + b Wo;  h2 = LN2(Y_Z);  Z' = Y_Z + (SiLU(h2 W1) * (h2 W3)) W2.
// A cluster of four CTAs owns 128 link rows.  CTA r merges rows 32r..32r+31
// straight into its A operand (bf16 hi + lo) and pushes those rows to the
// other three CTAs with shared-to-shared bulk copies (distributed shared
// memory, completion on the receiver's mbarrier).  Every CTA then runs b Wo
// and LN2 (split precision, identical in all four) and GatedMLP hidden chunk r
// only (64 of the 256 hidden units), stages its fp32 partial product, and
// pushes rows 32q..32q+31 of it to CTA q; CTA r sums the four partials of its
// rows, adds Y_Z and writes Z'.  No atomics; the summation order is fixed.
// 512 threads: thread (row, part) owns columns part*32 .. part*32+31.
constexpr int kTailSmem = 1024 + 12 * kBlk + kLnBytes + 64;

template <int L>
__global__ void __launch_bounds__(512, 1)
    k_link_tail(const bf16* __restrict__ Z, int64_t nrows, const bf16* __restrict__ g2,
                const bf16* __restrict__ b2, const uint8_t* __restrict__ ws, LayerWs Lw,
                bf16* __restrict__ Z_out, unsigned* status) {
  constexpr int HL = kH * L;
  constexpr uint32_t kQuarter = 32 * 128;        // 32 rows of a [128 x 64] block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1k(smem_raw);
  uint8_t* sAh = sm;                 // A operand hi: b, then h2; later the fp32 partial
  uint8_t* sAl = sm + 2 * kBlk;      // A operand lo
  uint8_t* sHh = sm + 4 * kBlk;      // hid hi [128 x 64]
  uint8_t* sHl = sm + 5 * kBlk;      // hid lo
  uint8_t* sWo = sm + 6 * kBlk;      // Wo image
  uint8_t* sRecv = sm + 4 * kBlk;    // 4 x 16 KB partial rows received (over hid and Wo)
  uint8_t* sW = sm + 8 * kBlk;       // [W1c | W3c] image, W2c (chunk = cluster rank)
  float* sY = reinterpret_cast<float*>(sm + 11 * kBlk);   // Y_Z of this CTA's 32 rows
  float* red = reinterpret_cast<float*>(sm + 12 * kBlk);
  uint8_t* sP = sAh;                 // fp32 partial [128 x 128] over sAh, sAl
  const uint32_t cr = cluster_rank();
  Cta c;
  cta_setup(sm + 12 * kBlk + kLnBytes, 5, c);  // bar: 0 Wo, 1 mma, 2 chunk, 3 b rows, 4 partials
  ln_stage(red + 1024, g2, b2);
  uint32_t mph = 0;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&c.bar[0], 2 * kBlk);
    bulk_load(sWo, ws + Lw.img_o, 2 * kBlk, &c.bar[0]);
    mbar_arrive_expect_tx(&c.bar[2], 3 * kBlk);
    bulk_load(sW, ws + Lw.img_13 + cr * 2 * kBlk, 2 * kBlk, &c.bar[2]);
    bulk_load(sW + 2 * kBlk, ws + Lw.img_2 + cr * kBlk, kBlk, &c.bar[2]);
    mbar_arrive_expect_tx(&c.bar[3], 3 * 4 * kQuarter);   // the other CTAs' b rows
    mbar_arrive_expect_tx(&c.bar[4], 3 * 32 * 512);       // the other CTAs' partial rows
  }
  cluster_arrive();    // (1) this CTA's barriers are initialised and armed
  const int64_t t0 = (int64_t)blockIdx.x * kTile;
  const int warp = threadIdx.x >> 5;
  const int part = warp >> 2;
  const int r = (warp & 3) * 32 + (threadIdx.x & 31);
  const int c0 = part * 32;
  const int64_t R = t0 + r;
  const bool valid = R < nrows;
  uint4 zr[4];                                     // this thread's Z values, loaded early
#pragma unroll
  for (int q = 0; q < 4; ++q)
    zr[q] = valid ? reinterpret_cast<const uint4*>(Z + R * kD + c0)[q] : make_uint4(0, 0, 0, 0);
  // 1. merge rows 32cr..32cr+31: four threads per (row, head) pair, 8
  //    columns each; pair p = 32h + row, so a warp reads the records of eight
  //    consecutive links of one head (contiguous, float4-aligned)
  {
    const int pr = threadIdx.x >> 2, q = threadIdx.x & 3;
    const int h = pr >> 5, lr = pr & 31;
    const int64_t Rm = t0 + 32 * cr + lr;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    float S = 0.f;
    if (Rm < nrows) {
      const int64_t u = Rm / L;
      const int k = (int)(Rm - u * L);
      const int* ts = reinterpret_cast<const int*>(ws + Lw.tile_start);
      const float* recs = reinterpret_cast<const float*>(ws + Lw.part);
      float M = -INFINITY;
      const int ta_ = ts[u], tb_ = ts[u + 1];
      // the user's run records (k_rec_merge): at its first tile and at every
      // multiple of kRun after it
      for (int t = ta_; t < tb_;) {
        // the records of up to eight runs are loaded before any is merged
        int slot[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          slot[i] = t;
          if (t < tb_) t = (t / kRun + 1) * kRun;
        }
        float2 ms[8];
        float4 a[8][2];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (slot[i] < tb_) {
            const float4* rec =
                reinterpret_cast<const float4*>(recs + ((size_t)slot[i] * HL + h * L + k) * kRec);
            ms[i] = *reinterpret_cast<const float2*>(rec);
            a[i][0] = rec[1 + 2 * q];
            a[i][1] = rec[2 + 2 * q];
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (slot[i] < tb_) {
            const float Mn = fmaxf(M, ms[i].x);
            const float so = M == -INFINITY ? 0.f : __expf(M - Mn);
            const float sn = __expf(ms[i].x - Mn);
            S = S * so + ms[i].y * sn;
            acc[0] = acc[0] * so + a[i][0].x * sn;
            acc[1] = acc[1] * so + a[i][0].y * sn;
            acc[2] = acc[2] * so + a[i][0].z * sn;
            acc[3] = acc[3] * so + a[i][0].w * sn;
            acc[4] = acc[4] * so + a[i][1].x * sn;
            acc[5] = acc[5] * so + a[i][1].y * sn;
            acc[6] = acc[6] * so + a[i][1].z * sn;
            acc[7] = acc[7] * so + a[i][1].w * sn;
            M = Mn;
          }
        }
      }
    }
    const float inv = S > 0.f ? 1.0f / S : 0.f;
    float h8[8], l8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float x = acc[j] * inv;
      h8[j] = __bfloat162float(__float2bfloat16_rn(x));
      l8[j] = x - h8[j];
    }
    sw_st16(sAh, kBlk, 32 * cr + lr, h * kDH + q * 8, pack8(h8));
    sw_st16(sAl, kBlk, 32 * cr + lr, h * kDH + q * 8, pack8(l8));
  }
  fence_proxy_async_smem();
  __syncthreads();     // this CTA's b rows are written
  cluster_wait();      // (1) every CTA's barriers are armed
  if (threadIdx.x == 0) {
    // rows 32cr..32cr+31 of the four 64-column blocks (hi 0, hi 1, lo 0, lo 1)
    // are 4 KB each and contiguous in the swizzled layout
    for (uint32_t p = 0; p < 4; ++p) {
      if (p == cr) continue;
      const uint32_t mb = cluster_map(&c.bar[3], p);
      for (int blk = 0; blk < 4; ++blk) {
        uint8_t* src = sAh + blk * kBlk + cr * kQuarter;
        bulk_push_cluster(cluster_map(src, p), src, kQuarter, mb);
      }
    }
  }
  mbar_wait(&c.bar[3], 0, status, c.abort_flag);
  cluster_arrive();    // (2) this CTA has received every row it was sent
  mbar_wait(&c.bar[0], 0, status, c.abort_flag);
  if (threadIdx.x == 0) {
    tc_fence_after();
    mma_tile(c.tmem, smem_u32(sAh), kBlk, smem_u32(sWo), kBlk, 128, 128, false);
    mma_tile(c.tmem, smem_u32(sAl), kBlk, smem_u32(sWo), kBlk, 128, 128, true);
    mma_commit(&c.bar[1]);
  }
  mbar_wait(&c.bar[1], mph, status, c.abort_flag);
  mph ^= 1u;
  tc_fence_after();
  const uint32_t ta = quad_addr(c);
  const bool mine = (uint32_t)(r >> 5) == cr;   // this CTA finishes row r
  // 2. Y_Z = Z + b Wo; LN2 -> A operand (hi + lo)
  {
    float y[32];
    tmem_ld16(ta + c0, y);
    tmem_ld16(ta + c0 + 16, y + 16);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float z8[8];
      unpack8(zr[q], z8);
#pragma unroll
      for (int k = 0; k < 8; ++k) y[q * 8 + k] += z8[k];
    }
    if (mine) {
      float4* dst = reinterpret_cast<float4*>(sY + (r & 31) * kD + c0);
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
    }
    layer_norm_part(y, c0, red, part, r);
    // (2) every CTA has received its rows, so no copy still reads our b rows
    cluster_wait();
    split_part_st(sAh, sAl, r, c0, y);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  mbar_wait(&c.bar[2], 0, status, c.abort_flag);
  if (threadIdx.x == 0) {
    tc_fence_after();
    // [G1 | G3] of hidden chunk cr in one N = 128 product
    mma_tile(c.tmem + 128, smem_u32(sAh), kBlk, smem_u32(sW), kBlk, 128, 128, false);
    mma_tile(c.tmem + 128, smem_u32(sAl), kBlk, smem_u32(sW), kBlk, 128, 128, true);
  }
  cta_mma_wait(&c.bar[1], mph, status, c.abort_flag);
  {
    float g[16], gg[16];
    tmem_ld16(ta + 128 + part * 16, g);
    tmem_ld16(ta + 192 + part * 16, gg);
    tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < 16; ++k) g[k] = silu_fast(g[k]) * gg[k];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float h8[8], l8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        h8[k] = __bfloat162float(__float2bfloat16_rn(g[q * 8 + k]));
        l8[k] = g[q * 8 + k] - h8[k];
      }
      sw_st16(sHh, kBlk, r, part * 16 + q * 8, pack8(h8));
      sw_st16(sHl, kBlk, r, part * 16 + q * 8, pack8(l8));
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_fence_after();
    mma_tile(c.tmem + 256, smem_u32(sHh), kBlk, smem_u32(sW + 2 * kBlk), kBlk, 128, 64, false);
    mma_tile(c.tmem + 256, smem_u32(sHl), kBlk, smem_u32(sW + 2 * kBlk), kBlk, 128, 64, true);
  }
  cta_mma_wait(&c.bar[1], mph, status, c.abort_flag);
  cluster_arrive();    // (3) this CTA's hid and Wo buffers are free to receive
  // 3. this chunk's fp32 partial -> shared memory (the A operand is dead);
  //    rows 32q..32q+31 form one contiguous 16 KB piece
  {
    float o[32];
    tmem_ld16(ta + 256 + c0, o);
    tmem_ld16(ta + 256 + c0 + 16, o + 16);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *f32_chunk(sP, r, part * 8 + q) = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
  }
  fence_proxy_async_smem();
  __syncthreads();     // this CTA's partial rows are written
  cluster_wait();      // (3) every CTA's hid and Wo buffers are free to receive
  if (threadIdx.x == 0) {
    for (uint32_t p = 0; p < 4; ++p) {
      if (p == cr) continue;
      uint8_t* src = sP + p * 32 * 512;
      bulk_push_cluster(cluster_map(sRecv + cr * 32 * 512, p), src, 32 * 512,
                        cluster_map(&c.bar[4], p));
    }
  }
  mbar_wait(&c.bar[4], 0, status, c.abort_flag);
  cluster_arrive();    // (4) this CTA has received every partial it was sent
  // 4. rows 32cr..32cr+31: Z' = Y_Z + the four partials (rank order)
  {
    const int lr = threadIdx.x >> 4, cc = threadIdx.x & 15;   // 8 columns each
    const int64_t Rr = t0 + 32 * cr + lr;
    float v[8];
    {
      const float4* y = reinterpret_cast<const float4*>(sY + lr * kD + cc * 8);
      const float4 a = y[0], b = y[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
#pragma unroll
    for (uint32_t p = 0; p < 4; ++p) {
      uint8_t* base = p == cr ? sP + cr * 32 * 512 : sRecv + p * 32 * 512;
      const float4 a = *f32_chunk(base, lr, cc * 2);
      const float4 b = *f32_chunk(base, lr, cc * 2 + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    if (Rr < nrows) reinterpret_cast<uint4*>(Z_out + Rr * kD)[cc] = pack8(v);
  }
  cluster_wait();   // (4) every CTA has received its partials: no copy still reads ours
  cta_teardown(c);
}

constexpr int kBarBytes = 64;

template <class K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

// A library-owned side stream (the device's highest priority) and two events
// per device, for running the link tail beside the history GatedMLP: both
// depend only on the attention kernel.  Created on the first call on the
// device that is not being captured into a graph (creating them during a
// capture could invalidate it); until then, and if creation fails, the layer
// runs its kernels in order on the caller's stream.  The mutex makes each
// fork (record, wait, launch, record, wait) atomic across host threads that
// share a device.
struct SideStream {
  bool tried = false;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
SideStream g_side[kMaxDevices];
std::mutex g_side_mu;

SideStream* side_stream(cudaStream_t st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  SideStream& r = g_side[dev];
  if (!r.tried) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
      return nullptr;
    r.tried = true;
    int least = 0, greatest = 0;
    bool ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
              cudaStreamCreateWithPriority(&r.s, cudaStreamNonBlocking, greatest) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      if (r.fork) cudaEventDestroy(r.fork);
      if (r.s) cudaStreamDestroy(r.s);
      r.s = nullptr;
      r.fork = r.join = nullptr;
      cudaGetLastError();
    }
  }
  return r.s ? &r : nullptr;
}

template <int L>
int run_layer(const lime_dims& D, int64_t B, const int64_t* off, int64_t nh, const void* E_in,
              const void* Z_in, const lime_layer_w& w, void* E_out, void* Z_out, uint8_t* ws,
              unsigned* status, cudaStream_t st) {
  const LayerWs Lw = layer_ws(L, B, nh, D.phi == LIME_PHI_SILU, D.window);
  const bool last = E_out == nullptr;
  // a window layer's history branch runs on its own kernels (after the link
  // branch); its link projections are those of a last layer (Q'g only)
  const bool window = D.window > 0 && !last;
  const bool link_only = last || window;
  const float scale = 1.0f / sqrtf((float)kDH);
  const int64_t nz = B * L;
  const int sms = num_sms();
  {
    const int64_t n = (5 * kD * kD + 3 * kD * kF) / 8;
    int rc = launch_pdl(k_prep_weights, dim3((unsigned)(2 + (n + 1023) / 1024)), dim3(1024), 0, st,
                        1, (const bf16*)w.Wq, (const bf16*)w.Wk, (const bf16*)w.Wv,
                        (const bf16*)w.Wo, (const bf16*)w.W1, (const bf16*)w.W3, (const bf16*)w.W2,
                        (const bf16*)w.g1, (const bf16*)w.b1, ws, Lw, off, B, nh, status);
    if (rc) return rc;
  }
  {
    // the last layer needs only Q' (its history branch is skipped)
    const int smem = 1024 + 8 * kBlk + kLnBytes + kBarBytes;
    if (!set_smem(k_link_proj<L>, smem)) return LIME_ERR_CUDA;
    int rc = launch_pdl(k_link_proj<L>, dim3((unsigned)((nz + kTile - 1) / kTile), link_only ? 1 : 3,
                                             link_only ? 4 : 2),
                        dim3(512), smem, st, 1, (const bf16*)Z_in, nz, (const bf16*)w.g1,
                        (const bf16*)w.b1, ws, Lw, scale, D.phi == LIME_PHI_SILU, status);
    if (rc) return rc;
  }
  CUtensorMap tmE_ffn{};
  if (nh > 0) {
    CUtensorMap tmE, tmY;
    if (!make_tmap_2d_bf16(&tmE, E_in, kD, (uint64_t)nh, kD * 2, 64, kTile) ||
        !make_tmap_2d_f16(&tmY, ws + Lw.yd, kD, (uint64_t)nh, kD * 2, 64, 32))   // a quadrant's rows
      return LIME_ERR_CUDA;
    tmE_ffn = tmE;
    const int64_t tiles_hi = Lw.max_tiles;
    const int grid = (int)(tiles_hi < sms ? tiles_hi : sms);
    {
      const bool silu = D.phi == LIME_PHI_SILU;
      auto kern = link_only ? (silu ? k_hist_xattn<L, false, true> : k_hist_xattn<L, false, false>)
                            : (silu ? k_hist_xattn<L, true, true> : k_hist_xattn<L, true, false>);
      if (!set_smem(kern, kXaSmem)) return LIME_ERR_CUDA;
      int rc = launch_pdl(kern, dim3(grid), dim3(kXaThreads), kXaSmem, st, 1, tmE, tmY, ws, Lw,
                          status);
      if (rc) return rc;
    }
    if (window) {
      const bool silu = D.phi == LIME_PHI_SILU;
      const bf16* g1 = (const bf16*)w.g1;
      const bf16* b1 = (const bf16*)w.b1;
      // LN1 and Q, K, V of the history rows; K, V of the link rows (fp32)
      constexpr int smem3 = 1024 + 12 * kBlk + kLnBytes + kBarBytes;
      constexpr int smem1 = 1024 + 10 * kBlk + kLnBytes + kBarBytes;
      auto kq = k_rows_proj<3, true, false, false>;
      auto ko = k_rows_proj<1, false, true, true>;
      if (!set_smem(kq, smem3) || !set_smem(ko, smem1)) return LIME_ERR_CUDA;
      auto f32map = [](CUtensorMap* m, void* base, int64_t rows) {
        return make_tmap_2d_f32(m, base, kD, (uint64_t)rows, kD * 4, 32, kTile);
      };
      auto pgrid = [&](int64_t tiles) { return dim3((unsigned)(tiles < sms ? tiles : sms)); };
      const int64_t th = (nh + kTile - 1) / kTile, tz = (nz + kTile - 1) / kTile;
      RowsMaps m3{};
      m3.x[0] = tmE;
      if (!make_tmap_2d_bf16(&m3.x[1], Z_in, kD, (uint64_t)nz, kD * 2, 64, kTile) ||
          !f32map(&m3.o[0], ws + Lw.qe, nh) || !f32map(&m3.o[1], ws + Lw.ke, nh) ||
          !f32map(&m3.o[2], ws + Lw.ve, nh) || !f32map(&m3.o[3], ws + Lw.kz, nz) ||
          !f32map(&m3.o[4], ws + Lw.vz, nz))
        return LIME_ERR_CUDA;
      const RowsImgs i3{{(uint32_t)Lw.img_q, (uint32_t)Lw.img_k, (uint32_t)Lw.img_v}};
      int rc = launch_pdl(kq, pgrid(th + tz), dim3(512), smem3, st, 1, m3, nh, nz, g1, b1,
                          (const uint8_t*)ws, i3, status);
      if (rc) return rc;
      if (!set_smem(k_win_attn, kWinSmem)) return LIME_ERR_CUDA;
      rc = launch_pdl(k_win_attn, dim3((unsigned)((nh + kWinRows - 1) / kWinRows)), dim3(256),
                      kWinSmem, st, 1,
                      (const float*)(ws + Lw.qe), (const float*)(ws + Lw.ke),
                      (const float*)(ws + Lw.ve), (const float*)(ws + Lw.kz),
                      (const float*)(ws + Lw.vz), off, B, nh, L, D.window, scale, silu ? 1 : 0,
                      (float*)(ws + Lw.att));
      if (rc) return rc;
      // Yd = A Wo (fp16), the attention delta the GatedMLP kernel adds to E
      RowsMaps m1{};
      if (!f32map(&m1.x[0], ws + Lw.att, nh) ||
          !make_tmap_2d_f16(&m1.o[0], ws + Lw.yd, kD, (uint64_t)nh, kD * 2, 64, kTile))
        return LIME_ERR_CUDA;
      const RowsImgs i1{{(uint32_t)Lw.img_o, 0u, 0u}};
      rc = launch_pdl(ko, pgrid(th), dim3(512), smem1, st, 1, m1, nh, (int64_t)0, g1, b1,
                      (const uint8_t*)ws, i1, status);
      if (rc) return rc;
    }
  }
  // one 4-CTA cluster per 128 link rows
  if (!set_smem(k_link_tail<L>, kTailSmem)) return LIME_ERR_CUDA;
  auto tail = [&](cudaStream_t s) {
    if (nh > 0) {
      int rc = launch_pdl(k_rec_merge<L>, dim3((unsigned)((Lw.max_tiles + kRun - 1) / kRun)),
                          dim3(kH * L * 4 < 512 ? kH * L * 4 : 512), 0, s, 1, ws, Lw);
      if (rc) return rc;
    }
    return launch_pdl(k_link_tail<L>, dim3((unsigned)((nz + kTile - 1) / kTile), kF / 64),
                      dim3(512), kTailSmem, s, kF / 64, (const bf16*)Z_in, nz,
                      (const bf16*)w.g2, (const bf16*)w.b2, (const uint8_t*)ws, Lw, (bf16*)Z_out,
                      status);
  };
  if (last || nh == 0) return tail(st);
  // the history GatedMLP and the link tail both read only what the attention
  // kernel left: the tail runs on the high-priority side stream, so its 4-CTA
  // clusters take SMs as the attention kernel's CTAs retire and the GatedMLP's
  // persistent CTAs fill the rest
  if (!set_smem(k_hist_ffn, kFfnSmem)) return LIME_ERR_CUDA;
  const int64_t tiles_hi = Lw.max_tiles;
  const int grid = (int)(tiles_hi < sms ? tiles_hi : sms);
  auto ffn = [&]() {
    return launch_pdl(k_hist_ffn, dim3(grid), dim3(kFfnEpi + 96), kFfnSmem, st, 1, tmE_ffn,
                      (const bf16*)w.g2, (const bf16*)w.b2, (const uint8_t*)ws, Lw,
                      (bf16*)E_out, status);
  };
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* side = side_stream(st);
  if (!side) {
    int rc = ffn();
    return rc ? rc : tail(st);
  }
  if (cudaEventRecord(side->fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
    return LIME_ERR_CUDA;
  int rc = tail(side->s);
  if (rc) return rc;
  rc = ffn();
  if (rc) return rc;
  if (cudaEventRecord(side->join, side->s) != cudaSuccess ||
      cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess)
    return LIME_ERR_CUDA;
  return LIME_OK;
}

}  // namespace

bool fast_layer_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && D.f == kF &&
         (D.l == 16 || D.l == 32 || D.l == 64);
}

size_t fast_layer_ws_bytes(const lime_dims& D, int64_t B, int64_t total_hist) {
  if (!fast_layer_supported(D)) return 0;
  return layer_ws(D.l, B, total_hist, D.phi == LIME_PHI_SILU, D.window).total;
}

int fast_xor_layer(const lime_dims& D, int64_t B, const int64_t* off, int64_t nh,
                   const void* E_in, const void* Z_in, const lime_layer_w& w, void* E_out,
                   void* Z_out, float* ws, unsigned* status, cudaStream_t st) {
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  if (D.l == 16) return run_layer<16>(D, B, off, nh, E_in, Z_in, w, E_out, Z_out, wsb, status, st);
  if (D.l == 64) return run_layer<64>(D, B, off, nh, E_in, Z_in, w, E_out, Z_out, wsb, status, st);
  return run_layer<32>(D, B, off, nh, E_in, Z_in, w, E_out, Z_out, wsb, status, st);
}

}  // namespace lime
