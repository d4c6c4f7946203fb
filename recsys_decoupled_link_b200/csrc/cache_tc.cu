// QK-cache build on the 5th-generation tensor cores (bf16, d = 128).
//
// LIME note, 关键设计 1: the candidate-side weights phi(T L^T) depend only on
// the item embedding and the global links, so they are computed offline for
// the whole catalogue.  With per-head scaled-softmax attention,
//     cache[m, h, :] = softmax_k( T_m · G[:, h*l + k] ),
//     G[:, h*l + k]  = s * Wq_c[:, h-cols] (L_k Wk_c[:, h-cols])^T,
// so the build is one catalogue x (H*l) GEMM with a softmax epilogue.
//
// k_fold_g_img folds G (d x H*l, fp32 then bf16) and writes it pre-swizzled in
// the K-major 128-byte-swizzle image the MMA reads, so each CTA loads it with
// one bulk copy.  k_cache_tc is persistent (one CTA per SM):
//   warp 0     TMA producer: 128-row tiles of T into a STAGES-deep ring
//   warp 1     tcgen05.mma issuer (M=128, N=H*l, K=128 as 8 K-steps) into one
//              of two TMEM accumulators
//   warps 2-   epilogue, up to four warps per TMEM lane quadrant, each taking
//              a share of the heads: tcgen05.ld of its row, softmax per head over l links
//              in fp32, bf16 into a 128-byte-swizzled staging tile, TMA store
//              of the tile (rows past n_items are clipped by TMA)
// Every wait is bounded; a timeout sets LIME_FLAG_TIMEOUT and the CTA drains
// and returns.  The catalogue read is the roofline: 2*(d + H*l) bytes/item.
#include "lime_fast.cuh"
#include "sm100.cuh"

namespace lime {

using namespace sm100;

namespace {

constexpr int kD = 128;    // model dim handled here
constexpr int kBM = 128;   // catalogue rows per tile

// U8: the cache is stored as bytes q = round(255 w) (an int8 cache).
template <int HL, int L, bool U8>
struct CacheCfg {
  static constexpr int STAGES = HL <= 128 ? 4 : 3;
  static constexpr int OUTB = HL <= 128 || U8 ? 2 : 1;
  static constexpr int A_BYTES = kBM * kD * 2;      // one T tile
  static constexpr int B_BYTES = HL * kD * 2;       // the G^T image
  static constexpr int ROW_BYTES = HL * (U8 ? 1 : 2);   // one cache row
  static constexpr int O_BYTES = kBM * ROW_BYTES;   // one output tile
  static constexpr int TMEM_COLS = 2 * HL;
  static constexpr int OFF_B = STAGES * A_BYTES;
  static constexpr int OFF_O = OFF_B + B_BYTES;
  static constexpr int OFF_BAR = OFF_O + OUTB * O_BYTES;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  // epilogue warps per TMEM lane quadrant: one head each for up to 4 heads
  // of l <= 32 links; two (half of the heads each) for l = 64, whose rows need
  // more registers than 18 warps leave per thread
  static constexpr int H_ = HL / L;
  static constexpr int WPQ = L >= 64 ? (H_ < 2 ? H_ : 2) : (H_ < 4 ? H_ : 4);
  static constexpr int EPI = 4 * WPQ * 32;          // epilogue threads
  static constexpr int THREADS = 64 + EPI;
};

// G^T image: block b (K columns [64b, 64b+64)) of HL rows x 128 bytes,
// element (row j = h*l + k, K index i) at b*HL*128 + sw128_offset(j, i % 64).
// CTA j = h*l + k stages L_k and the head-h columns of Wk_c and Wq_c in
// shared memory (all 16-byte loads issued before any is used), forms
// kc = L_k Wk_c[:, h-cols] (dh values; 128 threads, each a quarter of the
// K = 128 sum for one value when dh = 32) and writes row j of G^T.
__global__ void __launch_bounds__(128) k_fold_g_img(const bf16* __restrict__ L,
                                                    const bf16* __restrict__ Wq,
                                                    const bf16* __restrict__ Wk, int H, int l,
                                                    float scale, bf16* __restrict__ img) {
  __shared__ __align__(16) bf16 sWk[kD * 64];   // [kD][dh]
  __shared__ __align__(16) bf16 sWq[kD * 64];   // [kD][dh]
  __shared__ float sL[kD];
  __shared__ float part[8][64];   // dh >= 16: at most 8 partial sums
  __shared__ float kc[64];
  const int dh = kD / H, HL = H * l;
  const int j = blockIdx.x, h = j / l, k = j % l;
  pdl_launch();
  pdl_wait();
  {
    const int cw = dh / 8;                 // 16-byte chunks per head row (2, 4 or 8)
    const int nK = kD * cw;                // <= 1024 chunks for each of Wk, Wq
    uint4 vk[8], vq[8], vl;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = q * 128 + (int)threadIdx.x;
      if (e < nK) {
        vk[q] = reinterpret_cast<const uint4*>(Wk + (e / cw) * kD + h * dh)[e % cw];
        vq[q] = reinterpret_cast<const uint4*>(Wq + (e / cw) * kD + h * dh)[e % cw];
      }
    }
    if (threadIdx.x < 16) vl = reinterpret_cast<const uint4*>(L + (int64_t)k * kD)[threadIdx.x];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = q * 128 + (int)threadIdx.x;
      if (e < nK) {
        reinterpret_cast<uint4*>(sWk)[e] = vk[q];
        reinterpret_cast<uint4*>(sWq)[e] = vq[q];
      }
    }
    if (threadIdx.x < 16) unpack8(vl, sL + threadIdx.x * 8);
  }
  __syncthreads();
  {
    // kc[c] = sum_t L_k[t] Wk[t, h*dh + c]: thread (c, quarter of t)
    const int nq = 128 / dh, c = threadIdx.x % dh, q = threadIdx.x / dh;
    float acc = 0.f;
    for (int t = q; t < kD; t += nq) acc += sL[t] * __bfloat162float(sWk[t * dh + c]);
    part[q][c] = acc;
  }
  __syncthreads();
  if (threadIdx.x < dh) {
    float s = 0.f;
    for (int q = 0; q < 128 / dh; ++q) s += part[q][threadIdx.x];
    kc[threadIdx.x] = s;
  }
  __syncthreads();
  {
    const int i = threadIdx.x;   // K index of G^T row j
    float acc = 0.f;
    for (int c = 0; c < dh; ++c) acc += __bfloat162float(sWq[i * dh + c]) * kc[c];
    uint8_t* base = reinterpret_cast<uint8_t*>(img) + (size_t)(i >> 6) * HL * 128;
    *reinterpret_cast<bf16*>(base + sw128_offset(j, i & 63)) = __float2bfloat16_rn(acc * scale);
  }
}

template <int HL, int L, bool U8, bool SILU>
__global__ void __launch_bounds__(CacheCfg<HL, L, U8>::THREADS, 1)
    k_cache_tc(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmC,
               const bf16* __restrict__ gimg, int n_tiles, unsigned* status) {
  using C = CacheCfg<HL, L, U8>;
  constexpr int H = HL / L;
  constexpr uint32_t IDESC = idesc_bf16(kBM, HL);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sO = smem + C::OFF_O;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* ofull = tempty + 2;
  uint64_t* ofree = ofull + 2;
  uint64_t* bready = ofree + 2;
  uint64_t* mdone = bready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::EPI);
      mbar_init(&ofull[a], C::EPI);
      mbar_init(&ofree[a], 1);
    }
    mbar_init(bready, 1);
    mbar_init(mdone, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmT);
      prefetch_tmap(&tmC);
      mbar_arrive_expect_tx(bready, C::B_BYTES);
      bulk_load(sB, gimg, C::B_BYTES, bready);
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, status, &abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], C::A_BYTES);
        uint8_t* dst = sA + s * C::A_BYTES;
        tma_load_2d(dst, &tmT, 0, tile * kBM, &full[s]);
        tma_load_2d(dst + C::A_BYTES / 2, &tmT, 64, tile * kBM, &full[s]);
      }
      // drain: every issued load has landed before the CTA may exit
      const int issued = it;
      for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; ++j)
        mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1, status, &abort_flag);
      mbar_wait(bready, 0, status, &abort_flag);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (mbar_wait(bready, 0, status, &abort_flag)) {
        const uint32_t bBase = smem_u32(sB);
        int it = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          const int acc = it & 1;
          const uint32_t aph = (it >> 1) & 1;
          if (!mbar_wait(&tempty[acc], aph ^ 1, status, &abort_flag)) break;
          if (!mbar_wait(&full[s], ph, status, &abort_flag)) break;
          tc_fence_after();
          const uint32_t aBase = smem_u32(sA + s * C::A_BYTES);
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) {
            const uint32_t koff = (k & 3) * 32;
            const uint64_t ad = sdesc_sw128(aBase + (k >> 2) * (C::A_BYTES / 2) + koff);
            const uint64_t bd = sdesc_sw128(bBase + (k >> 2) * (C::B_BYTES / 2) + koff);
            mma_bf16(tmem + acc * HL, ad, bd, IDESC, k > 0);
          }
          mma_commit(&empty[s]);
          mma_commit(&tfull[acc]);
        }
      }
      mma_commit(mdone);
      mbar_wait(mdone, 0, status, &abort_flag);
    }
  } else {
    // epilogue: WPQ warps per TMEM lane quadrant; the warp's lane is tile row
    // `row` and it handles heads grp*HPW .. (group grp = (warp - 2) / 4)
    const int et = threadIdx.x - 64;
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;                // 0 .. WPQ-1
    constexpr int HPW = H / C::WPQ < 1 ? 1 : H / C::WPQ;   // heads per epilogue warp
    const int row = quad * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    // softmax (or SiLU) of head h of this thread's row, into the staging tile
    auto emit_head = [&](int h, uint32_t acc, uint8_t* stage) {
      float z[L];
#pragma unroll
      for (int q = 0; q < L / 16; ++q)
        tmem_ld16(tmem + lane_base + acc * HL + h * L + q * 16, z + q * 16);
      tmem_ld_wait();
      float inv;
      if constexpr (SILU) {
        // SiLU of each score over the l links (the int8 cache is softmax only)
#pragma unroll
        for (int k = 0; k < L; ++k) z[k] = __fdividef(z[k], 1.0f + __expf(-z[k]));
        inv = 1.0f / L;
      } else {
        float m = z[0];
#pragma unroll
        for (int k = 1; k < L; ++k) m = fmaxf(m, z[k]);
        float ssum = 0.f;
#pragma unroll
        for (int k = 0; k < L; ++k) {
          z[k] = __expf(z[k] - m);
          ssum += z[k];
        }
        inv = 1.0f / ssum;
      }
      if constexpr (U8) {
        // bytes q = round(255 w), ties to even; 16 per 16-byte chunk of the
        // row's 128-byte swizzled block
        const float sc = inv * 255.0f;
#pragma unroll
        for (int c = 0; c < L / 16; ++c) {
          const int bcol = h * L + c * 16;
          // z <= 1 and sum >= 1, so 255 z / sum rounds to at most 255.  Adding
          // 1.5 * 2^23 in the same FMA rounds the product to an integer (ties
          // to even) in the low mantissa bits: the low byte is q.
          uint32_t wv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float* zz = z + c * 16 + j * 4;
            const uint32_t q0 = __float_as_uint(fmaf(zz[0], sc, 12582912.0f));
            const uint32_t q1 = __float_as_uint(fmaf(zz[1], sc, 12582912.0f));
            const uint32_t q2 = __float_as_uint(fmaf(zz[2], sc, 12582912.0f));
            const uint32_t q3 = __float_as_uint(fmaf(zz[3], sc, 12582912.0f));
            wv[j] = __byte_perm(__byte_perm(q0, q1, 0x0040), __byte_perm(q2, q3, 0x0040), 0x5410);
          }
          // 64-byte rows (H*l = 64) are staged row-major without swizzle;
          // 128-byte boxes of wider rows in the 128-byte swizzle
          uint8_t* dst = HL == 64 ? stage + row * 64 + (bcol >> 4) * 16
                                  : stage + (bcol >> 7) * (kBM * 128) + row * 128 +
                                        ((((bcol & 127) >> 4) ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < L / 8; ++c) {
          const int col = h * L + c * 8;
          uint4 v;
          v.x = pack_bf16(z[c * 8 + 0] * inv, z[c * 8 + 1] * inv);
          v.y = pack_bf16(z[c * 8 + 2] * inv, z[c * 8 + 3] * inv);
          v.z = pack_bf16(z[c * 8 + 4] * inv, z[c * 8 + 5] * inv);
          v.w = pack_bf16(z[c * 8 + 6] * inv, z[c * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(stage + (col >> 6) * (kBM * 128) + sw128_offset(row, col & 63)) = v;
        }
      }
    };
    // HL = 256 with bf16 weights leaves room for one 64 KB staging tile only;
    // it is written and stored in two halves (the first half of the heads,
    // then the second), so that one half's TMA store overlaps the other
    // half's softmax instead of draining before the next tile may start.
    constexpr bool SPLIT = C::OUTB == 1;
    static_assert(!SPLIT || (HPW == 2 && C::WPQ * L == HL / 2), "two passes of one head each");
    // 128-byte-wide boxes: 64 bf16 or 128 bytes (one 64-byte box for H*l = 64 bytes)
    constexpr int per_box = U8 ? (HL == 64 ? 64 : 128) : 64;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if constexpr (SPLIT) {
        // ofull[p] / ofree[p]: half p of the staging tile written / its store
        // has read it (each completes once per tile)
        const uint32_t prev = (uint32_t)(it - 1) & 1u;
        if (it > 0 && !mbar_wait(&ofree[0], prev, status, &abort_flag)) break;
        if (!mbar_wait(&tfull[acc], aph, status, &abort_flag)) break;
        tc_fence_after();
        emit_head(grp, acc, sO);
        fence_proxy_async_smem();
        mbar_arrive(&ofull[0]);
        if (et == 0) {
          if (!mbar_wait(&ofull[0], (uint32_t)it & 1u, status, &abort_flag)) break;
#pragma unroll
          for (int b = 0; b < HL / per_box / 2; ++b)
            tma_store_2d(&tmC, sO + b * (kBM * 128), b * per_box, tile * kBM);
          bulk_commit();
          if (it > 0) {
            bulk_wait_read<1>();   // the previous tile's second half has been read
            mbar_arrive(&ofree[1]);
          }
        }
        if (it > 0 && !mbar_wait(&ofree[1], prev, status, &abort_flag)) break;
        emit_head(grp + C::WPQ, acc, sO);
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        fence_proxy_async_smem();
        mbar_arrive(&ofull[1]);
        if (et == 0) {
          if (!mbar_wait(&ofull[1], (uint32_t)it & 1u, status, &abort_flag)) break;
#pragma unroll
          for (int b = HL / per_box / 2; b < HL / per_box; ++b)
            tma_store_2d(&tmC, sO + b * (kBM * 128), b * per_box, tile * kBM);
          bulk_commit();
          bulk_wait_read<1>();     // this tile's first half has been read
          mbar_arrive(&ofree[0]);
        }
        continue;
      }
      const int ob = C::OUTB == 2 ? (it & 1) : 0;
      const uint32_t oph = (it / C::OUTB) & 1;
      if (!mbar_wait(&ofree[ob], oph ^ 1, status, &abort_flag)) break;
      if (!mbar_wait(&tfull[acc], aph, status, &abort_flag)) break;
      tc_fence_after();
      uint8_t* stage = sO + ob * C::O_BYTES;
#pragma unroll 1
      for (int h = grp * HPW; h < (grp + 1) * HPW && h < H; ++h) emit_head(h, acc, stage);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      fence_proxy_async_smem();
      mbar_arrive(&ofull[ob]);
      if (et == 0) {
        if (!mbar_wait(&ofull[ob], oph, status, &abort_flag)) break;
#pragma unroll
        for (int b = 0; b < HL / per_box; ++b)
          tma_store_2d(&tmC, stage + b * (kBM * 128), b * per_box, tile * kBM);
        bulk_commit();
        // the store issued OUTB-1 tiles ago has finished reading its buffer
        bulk_wait_read<C::OUTB - 1>();
        if (C::OUTB == 2) {
          if (it >= 1) mbar_arrive(&ofree[ob ^ 1]);
        } else {
          mbar_arrive(&ofree[0]);
        }
      }
    }
    if (et == 0) bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int HL, int L, bool U8, bool SILU>
int launch_cache(const void* T, int64_t n, const bf16* img, void* cache, int tiles_per_cta,
                 unsigned* status, cudaStream_t st) {
  using C = CacheCfg<HL, L, U8>;
  CUtensorMap tmT, tmC;
  if (!make_tmap_2d_bf16(&tmT, T, kD, (uint64_t)n, kD * 2, 64, kBM)) return LIME_ERR_CUDA;
  if (U8 && HL == 64) {
    if (!make_tmap_2d_u8_plain(&tmC, cache, HL, (uint64_t)n, HL, 64, kBM)) return LIME_ERR_CUDA;
  } else if (U8) {
    if (!make_tmap_2d_u8(&tmC, cache, HL, (uint64_t)n, HL, 128, kBM)) return LIME_ERR_CUDA;
  } else if (!make_tmap_2d_bf16(&tmC, cache, HL, (uint64_t)n, HL * 2, 64, kBM)) {
    return LIME_ERR_CUDA;
  }
  if (cudaFuncSetAttribute(k_cache_tc<HL, L, U8, SILU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return LIME_ERR_CUDA;
  const int n_tiles = (int)((n + kBM - 1) / kBM);
  // persistent (one CTA per SM), or CTAs of about tiles_per_cta tiles each, so
  // that the build can share the GPU with higher-priority work
  int grid = n_tiles < num_sms() ? n_tiles : num_sms();
  if (tiles_per_cta > 0) grid = (n_tiles + tiles_per_cta - 1) / tiles_per_cta;
  return launch_pdl(k_cache_tc<HL, L, U8, SILU>, dim3(grid), dim3(C::THREADS), C::SMEM, st, 1, tmT, tmC,
                    img, n_tiles, status);
}

}  // namespace

size_t fast_cache_ws_bytes(const lime_dims& D) { return (size_t)D.H * D.l * D.d * 2; }

bool fast_cache_supported(const lime_dims& D) {
  if (D.dtype != LIME_BF16 || D.d != kD) return false;
  const int HL = D.H * D.l, dh = D.d / D.H;
  if (dh != 16 && dh != 32 && dh != 64) return false;
  if (D.l != 16 && D.l != 32 && D.l != 64) return false;
  return HL == 64 || HL == 128 || HL == 256;
}

bool fast_cache_u8_supported(const lime_dims& D) {
  // 64-byte rows only with 16 links (the byte epilogue's 16-weight chunks)
  return fast_cache_supported(D) && (D.H * D.l >= 128 || D.l == 16);
}

namespace {
int launch_fold(const lime_dims& D, const void* L, const void* Wq, const void* Wk, bf16* img,
                cudaStream_t st) {
  const float scale = 1.0f / sqrtf((float)(D.d / D.H));
  return launch_pdl(k_fold_g_img, dim3(D.H * D.l), dim3(128), 0, st, 1, (const bf16*)L,
                    (const bf16*)Wq, (const bf16*)Wk, D.H, D.l, scale, img);
}

int launch_build(const lime_dims& D, const void* T, int64_t n, const bf16* img, void* cache,
                 bool u8, int tpc, unsigned* status, cudaStream_t st) {
  if (n == 0) return LIME_OK;
  switch (D.H * D.l * 1000 + D.l + (u8 ? 1000000 : 0)) {
    case 64016: return (D.phi == LIME_PHI_SILU ? launch_cache<64, 16, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<64, 16, false, false>(T, n, img, cache, tpc, status, st));
    case 64032: return (D.phi == LIME_PHI_SILU ? launch_cache<64, 32, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<64, 32, false, false>(T, n, img, cache, tpc, status, st));
    case 128016: return (D.phi == LIME_PHI_SILU ? launch_cache<128, 16, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<128, 16, false, false>(T, n, img, cache, tpc, status, st));
    case 128032: return (D.phi == LIME_PHI_SILU ? launch_cache<128, 32, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<128, 32, false, false>(T, n, img, cache, tpc, status, st));
    case 128064: return (D.phi == LIME_PHI_SILU ? launch_cache<128, 64, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<128, 64, false, false>(T, n, img, cache, tpc, status, st));
    case 256032: return (D.phi == LIME_PHI_SILU ? launch_cache<256, 32, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<256, 32, false, false>(T, n, img, cache, tpc, status, st));
    case 256064: return (D.phi == LIME_PHI_SILU ? launch_cache<256, 64, false, true>(T, n, img, cache, tpc, status, st)
                                          : launch_cache<256, 64, false, false>(T, n, img, cache, tpc, status, st));
    case 1064016: return launch_cache<64, 16, true, false>(T, n, img, cache, tpc, status, st);
    case 1128016: return launch_cache<128, 16, true, false>(T, n, img, cache, tpc, status, st);
    case 1128032: return launch_cache<128, 32, true, false>(T, n, img, cache, tpc, status, st);
    case 1128064: return launch_cache<128, 64, true, false>(T, n, img, cache, tpc, status, st);
    case 1256032: return launch_cache<256, 32, true, false>(T, n, img, cache, tpc, status, st);
    case 1256064: return launch_cache<256, 64, true, false>(T, n, img, cache, tpc, status, st);
    default: return LIME_ERR_SHAPE;
  }
}
}  // namespace

int fast_build_qk_cache(const lime_dims& D, const void* T, int64_t n, const void* L,
                        const void* Wq, const void* Wk, void* cache, float* ws,
                        unsigned* status, cudaStream_t st) {
  bf16* img = reinterpret_cast<bf16*>(ws);
  int rc = launch_fold(D, L, Wq, Wk, img, st);
  return rc ? rc : launch_build(D, T, n, img, cache, false, 0, status, st);
}

int fast_build_qk_cache_u8(const lime_dims& D, const void* T, int64_t n, const void* L,
                           const void* Wq, const void* Wk, void* cache, float* ws,
                           unsigned* status, cudaStream_t st) {
  bf16* img = reinterpret_cast<bf16*>(ws);
  int rc = launch_fold(D, L, Wq, Wk, img, st);
  return rc ? rc : launch_build(D, T, n, img, cache, true, 0, status, st);
}

int fast_fold_qk(const lime_dims& D, const void* L, const void* Wq, const void* Wk, void* image,
                 cudaStream_t st) {
  return launch_fold(D, L, Wq, Wk, reinterpret_cast<bf16*>(image), st);
}

int fast_build_qk_cache_folded(const lime_dims& D, const void* T, int64_t n, const void* image,
                               void* cache, int tiles_per_cta, unsigned* status, cudaStream_t st) {
  return launch_build(D, T, n, reinterpret_cast<const bf16*>(image), cache, false, tiles_per_cta,
                      status, st);
}

}  // namespace lime
