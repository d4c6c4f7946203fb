// Uncached (online) candidate scoring on the 5th-generation tensor cores
// (bf16, d = 128, 4 heads of 32, l in {16, 32}).
//
// LIME note, 关键设计 1: O_m = MHA(T_m, L, L^P), whose weights phi(T_m L^T)
// depend only on the item and the global links.  Cached scoring reads them
// per candidate; LIME listing Table 10 ("uncached global") and the cold-start
// fallback for items missing from the cache compute them online instead.
// Per 128 candidates of one user:
//   gather   the item rows T[id_m] (256 bytes each) with cp.async straight into
//            the K-major 128B-swizzled A operand, a tile ahead (two stages)
//   MMA 1    S = T_m G ([128 x H*l], TMEM [0, H*l)), G = the folded
//            s Wq_c,h (L Wk_c,h)^T of lime_fold_qk (its image, one bulk copy)
//   softmax  per head over l in fp32 (thread = candidate row); the bf16
//            weights overwrite the gathered rows (MMA 1 is done with them)
//   MMA 2    per head [128 x l] x [l x 32] against L^P_u^T, as in cached
//            scoring (TMEM [128, 256))
//   out      O rows in bf16 through the same stage, coalesced 16-byte stores.
// CTA (u, g) walks tiles g, g + G, ... of user u's candidates; 128 threads.
// An out-of-range ID gives a zero row of T (so uniform weights) and
// LIME_FLAG_BAD_ID; its O row is written as zero.  No workspace is used.
#include "lime_fast.cuh"
#include "sm100.cuh"

namespace lime {

using namespace sm100;

namespace {

constexpr int kD = 128, kH = 4, kDH = 32, kTile = 128;
constexpr uint32_t kBlk = 128 * 128;

template <int L>
struct OnlineCfg {
  static constexpr int HL = kH * L;
  static constexpr uint32_t kStage = 2 * kBlk;         // [128 x 128] bf16 gather stage
  static constexpr uint32_t OFF_B = 2 * kStage;        // L^P_u^T
  static constexpr uint32_t OFF_G = OFF_B + kBlk;      // G image: 2 blocks of HL x 128 bytes
  static constexpr uint32_t OFF_BAR = OFF_G + 2 * HL * 128;
  static constexpr int SMEM = 1024 + OFF_BAR + 64 + 2 * 128 * 8;
};

template <int L>
__global__ void __launch_bounds__(128)
    k_score_online(const bf16* __restrict__ T, int64_t n_items, const uint8_t* __restrict__ gimg,
                   const int32_t* __restrict__ ids, const int64_t* __restrict__ off, int64_t B,
                   int64_t total, const bf16* __restrict__ LP, bf16* __restrict__ O,
                   unsigned* status) {
  using C = OnlineCfg<L>;
  constexpr int HL = C::HL;
  constexpr int CH = 2 * kD / 16;            // 16-byte chunks per item row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA0 = sm;                         // 2 gather stages
  uint8_t* sB = sm + C::OFF_B;
  uint8_t* sG = sm + C::OFF_G;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);   // [0] mma, [1] G image
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);
  int* abort_flag = reinterpret_cast<int*>(bar + 3);
  int64_t* s_ids = reinterpret_cast<int64_t*>(bar + 4);   // [2][128] IDs per stage (-1: zero row)

  pdl_wait();
  const int64_t u = blockIdx.x;
  int64_t a, b;
  user_range(off, u, B, total, &a, &b, status);
  const int nt = (int)((b - a + kTile - 1) / kTile);
  if ((int)blockIdx.y >= nt) return;   // uniform over the CTA: nothing allocated yet

  const int i = threadIdx.x;
  if (i == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (i < 32) tmem_alloc(slot, 256);
  __syncthreads();
  pdl_launch();   // after the TMEM allocation (the next kernel may allocate before it waits)
  if (i == 0) {
    mbar_arrive_expect_tx(&bar[1], 2 * HL * 128);
    bulk_load(sG, gimg, 2 * HL * 128, &bar[1]);
  }
  const int G = (int)gridDim.y;
  constexpr int64_t kNoRow = INT64_MIN;
  auto load_id = [&](int t) -> int64_t {
    const int64_t m = a + (int64_t)t * kTile + i;
    return (t < nt && m < b) ? (int64_t)ids[m] : kNoRow;
  };
  auto put_id = [&](int stage, int64_t id) {
    if (id == kNoRow) {
      id = -1;
    } else if (id < 0 || id >= n_items) {
      raise_flag(status, LIME_FLAG_BAD_ID);
      id = -2;   // a zero row whose output is written as zero
    }
    s_ids[stage * kTile + i] = id;
  };
  // gather of one tile's item rows: chunk q*128 + i is chunk (idx % CH) of
  // row idx / CH, so a warp reads whole rows; rows without an item are zero
  auto gather = [&](int stage) {
    uint8_t* dstA = sA0 + stage * C::kStage;
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int idx = q * 128 + i, r = idx / CH, cc = idx % CH;
      const int64_t id = s_ids[stage * kTile + r];
      const uint8_t* src = reinterpret_cast<const uint8_t*>(T) + (id < 0 ? 0 : id * 2 * kD) + cc * 16;
      cp_async16(dstA + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8), src, id >= 0);
    }
    cp_async_commit();
  };
  int64_t id_cur = load_id(blockIdx.y);
  int64_t id_nxt = load_id(blockIdx.y + G);
  // L^P_u transposed into sB: element (c, k) at sw128_offset(c, k), k >= L zero
  {
    const uint4* lp = reinterpret_cast<const uint4*>(LP + (u * L) * kD);
    uint4* stage = reinterpret_cast<uint4*>(sA0 + C::kStage);   // [L][128] bf16 in stage 1
    uint4 lv[L * kD / 8 / 128];
#pragma unroll
    for (int q = 0; q < L * kD / 8 / 128; ++q) lv[q] = __ldg(lp + q * 128 + i);
#pragma unroll
    for (int q = 0; q < L * kD / 8 / 128; ++q) stage[q * 128 + i] = lv[q];
    put_id(0, id_cur);
    __syncthreads();
    gather(0);
    const bf16* st = reinterpret_cast<const bf16*>(sA0 + C::kStage);
#pragma unroll
    for (int k8 = 0; k8 < 8; ++k8) {
      float f[8];
#pragma unroll
      for (int z = 0; z < 8; ++z) {
        const int k = k8 * 8 + z;
        f[z] = k < L ? __bfloat162float(st[k * kD + i]) : 0.f;
      }
      sw_st16(sB, kBlk, i, k8 * 8, pack8(f));
    }
  }
  __syncthreads();   // stage 1 is free again
  mbar_wait(&bar[1], 0, status, abort_flag);   // the G image
  const uint32_t tmem = *slot;
  const uint32_t ta = tmem + ((uint32_t)(i & ~31) << 16);
  uint32_t ph = 0;
  int it = 0;
  for (int t = blockIdx.y; t < nt; t += G, ++it) {
    const int cur = it & 1, nxt = cur ^ 1;
    const int64_t m0 = a + (int64_t)t * kTile;
    const int nv = b - m0 < kTile ? (int)(b - m0) : kTile;
    const bool more = t + G < nt;
    if (more) {
      put_id(nxt, id_nxt);
      __syncthreads();
      gather(nxt);                  // tile t+G streams in during tile t
      id_nxt = load_id(t + 2 * G);
    }
    if (more) cp_async_wait<1>(); else cp_async_wait<0>();
    uint8_t* sA = sA0 + cur * C::kStage;
    const bool bad = s_ids[cur * kTile + i] == -2;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (i == 0) {
      tc_fence_after();
      mma_tile(tmem, smem_u32(sA), kBlk, smem_u32(sG), HL * 128, HL, kD, false);
      mma_commit(&bar[0]);
    }
    mbar_wait(&bar[0], ph, status, abort_flag);
    ph ^= 1u;
    tc_fence_after();
    {
      // thread = candidate row: per head softmax over the L scores; the bf16
      // weights overwrite the row's gathered item values (MMA 1 has read them)
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        float z[L];
#pragma unroll
        for (int q = 0; q < L / 16; ++q) tmem_ld16(ta + h * L + q * 16, z + q * 16);
        tmem_ld_wait();
        float m = z[0];
#pragma unroll
        for (int k = 1; k < L; ++k) m = fmaxf(m, z[k]);
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < L; ++k) { z[k] = __expf(z[k] - m); s += z[k]; }
        const float inv = 1.0f / s;
#pragma unroll
        for (int k = 0; k < L; ++k) z[k] *= inv;
#pragma unroll
        for (int q = 0; q < L / 8; ++q) sw_st16(sA, kBlk, i, h * L + q * 8, pack8(z + q * 8));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (i == 0) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        const uint32_t aa = smem_u32(sA + ((h * L) >> 6) * kBlk + ((h * L) & 63) * 2);
        const uint32_t bb = smem_u32(sB + h * kDH * 128);
        mma_tile(tmem + 128 + h * kDH, aa, kBlk, bb, kBlk, kDH, L, false);
      }
      mma_commit(&bar[0]);
    }
    mbar_wait(&bar[0], ph, status, abort_flag);
    ph ^= 1u;
    tc_fence_after();
    {
      // thread = row: TMEM -> bf16 -> swizzled staging in sA (MMA 2 is done with it)
      float row[kD];
#pragma unroll
      for (int q = 0; q < 8; ++q) tmem_ld16(ta + 128 + q * 16, row + q * 16);
      tmem_ld_wait();
      if (bad) {
#pragma unroll
        for (int c = 0; c < kD; ++c) row[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) sw_st16(sA, kBlk, i, c * 8, pack8(row + c * 8));
    }
    tc_fence_before();
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int idx = q * 128 + i, r = idx / 16, cc = idx % 16;
      if (r < nv)
        reinterpret_cast<uint4*>(O + (m0 + r) * kD)[cc] = sw_ld16(sA, kBlk, r, cc * 8);
    }
    __syncthreads();   // this stage and TMEM are reused two tiles on
  }
  if (i < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int L>
int launch_online(int64_t B, const void* T, int64_t n_items, const void* image, const int32_t* ids,
                  const int64_t* off, int64_t total, const void* LP, void* O, unsigned* status,
                  cudaStream_t st) {
  using C = OnlineCfg<L>;
  if (cudaFuncSetAttribute(k_score_online<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return LIME_ERR_CUDA;
  const int64_t target = 2LL * num_sms();
  int64_t G = (target + B - 1) / B;
  const int64_t tiles_hi = (total + kTile - 1) / kTile;
  if (G > tiles_hi) G = tiles_hi;
  if (G < 1) G = 1;
  if (G > 65535) G = 65535;
  return launch_pdl(k_score_online<L>, dim3((unsigned)B, (unsigned)G), dim3(128), C::SMEM, st, 1,
                    (const bf16*)T, n_items, (const uint8_t*)image, ids, off, B, total,
                    (const bf16*)LP, (bf16*)O, status);
}

}  // namespace

bool fast_online_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && (D.l == 16 || D.l == 32);
}

int fast_score_online(const lime_dims& D, int64_t B, const void* T, int64_t n_items,
                      const void* image, const int32_t* ids, const int64_t* off, int64_t total,
                      const void* LP, void* O, unsigned* status, cudaStream_t st) {
  if (D.l == 16)
    return launch_online<16>(B, T, n_items, image, ids, off, total, LP, O, status, st);
  return launch_online<32>(B, T, n_items, image, ids, off, total, LP, O, status, st);
}

}  // namespace lime
