// Uncached (online) candidate scoring on the 5th-generation tensor cores
// (bf16, d = 128, 4 heads of 32, l in {16, 32, 64}).
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
// CTA (u, g) walks tiles g, g + G, ... of user u's candidates with four
// warpgroups (two for l = 64) that take turns (tile j of the CTA goes to
// group j % groups): each has its own gather stage, H*l TMEM columns (S, then
// O over it) and MMA barrier, so the groups' gathers, MMAs and softmaxes
// overlap one another.  With l = 64 a stage is 64 KB, since the [128 x 256]
// bf16 weights overwrite the gathered rows.  Thread = candidate row (a TMEM
// lane) within its group.
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
  static constexpr int GROUPS = HL > 128 ? 2 : 4;      // warpgroups (HL TMEM columns each)
  static constexpr int THREADS = 128 * GROUPS;
  static constexpr uint32_t TCOLS = HL > 128 ? 256 : 128;   // TMEM columns per group
  // a gather stage: the [128 x 128] bf16 item rows, later the [128 x HL] weights
  static constexpr uint32_t kStage = (HL > 128 ? HL / 64 : 2) * kBlk;
  static constexpr uint32_t OFF_B = GROUPS * kStage;   // L^P_u^T (after the groups' stages)
  static constexpr uint32_t OFF_G = OFF_B + kBlk;      // G image: 2 blocks of HL x 128 bytes
  static constexpr uint32_t OFF_BAR = OFF_G + 2 * HL * 128;
  static constexpr int SMEM = 1024 + OFF_BAR + 64 + 4 * 128 * 4;
};

template <int L>
__global__ void __launch_bounds__(OnlineCfg<L>::THREADS, 1)
    k_score_online(const bf16* __restrict__ T, int64_t n_items, const uint8_t* __restrict__ gimg,
                   const int32_t* __restrict__ ids, const int64_t* __restrict__ off, int64_t B,
                   int64_t total, const bf16* __restrict__ LP, bf16* __restrict__ O, int phi,
                   unsigned* status) {
  using C = OnlineCfg<L>;
  constexpr int HL = C::HL;
  constexpr int kGroups = C::GROUPS, kOnThreads = C::THREADS;
  constexpr int CH = 2 * kD / 16;            // 16-byte chunks per item row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = sm + C::OFF_B;
  uint8_t* sG = sm + C::OFF_G;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);   // [0..3] mma per group, [4] G
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 5);
  int* abort_flag = reinterpret_cast<int*>(bar + 6);
  int32_t* s_ids_all = reinterpret_cast<int32_t*>(bar + 8);   // [group][128]

  pdl_wait();
  const int64_t u = blockIdx.x;
  int64_t a, b;
  user_range(off, u, B, total, &a, &b, status);
  const int nt = (int)((b - a + kTile - 1) / kTile);
  if ((int)blockIdx.y >= nt) return;   // uniform over the CTA: nothing allocated yet

  const int tid = threadIdx.x;
  const int i = tid & 127;                   // row (and TMEM lane) within the group
  const int grp = tid >> 7;                  // warpgroup 0 .. kGroups-1
  if (tid == 0) {
    for (int q = 0; q <= kGroups; ++q) mbar_init(&bar[q], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 32) tmem_alloc(slot, 512);
  __syncthreads();
  pdl_launch();   // after the TMEM allocation (the next kernel may allocate before it waits)
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar[kGroups], 2 * HL * 128);
    bulk_load(sG, gimg, 2 * HL * 128, &bar[kGroups]);
  }
  // L^P_u transposed into sB: element (c, k) at sw128_offset(c, k), k >= L zero;
  // staged through the first gather stage (unused yet)
  {
    const uint4* lp = reinterpret_cast<const uint4*>(LP + (u * L) * kD);
    uint4* stage = reinterpret_cast<uint4*>(sm);
    for (int idx = tid; idx < L * kD / 8; idx += kOnThreads) stage[idx] = __ldg(lp + idx);
    __syncthreads();
    const bf16* st = reinterpret_cast<const bf16*>(sm);
#pragma unroll
    for (int k8 = grp * (8 / kGroups); k8 < (grp + 1) * (8 / kGroups); ++k8) {
      float f[8];
#pragma unroll
      for (int z = 0; z < 8; ++z) {
        const int k = k8 * 8 + z;
        f[z] = k < L ? __bfloat162float(st[k * kD + i]) : 0.f;
      }
      sw_st16(sB, kBlk, i, k8 * 8, pack8(f));
    }
  }
  fence_proxy_async_smem();
  __syncthreads();   // sB is complete and the staging stage is free again
  mbar_wait(&bar[kGroups], 0, status, abort_flag);   // the G image
  const uint32_t tmem = *slot + (uint32_t)grp * C::TCOLS;   // this group's S, then O
  const uint32_t ta = tmem + ((uint32_t)(i & ~31) << 16);
  const int G = (int)gridDim.y;
  const int step = kGroups * G;              // a group's stride over the user's tiles
  const int t0 = blockIdx.y + grp * G;
  uint8_t* sA = sm + grp * C::kStage;        // this group's stage
  int32_t* s_ids = s_ids_all + grp * 128;
  uint64_t* mbar = &bar[grp];
  auto gsync = [&]() { named_bar_sync(1 + grp, 128); };
  constexpr int64_t kNoRow = INT64_MIN;
  auto load_id = [&](int t) -> int64_t {
    const int64_t m = a + (int64_t)t * kTile + i;
    return (t < nt && m < b) ? (int64_t)ids[m] : kNoRow;
  };
  auto put_id = [&](int64_t id) {
    int32_t v;
    if (id == kNoRow) {
      v = -1;
    } else if (id < 0 || id >= n_items) {
      raise_flag(status, LIME_FLAG_BAD_ID);
      v = -2;   // a zero row whose output is written as zero
    } else {
      v = (int32_t)id;
    }
    s_ids[i] = v;
  };
  // gather of one tile's item rows: chunk q*128 + i is chunk (idx % CH) of row
  // idx / CH, so a warp reads whole rows; rows without an item are zero
  auto gather = [&]() {
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int idx = q * 128 + i, r = idx / CH, cc = idx % CH;
      const int64_t id = s_ids[r];
      const uint8_t* src = reinterpret_cast<const uint8_t*>(T) + (id < 0 ? 0 : id * 2 * kD) + cc * 16;
      cp_async16(sA + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8), src, id >= 0);
    }
    cp_async_commit();
  };
  int64_t id_cur = load_id(t0);
  uint32_t ph = 0;
  for (int t = t0; t < nt; t += step) {
    const int64_t m0 = a + (int64_t)t * kTile;
    const int nv = b - m0 < kTile ? (int)(b - m0) : kTile;
    put_id(id_cur);
    gsync();
    gather();
    id_cur = load_id(t + step);     // the group's next IDs while the rows stream in
    cp_async_wait<0>();
    const bool bad = s_ids[i] == -2;
    fence_proxy_async_smem();
    tc_fence_before();
    gsync();
    if (i == 0) {
      tc_fence_after();
      mma_tile(tmem, smem_u32(sA), kBlk, smem_u32(sG), HL * 128, HL, kD, false);
      mma_commit(mbar);
    }
    mbar_wait(mbar, ph, status, abort_flag);
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
        if (phi == LIME_PHI_SILU) {
#pragma unroll
          for (int k = 0; k < L; ++k) z[k] = __fdividef(z[k], 1.0f + __expf(-z[k])) * (1.0f / L);
        } else {
          float m = z[0];
#pragma unroll
          for (int k = 1; k < L; ++k) m = fmaxf(m, z[k]);
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < L; ++k) { z[k] = __expf(z[k] - m); s += z[k]; }
          const float inv = 1.0f / s;
#pragma unroll
          for (int k = 0; k < L; ++k) z[k] *= inv;
        }
#pragma unroll
        for (int q = 0; q < L / 8; ++q) sw_st16(sA, kBlk, i, h * L + q * 8, pack8(z + q * 8));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    gsync();
    if (i == 0) {
      tc_fence_after();
      // O over the score columns (every thread has read its scores)
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        const uint32_t aa = smem_u32(sA + ((h * L) >> 6) * kBlk + ((h * L) & 63) * 2);
        const uint32_t bb = smem_u32(sB + h * kDH * 128);
        mma_tile(tmem + h * kDH, aa, kBlk, bb, kBlk, kDH, L, false);
      }
      mma_commit(mbar);
    }
    mbar_wait(mbar, ph, status, abort_flag);
    ph ^= 1u;
    tc_fence_after();
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      // thread = row, half hf of its columns: TMEM -> bf16 -> swizzled staging
      // in sA (MMA 2 is done with it)
      float row[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(ta + hf * 64 + q * 16, row + q * 16);
      tmem_ld_wait();
      if (bad) {
#pragma unroll
        for (int c = 0; c < 64; ++c) row[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) sw_st16(sA, kBlk, i, hf * 64 + c * 8, pack8(row + c * 8));
    }
    tc_fence_before();
    gsync();
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int idx = q * 128 + i, r = idx / 16, cc = idx % 16;
      if (r < nv)
        reinterpret_cast<uint4*>(O + (m0 + r) * kD)[cc] = sw_ld16(sA, kBlk, r, cc * 8);
    }
  }
  __syncthreads();
  if (tid < 32) {
    tc_fence_after();
    tmem_dealloc(*slot, 512);
  }
}

template <int L>
int launch_online(int64_t B, const void* T, int64_t n_items, const void* image, const int32_t* ids,
                  const int64_t* off, int64_t total, const void* LP, void* O, int phi,
                  unsigned* status, cudaStream_t st) {
  constexpr int kOnThreads = OnlineCfg<L>::THREADS;
  using C = OnlineCfg<L>;
  if (cudaFuncSetAttribute(k_score_online<L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return LIME_ERR_CUDA;
  // one CTA per SM (its TMEM allocation is all 512 columns): (user, slot) CTAs
  // in a single wave, as many slots per user as fit
  int64_t G = num_sms() / B;
  const int64_t tiles_hi = (total + kTile - 1) / kTile;
  if (G > tiles_hi) G = tiles_hi;
  if (G < 1) G = 1;
  if (G > 65535) G = 65535;
  return launch_pdl(k_score_online<L>, dim3((unsigned)B, (unsigned)G), dim3(kOnThreads), C::SMEM, st, 1,
                    (const bf16*)T, n_items, (const uint8_t*)image, ids, off, B, total,
                    (const bf16*)LP, (bf16*)O, phi, status);
}

}  // namespace

bool fast_online_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && (D.l == 16 || D.l == 32 || D.l == 64);
}

int fast_score_online(const lime_dims& D, int64_t B, const void* T, int64_t n_items,
                      const void* image, const int32_t* ids, const int64_t* off, int64_t total,
                      const void* LP, void* O, unsigned* status, cudaStream_t st) {
  if (D.l == 16)
    return launch_online<16>(B, T, n_items, image, ids, off, total, LP, O, D.phi, status, st);
  if (D.l == 64)
    return launch_online<64>(B, T, n_items, image, ids, off, total, LP, O, D.phi, status, st);
  return launch_online<32>(B, T, n_items, image, ids, off, total, LP, O, D.phi, status, st);
}

}  // namespace lime
