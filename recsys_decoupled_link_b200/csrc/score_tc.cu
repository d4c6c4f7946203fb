// Cached candidate scoring on the 5th-generation tensor cores (bf16, d = 128,
// 4 heads of 32, l in {16, 32, 64}).
//
// LIME note, 关键设计 1 and 一个完整示例 step 3: O_m = phi(T_m L^T) L^P, i.e.
// for candidate m of user u and head h, O[m, h-cols] = sum_k cache[id_m, h, k]
// L^P_u[k, h-cols].  Per 128 candidates of one user this is, for each head, a
// [128 x l] x [l x 32] product: the gathered cache rows (row = candidate, H*l
// weights) are the A operand, the user's L^P transposed is the B operand.
// Arithmetic intensity is 16 flop per byte, above what the CUDA cores can
// sustain at HBM speed, so the contraction runs on the tensor cores and the
// kernel stays bound by the gather.
//
// CTA (u, g) stages L^P_u^T once (a [128 c x 64 k] 128B-swizzled block, k >= l
// zero) and walks tiles g, g + G, ... of user u's candidates.  Per tile each
// thread gathers one candidate's row with 16-byte loads into the swizzled A
// tile (an out-of-range ID gives a zero row and LIME_FLAG_BAD_ID), thread 0
// issues one MMA group per head into TMEM, and each thread stores its row of
// O as bf16.  No workspace is used.
#include "lime_fast.cuh"
#include "sm100.cuh"

namespace lime {

using namespace sm100;

namespace {

constexpr int kD = 128, kH = 4, kDH = 32, kTile = 128;
constexpr uint32_t kBlk = 128 * 128;

template <int L>
__global__ void __launch_bounds__(128)
    k_score_tc(const bf16* __restrict__ cache, int64_t n_items, const int32_t* __restrict__ ids,
               const int64_t* __restrict__ off, int64_t B, int64_t total,
               const bf16* __restrict__ LP, bf16* __restrict__ O, unsigned* status) {
  constexpr int HL = kH * L;
  constexpr int ABLK = HL / 64;             // A blocks of 64 columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = sm;
  uint8_t* sB = sm + ABLK * kBlk;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + kBlk);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(bar + 2);

  const int64_t u = blockIdx.x;
  int64_t a, b;
  user_range(off, u, B, total, &a, &b, status);
  const int nt = (int)((b - a + kTile - 1) / kTile);
  if ((int)blockIdx.y >= nt) return;   // uniform over the CTA: nothing allocated yet

  const int i = threadIdx.x;
  if (i == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (i < 32) tmem_alloc(slot, 128);
  // L^P_u transposed: thread i owns output column c = i
  {
    const bf16* lp = LP + (u * L) * kD + i;
    for (int k = 0; k < 64; ++k)
      *reinterpret_cast<bf16*>(sB + sw128_offset(i, k)) =
          k < L ? lp[(int64_t)k * kD] : __float2bfloat16_rn(0.f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t ta = tmem + ((uint32_t)(i & ~31) << 16);
  uint32_t ph = 0;
  for (int t = blockIdx.y; t < nt; t += gridDim.y) {
    const int64_t m0 = a + (int64_t)t * kTile;
    const int nv = b - m0 < kTile ? (int)(b - m0) : kTile;
    {
      int64_t id = -1;
      if (i < nv) {
        id = ids[m0 + i];
        if (id < 0 || id >= n_items) {
          raise_flag(status, LIME_FLAG_BAD_ID);
          id = -1;
        }
      }
      uint4 v[HL / 8];
      const uint4* src = reinterpret_cast<const uint4*>(cache + (id < 0 ? 0 : id) * HL);
#pragma unroll
      for (int c = 0; c < HL / 8; ++c) v[c] = id < 0 ? make_uint4(0, 0, 0, 0) : __ldg(src + c);
#pragma unroll
      for (int c = 0; c < HL / 8; ++c) sw_st16(sA, kBlk, i, c * 8, v[c]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (i == 0) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < kH; ++h)
        mma_tile(tmem + h * kDH, smem_u32(sA + ((h * L) >> 6) * kBlk + ((h * L) & 63) * 2), kBlk,
                 smem_u32(sB + h * kDH * 128), kBlk, kDH, L, false);
      mma_commit(bar);
    }
    mbar_wait(bar, ph, status, abort_flag);
    ph ^= 1u;
    tc_fence_after();
    float row[kD];
#pragma unroll
    for (int q = 0; q < 8; ++q) tmem_ld16(ta + q * 16, row + q * 16);
    tmem_ld_wait();
    if (i < nv) {
      uint4* dst = reinterpret_cast<uint4*>(O + (m0 + i) * kD);
#pragma unroll
      for (int c = 0; c < 16; ++c) dst[c] = pack8(row + c * 8);
    }
    tc_fence_before();
    __syncthreads();   // TMEM and the A tile are reused by the next tile
  }
  if (i < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int L>
int launch_score(int64_t B, const void* cache, int64_t n_items, const int32_t* ids,
                 const int64_t* off, int64_t total, const void* LP, void* O, unsigned* status,
                 cudaStream_t st) {
  constexpr int HL = kH * L;
  const int smem = 1024 + (HL / 64 + 1) * kBlk + 64;
  if (cudaFuncSetAttribute(k_score_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return LIME_ERR_CUDA;
  // enough (user, slot) CTAs to fill every SM a few times over
  const int64_t target = 4LL * num_sms();
  int64_t G = (target + B - 1) / B;
  const int64_t tiles_hi = (total + kTile - 1) / kTile;
  if (G > tiles_hi) G = tiles_hi;
  if (G < 1) G = 1;
  if (G > 65535) G = 65535;
  dim3 grid((unsigned)B, (unsigned)G);
  k_score_tc<L><<<grid, 128, smem, st>>>((const bf16*)cache, n_items, ids, off, B, total,
                                          (const bf16*)LP, (bf16*)O, status);
  note_launches(1);
  return LIME_OK;
}

}  // namespace

bool fast_score_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && (D.l == 16 || D.l == 32 || D.l == 64);
}

int fast_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
               const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
               float* ws, unsigned* status, cudaStream_t st) {
  (void)ws;
  switch (D.l) {
    case 16: return launch_score<16>(B, cache, n_items, ids, off, total, LP, O, status, st);
    case 32: return launch_score<32>(B, cache, n_items, ids, off, total, LP, O, status, st);
    default: return launch_score<64>(B, cache, n_items, ids, off, total, LP, O, status, st);
  }
}

}  // namespace lime
