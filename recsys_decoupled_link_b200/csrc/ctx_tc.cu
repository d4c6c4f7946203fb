// Context links on the 5th-generation tensor cores (bf16, d = 128, c = 64 or
// 128 context features).
//
// LIME note, 整体框架 (flowchart node "L^C = MLP(L ⊕ E^C)"): every user's
// links are the global links L fused with the user's context features,
//     L^C_u = SiLU([L ⊕ ctx_u] Wc1 + bc1) Wc2 + bc2,
// one [l x (d + c)] -> [l x d] -> [l x d] MLP per user.  Over all users this
// is two GEMMs with B*l rows; row r is link k = r % l of user u = r / l.
//
// One CTA per 128 rows (persistent over more tiles when there are more tiles
// than SMs).  Wc1 and Wc2 are loaded once per CTA with TMA as MN-major operand
// images (row-major [K x 128] tiles in 128-byte-swizzled 64-column blocks);
// per tile the [128 x (d + c)] input rows are gathered with asynchronous
// copies into a K-major operand, GEMM 1
// runs into TMEM, the epilogue adds bc1, applies SiLU and writes the hidden
// rows as bf16 hi + lo halves (hi = bf16(x), lo = bf16(x - hi)), GEMM 2 takes
// both halves (so the hidden layer keeps about 16 mantissa bits), and the
// second epilogue adds bc2 and stores bf16 rows with coalesced 16-byte stores.
// 512 threads: thread (row, part) handles 32 of the 128 columns of a row.
#include "lime_fast.cuh"
#include "sm100.cuh"

namespace lime {

using namespace sm100;

namespace {

constexpr int kD = 128;
constexpr uint32_t kBlk = 128 * 128;   // one [128 x 64] bf16 block

__global__ void __launch_bounds__(512, 1)
    k_context_tc(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                 int c, int l, int64_t rows, const bf16* __restrict__ L,
                 const bf16* __restrict__ ctx, const bf16* __restrict__ bc1,
                 const bf16* __restrict__ bc2, bf16* __restrict__ LC, unsigned* status) {
  const int din = kD + c;                 // 192 or 256
  const uint32_t w1_blk = (uint32_t)din * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = sm;                       // [128 x din] K-major -> hidden hi -> output staging
  uint8_t* sHlo = sm + 4 * kBlk;          // hidden lo
  uint8_t* sW2 = sm + 6 * kBlk;           // Wc2 [128 x 128] MN-major
  uint8_t* sW1 = sm + 8 * kBlk;           // Wc1 [din x 128] MN-major (2 blocks of din rows)
  float* sbias = reinterpret_cast<float*>(sW1 + 2 * w1_blk);        // bc1 [128], bc2 [128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sbias + 2 * kD);      // [0] mma, [1] weights
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);
  int* abort_flag = reinterpret_cast<int*>(bar + 3);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 32) tmem_alloc(slot, 256);
  tc_fence_before();
  __syncthreads();
  pdl_launch();
  pdl_wait();
  // the biases as fp32 in shared memory (the epilogues read them per column;
  // the gather's barrier below orders these writes before those reads)
  if (tid < 2 * kD) sbias[tid] = __bfloat162float(tid < kD ? bc1[tid] : bc2[tid - kD]);
  // weights: TMA tiles of the row-major [K x 128] matrices in 128-byte
  // swizzle are exactly the MN-major operand images (64 columns per block)
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar[1], 2 * w1_blk + 2 * kBlk);
    tma_load_2d(sW1, &tmW1, 0, 0, &bar[1]);
    tma_load_2d(sW1 + w1_blk, &tmW1, 64, 0, &bar[1]);
    tma_load_2d(sW2, &tmW2, 0, 0, &bar[1]);
    tma_load_2d(sW2 + kBlk, &tmW2, 64, 0, &bar[1]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const int warp = tid >> 5, part = warp >> 2;
  const int row = (warp & 3) * 32 + (tid & 31);
  const int c0 = part * 32;
  const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const int64_t n_tiles = (rows + 127) / 128;
  const int cpr = din / 8;                // 16-byte chunks per input row
  uint32_t ph = 0;
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int64_t r0 = t * 128;
    const int nv = rows - r0 < 128 ? (int)(rows - r0) : 128;
    // gather the input rows [L_k ⊕ ctx_u] with asynchronous copies; rows past
    // the end are zero
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int idx = q * 512 + tid, r = idx / cpr, cc = idx - r * cpr;
      if (idx < 128 * cpr) {
        const bool ok = r < nv;
        const int64_t R = ok ? r0 + r : 0, u = R / l, k = R - u * l;
        const void* src = cc < 16 ? (const void*)(L + k * kD + cc * 8)
                                  : (const void*)(ctx + u * c + (cc - 16) * 8);
        cp_async16(sX + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8), src, ok);
      }
    }
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      if (t == blockIdx.x) mbar_wait(&bar[1], 0, status, abort_flag);   // weights landed
      tc_fence_after();
      mma_tile_bmn(tmem, smem_u32(sX), kBlk, smem_u32(sW1), w1_blk, 128, din, false);
    }
    cta_mma_wait(&bar[0], ph, status, abort_flag);
    {
      float x[32];
      tmem_ld16(ta + c0, x);
      tmem_ld16(ta + c0 + 16, x + 16);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float h8[8], l8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // SiLU with the hardware exp2 / reciprocal approximations (a few
          // ulp; the hidden value is kept to about 16 bits as hi + lo)
          const float a = x[q * 8 + j] + sbias[c0 + q * 8 + j];
          const float v = __fdividef(a, 1.0f + __expf(-a));
          h8[j] = __bfloat162float(__float2bfloat16_rn(v));
          l8[j] = v - h8[j];
        }
        sw_st16(sX, kBlk, row, c0 + q * 8, pack8(h8));
        sw_st16(sHlo, kBlk, row, c0 + q * 8, pack8(l8));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      mma_tile_bmn(tmem + 128, smem_u32(sX), kBlk, smem_u32(sW2), kBlk, 128, kD, false);
      mma_tile_bmn(tmem + 128, smem_u32(sHlo), kBlk, smem_u32(sW2), kBlk, 128, kD, true);
    }
    cta_mma_wait(&bar[0], ph, status, abort_flag);
    {
      float x[32];
      tmem_ld16(ta + 128 + c0, x);
      tmem_ld16(ta + 128 + c0 + 16, x + 16);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] += sbias[kD + c0 + j];
      // the hidden-hi operand (GEMM 2 is done with it) becomes the output staging
#pragma unroll
      for (int q = 0; q < 4; ++q) sw_st16(sX, kBlk, row, c0 + q * 8, pack8(x + q * 8));
    }
    tc_fence_before();
    __syncthreads();
    tile_store_rows(sX, LC + r0 * kD, nv);
    __syncthreads();   // sX is rewritten by the next tile's gather
  }
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool fast_ctx_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && (D.c == 64 || D.c == 128);
}

size_t fast_ctx_smem(const lime_dims& D) {
  return 1024 + 8 * (size_t)kBlk + 2 * (size_t)(kD + D.c) * 128 + 2 * kD * 4 + 64;   // + biases, barriers
}

int fast_context_links(const lime_dims& D, int64_t B, const void* L, const void* ctx,
                       const lime_ctx_mlp& w, void* LC, unsigned* status, cudaStream_t st) {
  const int64_t rows = B * D.l;
  const int smem = (int)fast_ctx_smem(D);
  if (cudaFuncSetAttribute(k_context_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return LIME_ERR_CUDA;
  int64_t grid = (rows + 127) / 128;
  if (grid > num_sms()) grid = num_sms();
  CUtensorMap tmW1, tmW2;
  if (!make_tmap_2d_bf16(&tmW1, w.Wc1, kD, (uint64_t)(kD + D.c), kD * 2, 64, kD + D.c) ||
      !make_tmap_2d_bf16(&tmW2, w.Wc2, kD, kD, kD * 2, 64, kD))
    return LIME_ERR_CUDA;
  return launch_pdl(k_context_tc, dim3((unsigned)grid), dim3(512), smem, st, 1, tmW1, tmW2, D.c,
                    D.l, rows, (const bf16*)L, (const bf16*)ctx, (const bf16*)w.bc1,
                    (const bf16*)w.bc2, (bf16*)LC, status);
}

}  // namespace lime
