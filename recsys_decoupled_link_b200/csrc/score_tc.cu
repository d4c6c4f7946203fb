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
// zero) and walks tiles g, g + G, ... of user u's candidates.  The rows of
// tile t+G are gathered with asynchronous 16-byte copies (cp.async) into the
// second of two stages while tile t is multiplied and written, and the IDs of
// tile t+2G are read meanwhile.  A warp's copies cover whole cache rows, so
// the gather is coalesced; an out-of-range ID gives a zero row and
// LIME_FLAG_BAD_ID.  Thread 0 issues one MMA group per head into TMEM, each
// thread stages its row of O in bf16, and the tile is written back with
// coalesced 16-byte stores.  No workspace is used.
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
  // A tile blocks of 64 columns; at least 2 because the same region later
  // stages the [128 x 128] output tile
  constexpr int ABLK = HL / 64 < 2 ? 2 : HL / 64;
  constexpr uint32_t kStage = ABLK * kBlk;
  constexpr int CH = HL / 8;                 // 16-byte chunks per cache row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA0 = sm;                         // 2 stages: gathered rows, then output staging
  uint8_t* sB = sm + 2 * kStage;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + kBlk);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(bar + 2);
  int64_t* s_ids = reinterpret_cast<int64_t*>(bar + 4);   // [2][128] candidate IDs per stage

  pdl_wait();
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
  __syncthreads();
  pdl_launch();   // after the TMEM allocation (the next kernel may allocate before it waits)
  const int G = (int)gridDim.y;
  // candidate ID of row i of tile t (kNoRow past the user's rows); loaded a
  // tile ahead.  A staged ID of -1 means "zero row".
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
      id = -1;
    }
    s_ids[stage * kTile + i] = id;
  };
  // gather of one tile into a stage: chunk q*128 + i is chunk (idx % CH) of
  // row idx / CH, so a warp reads whole cache rows; bad or missing IDs give
  // zero rows
  auto gather = [&](int stage) {
    uint8_t* sA = sA0 + stage * kStage;
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int idx = q * 128 + i, r = idx / CH, cc = idx % CH;
      const int64_t id = s_ids[stage * kTile + r];
      const bf16* src = cache + (id < 0 ? 0 : id * HL) + cc * 8;
      cp_async16(sA + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8), src, id >= 0);
    }
    cp_async_commit();
  };
  int64_t id_cur = load_id(blockIdx.y);
  int64_t id_nxt = load_id(blockIdx.y + G);
  // L^P_u transposed into sB: element (c, k) at sw128_offset(c, k), k >= L zero.
  // Coalesced 16-byte copies of L^P_u into stage 1 (unused yet), then each
  // thread builds its own row c of the transpose with 16-byte swizzled stores.
  {
    const uint4* lp = reinterpret_cast<const uint4*>(LP + (u * L) * kD);
    uint4* stage = reinterpret_cast<uint4*>(sA0 + kStage);   // [L][128] bf16, plain row-major
    uint4 lv[L * kD / 8 / 128];
#pragma unroll
    for (int q = 0; q < L * kD / 8 / 128; ++q) lv[q] = __ldg(lp + q * 128 + i);
#pragma unroll
    for (int q = 0; q < L * kD / 8 / 128; ++q) stage[q * 128 + i] = lv[q];
    put_id(0, id_cur);
    __syncthreads();
    gather(0);       // the first tile's rows stream in while L^P is transposed
    const bf16* st = reinterpret_cast<const bf16*>(sA0 + kStage);
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
      id_nxt = load_id(t + 2 * G);  // and the IDs of tile t+2G
    }
    if (more) cp_async_wait<1>(); else cp_async_wait<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    uint8_t* sA = sA0 + cur * kStage;
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
    {
      // thread = row: TMEM -> bf16 -> swizzled staging in sA (the MMA is done with it)
      float row[kD];
#pragma unroll
      for (int q = 0; q < 8; ++q) tmem_ld16(ta + q * 16, row + q * 16);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 16; ++c) sw_st16(sA, kBlk, i, c * 8, pack8(row + c * 8));
    }
    tc_fence_before();
    __syncthreads();
    // cooperative, coalesced store of the valid rows
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
    tmem_dealloc(tmem, 128);
  }
}

template <int L>
int launch_score(int64_t B, const void* cache, int64_t n_items, const int32_t* ids,
                 const int64_t* off, int64_t total, const void* LP, void* O, unsigned* status,
                 cudaStream_t st) {
  constexpr int HL = kH * L;
  const int smem = 1024 + (2 * (HL / 64 < 2 ? 2 : HL / 64) + 1) * kBlk + 64 + 2 * 128 * 8;
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
  return launch_pdl(k_score_tc<L>, grid, dim3(128), smem, st, 1, (const bf16*)cache, n_items,
                    ids, off, B, total, (const bf16*)LP, (bf16*)O, status);
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
