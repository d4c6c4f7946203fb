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

// Shared memory of k_score_tc<L, U8>: bf16 cache = two A stages (the gather
// lands in the MMA operand directly); int8 cache = one A tile plus two byte
// stages (the gather lands in a byte stage, which is widened into A).
template <int L, bool U8>
struct ScoreCfg {
  static constexpr int HL = kH * L;
  // A tile blocks of 64 columns; at least 2 because the same region later
  // stages the [128 x 128] output tile
  static constexpr int ABLK = HL / 64 < 2 ? 2 : HL / 64;
  static constexpr uint32_t kA = ABLK * kBlk;
  static constexpr int RB = U8 ? HL : 2 * HL;          // bytes per cache row
  static constexpr uint32_t kG = U8 ? 128u * RB : kA;  // one gather stage
  static constexpr uint32_t OFF_G = U8 ? kA : 0;
  static constexpr uint32_t OFF_B = OFF_G + 2 * kG;
  static constexpr int SMEM = 1024 + OFF_B + kBlk + 64 + 2 * 128 * 8;
};

template <int L, bool U8>
__global__ void __launch_bounds__(128)
    k_score_tc(const void* __restrict__ cache_v, int64_t n_items, const int32_t* __restrict__ ids,
               const int64_t* __restrict__ off, int64_t B, int64_t total,
               const bf16* __restrict__ LP, bf16* __restrict__ O, unsigned* status) {
  using C = ScoreCfg<L, U8>;
  constexpr int HL = C::HL;
  constexpr uint32_t kStage = C::kG;
  constexpr int CH = C::RB / 16;             // 16-byte chunks per cache row
  constexpr int kSw = CH >= 8 ? 7 : CH - 1;  // XOR swizzle of the byte stages
  const uint8_t* cache = reinterpret_cast<const uint8_t*>(cache_v);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA0 = sm + C::OFF_G;              // 2 gather stages
  uint8_t* sAu = sm;                         // int8 cache: the widened A tile
  uint8_t* sB = sm + C::OFF_B;
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
  // zero rows.  bf16 rows land in the swizzled MMA operand; byte rows in a
  // [128 x RB] stage with chunk c of row r at r*RB + ((c ^ (r & kSw)) * 16).
  auto gather = [&](int stage) {
    uint8_t* sG = sA0 + stage * kStage;
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int idx = q * 128 + i, r = idx / CH, cc = idx % CH;
      const int64_t id = s_ids[stage * kTile + r];
      const uint8_t* src = cache + (id < 0 ? 0 : id * C::RB) + cc * 16;
      uint8_t* dst = U8 ? sG + r * C::RB + ((cc ^ (r & kSw)) << 4)
                        : sG + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8);
      cp_async16(dst, src, id >= 0);
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
    uint4* stage = reinterpret_cast<uint4*>(sA0 + kStage);   // [L][128] bf16 in gather stage 1
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
      // int8 cache: fp16 operands (A holds the bytes exactly, L^P converts exactly)
      sw_st16(sB, kBlk, i, k8 * 8, U8 ? pack8_f16(f) : pack8(f));
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
    uint8_t* sA = sA0 + cur * kStage;
    if constexpr (U8) {
      // widen this thread's row of bytes into the fp16 operand, exactly: the
      // half with bits 0x64 | b is 1024 + b, minus 1024 gives b
      __syncthreads();
      const uint8_t* sG = sA0 + cur * kStage;
      const __half2 k1024 = __float2half2_rn(1024.0f);
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(sG + i * C::RB + ((c ^ (i & kSw)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t lo = __byte_perm(w[j], 0x64646464u, 0x4140);
          uint32_t hi = __byte_perm(w[j], 0x64646464u, 0x4342);
          __half2 l2 = __hsub2(*reinterpret_cast<__half2*>(&lo), k1024);
          __half2 h2 = __hsub2(*reinterpret_cast<__half2*>(&hi), k1024);
          h[2 * j] = *reinterpret_cast<uint32_t*>(&l2);
          h[2 * j + 1] = *reinterpret_cast<uint32_t*>(&h2);
        }
        sw_st16(sAu, kBlk, i, c * 16, make_uint4(h[0], h[1], h[2], h[3]));
        sw_st16(sAu, kBlk, i, c * 16 + 8, make_uint4(h[4], h[5], h[6], h[7]));
      }
      sA = sAu;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (i == 0) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        const uint32_t a = smem_u32(sA + ((h * L) >> 6) * kBlk + ((h * L) & 63) * 2);
        const uint32_t bb = smem_u32(sB + h * kDH * 128);
        if constexpr (U8) mma_tile_f16(tmem + h * kDH, a, kBlk, bb, kBlk, kDH, L, false);
        else mma_tile(tmem + h * kDH, a, kBlk, bb, kBlk, kDH, L, false);
      }
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
      if constexpr (U8) {
#pragma unroll
        for (int c = 0; c < kD; ++c) row[c] *= (1.0f / 255.0f);   // dequantise
      }
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

template <int L, bool U8>
int launch_score(int64_t B, const void* cache, int64_t n_items, const int32_t* ids,
                 const int64_t* off, int64_t total, const void* LP, void* O, unsigned* status,
                 cudaStream_t st) {
  using C = ScoreCfg<L, U8>;
  if (cudaFuncSetAttribute(k_score_tc<L, U8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM) != cudaSuccess)
    return LIME_ERR_CUDA;
  // enough (user, slot) CTAs to fill every SM a few times over, but at least
  // two tiles per CTA on average: a CTA overlaps its next tile's gather with
  // the current tile's MMA and epilogue, which one-tile CTAs in two waves of
  // residency cannot do
  const int64_t target = 4LL * num_sms();
  int64_t G = (target + B - 1) / B;
  const int64_t tiles_hi = (total + kTile - 1) / kTile;
  const int64_t two_per_cta = (tiles_hi / (B > 0 ? B : 1) + 1) / 2;
  if (G > two_per_cta) G = two_per_cta;
  if (G > tiles_hi) G = tiles_hi;
  if (G < 1) G = 1;
  if (G > 65535) G = 65535;
  dim3 grid((unsigned)B, (unsigned)G);
  return launch_pdl(k_score_tc<L, U8>, grid, dim3(128), C::SMEM, st, 1, cache, n_items, ids, off, B,
                    total, (const bf16*)LP, (bf16*)O, status);
}

}  // namespace

bool fast_score_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && (D.l == 16 || D.l == 32 || D.l == 64);
}

bool fast_score_u8_supported(const lime_dims& D) {
  return fast_score_supported(D) && D.H * D.l >= 128;
}

int fast_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
               const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
               float* ws, unsigned* status, cudaStream_t st) {
  (void)ws;
  switch (D.l) {
    case 16: return launch_score<16, false>(B, cache, n_items, ids, off, total, LP, O, status, st);
    case 32: return launch_score<32, false>(B, cache, n_items, ids, off, total, LP, O, status, st);
    default: return launch_score<64, false>(B, cache, n_items, ids, off, total, LP, O, status, st);
  }
}

int fast_score_u8(const lime_dims& D, int64_t B, const uint8_t* cache, int64_t n_items,
                  const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
                  unsigned* status, cudaStream_t st) {
  switch (D.l) {
    case 16: return launch_score<16, true>(B, cache, n_items, ids, off, total, LP, O, status, st);
    case 32: return launch_score<32, true>(B, cache, n_items, ids, off, total, LP, O, status, st);
    default: return launch_score<64, true>(B, cache, n_items, ids, off, total, LP, O, status, st);
  }
}

}  // namespace lime
