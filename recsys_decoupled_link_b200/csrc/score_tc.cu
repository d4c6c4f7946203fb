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

struct ScoreTile {
  int64_t p;   // first packed position
  int n;       // candidates (1 .. 128)
  int64_t u;   // user, or -1 when no valid user range holds position p
};

// The tile starting at packed position p of a range ending at r1: the user
// holding p (the last u with off[u] <= p, by binary search) and its rows up to
// 128, the user's end or the range's end.  Offsets that do not give p a valid
// owner yield u = -1 (zero rows) for up to 128 positions.
__device__ __forceinline__ ScoreTile score_tile_at(int64_t p, int64_t r1, const int64_t* off,
                                                   int64_t B, int64_t total) {
  ScoreTile t;
  t.p = p;
  const int64_t u = owner_of(off, B, p);
  int64_t a = off[u], b = off[u + 1];
  a = a < 0 ? 0 : a;
  b = b > total ? total : b;
  int64_t e = p + kTile < r1 ? p + kTile : r1;
  if (a <= p && p < b) {
    t.u = u;
    e = e < b ? e : b;
  } else {
    t.u = -1;
  }
  t.n = (int)(e - p);
  return t;
}

// ------------------------------------------------ cached scoring, bf16 cache
// k_score_ws<L>: one persistent CTA per SM with warp-specialised roles and a
// flat, balanced schedule.  The packed candidate positions [0, total) are cut
// into one contiguous range per CTA (a multiple of 128 positions); inside its
// range a CTA walks tiles of at most 128 candidates that never cross a user
// boundary (a user's last tile in the range may be partial).  Every role
// derives the same tile sequence from the offsets on its own, so nothing but
// the barriers passes between them.
//   warps 0-3  producers: a tile's candidate IDs (validated: a bad ID gives a
//              zero row and LIME_FLAG_BAD_ID) and its row gather with 16-byte
//              asynchronous copies (a warp's copies cover whole rows) into a
//              ring of NS stages, in the swizzled K-major operand layout; the
//              hardware arrives on the stage's barrier for each producer once
//              that thread's copies have landed, so up to NS tiles are in
//              flight and no stage waits for later progress.  On every change of user
//              they stage L^P_u transposed ([128 c x 64 k] bf16, k >= l zero)
//              into one of two B slots.
//   warp 4     one lane issues, per tile and head, the [128 x l] x [l x 32]
//              product into one of two TMEM accumulators.
//   warps 5-8  epilogue: TMEM -> bf16 -> a swizzled staging tile -> coalesced
//              16-byte stores of the tile's rows.
// The gather ring holds about 128 KB (NS = 8, 4, 2 tiles for l = 16, 32, 64),
// which keeps an SM's share of the HBM bandwidth in flight at every l.
template <int L>
struct WsCfg {
  static constexpr int HL = kH * L;
  static constexpr int ABLK = HL / 64 < 1 ? 1 : HL / 64;   // 64-column blocks of a gathered tile
  static constexpr uint32_t kStage = ABLK * kBlk;           // = 128 rows x 2*HL bytes
  static constexpr int NS = L == 16 ? 8 : (L == 32 ? 4 : 2);
  static constexpr int RB = 2 * HL;                         // bytes per cache row
  static constexpr int CH = RB / 16;                        // 16-byte chunks per row
  static constexpr uint32_t OFF_OUT = NS * kStage;          // [128 x 128] bf16 output staging
  static constexpr uint32_t OFF_B = OFF_OUT + 2 * kBlk;     // two B slots, one block each
  static constexpr uint32_t OFF_T = OFF_B + 2 * kBlk;       // L^P_u row-major [L x 128] bf16
  static constexpr uint32_t OFF_IDS = OFF_T + L * kD * 2;   // [NS][128] int64 candidate IDs
  static constexpr uint32_t OFF_BAR = OFF_IDS + NS * 128 * 8;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static constexpr int THREADS = 288;
};

template <int L>
__global__ void __launch_bounds__(WsCfg<L>::THREADS, 1)
    k_score_ws(const bf16* __restrict__ cache, int64_t n_items, const int32_t* __restrict__ ids,
               const int64_t* __restrict__ off, int64_t B, int64_t total, int64_t span,
               const bf16* __restrict__ LP, bf16* __restrict__ O, unsigned* status) {
  using C = WsCfg<L>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sOut = sm + C::OFF_OUT;
  uint8_t* sBs = sm + C::OFF_B;
  bf16* sT = reinterpret_cast<bf16*>(sm + C::OFF_T);
  int64_t* s_ids = reinterpret_cast<int64_t*>(sm + C::OFF_IDS);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* empty = full + NS;
  uint64_t* bready = empty + NS;    // [2] B slot staged (128 producer arrivals)
  uint64_t* bfree = bready + 2;     // [2] B slot's last MMA done (commit)
  uint64_t* tfull = bfree + 2;      // [2] accumulator ready (commit)
  uint64_t* tempty = tfull + 2;     // [2] accumulator read (128 epilogue arrivals)
  uint64_t* mdone = tempty + 2;
  uint32_t* slot = reinterpret_cast<uint32_t*>(mdone + 1);
  int* abort_flag = reinterpret_cast<int*>(mdone + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int q = 0; q < NS; ++q) {
      mbar_init(&full[q], 128);
      mbar_init(&empty[q], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bready[q], 128);
      mbar_init(&bfree[q], 1);
      mbar_init(&tfull[q], 1);
      mbar_init(&tempty[q], 128);
    }
    mbar_init(mdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) tmem_alloc(slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  pdl_launch();
  pdl_wait();
  const int64_t r0 = (int64_t)blockIdx.x * span;
  const int64_t r1 = r0 + span < total ? r0 + span : total;

  if (warp < 4) {
    // ---- producers (128 threads, i = tid)
    const int i = tid;
    if (blockIdx.x == 0) {
      // the offsets as a whole: monotone, from 0 to total
      for (int64_t u = i; u < B; u += 128) {
        const int64_t x = off[u], y = off[u + 1];
        if (x > y || x < 0 || y > total || (u == 0 && x != 0) || (u == B - 1 && y != total))
          raise_flag(status, LIME_FLAG_BAD_OFFSETS);
      }
    }
    int64_t p = r0, cur_u = -1;
    int k = 0, nsw = 0;
    while (p < r1) {
      const ScoreTile t = score_tile_at(p, r1, off, B, total);
      const int s = k % NS;
      if (k >= NS && !mbar_wait(&empty[s], (uint32_t)((k / NS) - 1) & 1u, status, abort_flag)) break;
      if (t.u >= 0 && t.u != cur_u) {
        // L^P_u transposed into B slot nsw % 2, once the MMAs of the user
        // that held it before (user nsw - 2) are done
        if (nsw >= 2 && !mbar_wait(&bfree[nsw & 1], (uint32_t)((nsw - 2) >> 1) & 1u, status,
                                   abort_flag))
          break;
        const uint4* src = reinterpret_cast<const uint4*>(LP + t.u * L * kD);
#pragma unroll
        for (int q = 0; q < L * kD / 8 / 128; ++q)
          reinterpret_cast<uint4*>(sT)[q * 128 + i] = __ldg(src + q * 128 + i);
        named_bar_sync(1, 128);
        uint8_t* sB = sBs + (nsw & 1) * kBlk;
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          float f[8];
#pragma unroll
          for (int z = 0; z < 8; ++z) {
            const int kk = k8 * 8 + z;
            f[z] = kk < L ? __bfloat162float(sT[kk * kD + i]) : 0.f;
          }
          sw_st16(sB, kBlk, i, k8 * 8, pack8(f));
        }
        fence_proxy_async_smem();
        mbar_arrive(&bready[nsw & 1]);
        cur_u = t.u;
        ++nsw;
      }
      int64_t id = -1;
      if (t.u >= 0 && i < t.n) {
        id = (int64_t)ids[t.p + i];
        if (id < 0 || id >= n_items) {
          raise_flag(status, LIME_FLAG_BAD_ID);
          id = -1;
        }
      }
      if (t.u < 0 && i == 0) raise_flag(status, LIME_FLAG_BAD_OFFSETS);
      s_ids[s * kTile + i] = id;
      named_bar_sync(1, 128);
      // chunk q*128 + i is chunk (idx % CH) of row idx / CH: a warp reads whole rows
      uint8_t* sA = sm + s * C::kStage;
#pragma unroll
      for (int q = 0; q < C::CH; ++q) {
        const int idx = q * 128 + i, r = idx / C::CH, cc = idx % C::CH;
        const int64_t rid = s_ids[s * kTile + r];
        const bf16* srow = cache + (rid < 0 ? 0 : rid * C::HL) + cc * 8;
        cp_async16(sA + (cc >> 3) * kBlk + sw128_offset(r, (cc & 7) * 8), srow, rid >= 0);
      }
      // the stage is full once every producer's copies have landed (the
      // hardware arrives for this thread; no later progress is needed)
      cp_async_arrive_noinc(&full[s]);
      p += t.n;
      ++k;
    }
    cp_async_wait_all();   // nothing of ours is in flight when the CTA exits
  } else if (warp == 4) {
    // ---- MMA issuer (one lane)
    if (lane == 0) {
      int64_t p = r0, cur_u = -1;
      int k = 0, nsw = 0, bs = 0;
      bool ok = true;
      while (p < r1 && ok) {
        const ScoreTile t = score_tile_at(p, r1, off, B, total);
        const int s = k % NS, acc = k & 1;
        if (!(ok = mbar_wait(&full[s], (uint32_t)(k / NS) & 1u, status, abort_flag))) break;
        if (t.u >= 0 && t.u != cur_u) {
          if (nsw >= 1) mma_commit(&bfree[(nsw - 1) & 1]);   // the previous user's slot
          if (!(ok = mbar_wait(&bready[nsw & 1], (uint32_t)(nsw >> 1) & 1u, status, abort_flag)))
            break;
          bs = nsw & 1;
          cur_u = t.u;
          ++nsw;
        }
        if (k >= 2 && !(ok = mbar_wait(&tempty[acc], (uint32_t)((k >> 1) - 1) & 1u, status,
                                       abort_flag)))
          break;
        fence_proxy_async_smem();   // the gathered rows (generic-proxy copies) -> the MMA
        tc_fence_after();
        if (t.u >= 0) {
          const uint8_t* sA = sm + s * C::kStage;
#pragma unroll
          for (int h = 0; h < kH; ++h)
            mma_tile(tmem + acc * 128 + h * kDH,
                     smem_u32(sA + ((h * L) >> 6) * kBlk + ((h * L) & 63) * 2), kBlk,
                     smem_u32(sBs + bs * kBlk + h * kDH * 128), kBlk, kDH, L, false);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[acc]);
        p += t.n;
        ++k;
      }
      // drain: no MMA of ours may be in flight when TMEM is freed
      mma_commit(mdone);
      mbar_wait(mdone, 0, status, abort_flag);
    }
  } else {
    // ---- epilogue (128 threads): row = TMEM lane of this warp's quadrant
    const int e = tid - 160;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    int64_t p = r0;
    int k = 0;
    while (p < r1) {
      const ScoreTile t = score_tile_at(p, r1, off, B, total);
      const int acc = k & 1;
      if (!mbar_wait(&tfull[acc], (uint32_t)(k >> 1) & 1u, status, abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float v[64];
        if (t.u >= 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld16(ta + acc * 128 + hh * 64 + q * 16, v + q * 16);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) v[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) sw_st16(sOut, kBlk, row, hh * 64 + c * 8, pack8(v + c * 8));
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      named_bar_sync(2, 128);   // the staging tile is complete
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int idx = q * 128 + e, r = idx >> 4, cc = idx & 15;
        if (r < t.n)
          reinterpret_cast<uint4*>(O + (t.p + r) * kD)[cc] = sw_ld16(sOut, kBlk, r, cc * 8);
      }
      named_bar_sync(2, 128);   // every thread has read the staging tile
      p += t.n;
      ++k;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int L>
int launch_score_ws(int64_t B, const void* cache, int64_t n_items, const int32_t* ids,
                    const int64_t* off, int64_t total, const void* LP, void* O, unsigned* status,
                    cudaStream_t st) {
  using C = WsCfg<L>;
  if (cudaFuncSetAttribute(k_score_ws<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return LIME_ERR_CUDA;
  // one CTA per SM, each a contiguous range of a whole number of 128-position
  // tiles (users split across ranges freely)
  const int64_t tiles = (total + kTile - 1) / kTile;
  int64_t G = num_sms();
  if (G > tiles) G = tiles;
  if (G < 1) G = 1;
  const int64_t span = ((tiles + G - 1) / G) * kTile;
  G = (total + span - 1) / span;
  return launch_pdl(k_score_ws<L>, dim3((unsigned)G), dim3(C::THREADS), C::SMEM, st, 1,
                    (const bf16*)cache, n_items, ids, off, B, total, span, (const bf16*)LP,
                    (bf16*)O, status);
}

}  // namespace

bool fast_score_supported(const lime_dims& D) {
  return D.dtype == LIME_BF16 && D.d == kD && D.H == kH && (D.l == 16 || D.l == 32 || D.l == 64);
}

bool fast_score_u8_supported(const lime_dims& D) {
  return fast_score_supported(D) && D.H * D.l >= 64;
}

int fast_score(const lime_dims& D, int64_t B, const void* cache, int64_t n_items,
               const int32_t* ids, const int64_t* off, int64_t total, const void* LP, void* O,
               float* ws, unsigned* status, cudaStream_t st) {
  (void)ws;
  switch (D.l) {
    // l <= 32: (user, slot) CTAs of 128 threads that gather, multiply and store
    // in turn; l = 64 (one CTA per SM either way): the warp-specialised kernel
    case 16: return launch_score<16, false>(B, cache, n_items, ids, off, total, LP, O, status, st);
    case 32: return launch_score<32, false>(B, cache, n_items, ids, off, total, LP, O, status, st);
    default: return launch_score_ws<64>(B, cache, n_items, ids, off, total, LP, O, status, st);
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
