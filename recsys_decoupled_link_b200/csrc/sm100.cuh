// Thin wrappers over the sm_100a instructions the tensor-core kernels use:
// mbarriers with bounded waits, TMA tile loads/stores, bulk copies, tcgen05
// MMA / TMEM allocation / TMEM loads, and the shared-memory matrix
// descriptors of the 128-byte-swizzled K-major layout.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lime_common.cuh"

namespace lime {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// ------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that suspends for at most about `ns` nanoseconds (a hint), for
// a thread that polls two barriers in turn.
__device__ __forceinline__ bool mbar_try_wait_ns(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase of `bar` with the given parity to complete.  try_wait
// suspends the thread in hardware until the phase completes or a short
// system time limit passes, so the loop needs no sleep of its own (a software
// sleep would add its wake-up delay to every producer -> consumer hand-off).
// The wait is bounded by the global timer (two seconds); on expiry it sets
// LIME_FLAG_TIMEOUT in the status word, raises the CTA's abort flag and
// returns false.  A raised abort flag ends every later wait of the CTA.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* status,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > 2000000000ull) break;
  }
  raise_flag(status, LIME_FLAG_TIMEOUT);
  *abort_flag = 1;
  return false;
}

// Programmatic dependent launch.  Kernels launched with launch_pdl call
// pdl_launch once their TMEM is allocated (so that the next kernel's CTAs,
// which may allocate TMEM before they wait, cannot take it first) and
// pdl_wait before their first global-memory access: the previous kernel in
// the stream has then completed and its writes are visible.
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Makes this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA stores, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x,
                                             int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   (uint64_t)map),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}

// L2 prefetch of one tensor-map box (no shared memory, no barrier; parts of
// the box outside the tensor are ignored).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   (uint64_t)map),
               "r"(x), "r"(y)
               : "memory");
}

// 1-D bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Asynchronous 16-byte copy global -> shared (LDGSTS); with valid == false
// nothing is read and the 16 bytes are zero-filled.  Tracked per thread by
// cp_async_commit / cp_async_wait; the data is written through the generic
// proxy (fence before a tensor-core read).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Arrive-on `bar` (without incrementing its pending count) once every
// cp.async this thread has issued so far has landed: the barrier's expected
// count must include one such arrival per producing thread and phase.  The
// copies are generic-proxy writes: a consumer that reads them through the
// async proxy fences (fence_proxy_async_smem) after its wait.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Bulk prefetch of global memory into L2 (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 1-D bulk copy shared -> global (both 16-byte aligned, bytes % 16 == 0),
// tracked by the issuing thread's bulk group (bulk_commit / bulk_wait*).
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(dst), "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ---------------------------------------------------------------- tcgen05

// Allocates `ncols` TMEM columns (power of two >= 32); whole warp executes.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor: fp16 x fp16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory descriptor of a K-major operand stored as 128-byte-swizzled
// 8-row x 128-byte atoms (rows 128 bytes apart, 8-row groups 1024 bytes
// apart).  `addr` is the byte address of the first row's current K slice; a
// K step of 16 bf16 elements advances it by 32 bytes inside the atom.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Byte offset of element (row, col) inside one [rows x 64] bf16 block stored
// in the 128-byte-swizzled layout (block base 1024-byte aligned).
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 3) ^ (row & 7u)) & 7u) << 4) + ((col & 7u) << 1);
}

// tcgen05.ld of 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

}  // namespace sm100

// Host: encode a 2-D bf16 tensor map (inner dim `inner` elements, `outer`
// rows, row pitch `pitch_bytes`) with a box of box_inner x box_outer and
// 128-byte swizzle.  Returns false if the driver rejects it.
bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// Host: the same for a 2-D fp16 tensor (128-byte swizzle; box_inner <= 64).
bool make_tmap_2d_f16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// Host: the same for a 2-D uint8 tensor (128-byte swizzle; box_inner <= 128).
bool make_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// Host: a 2-D uint8 tensor without swizzle (row-major staging; box_inner a
// multiple of 16).
bool make_tmap_2d_u8_plain(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                           uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);
// Host: the same for a 2-D fp32 tensor (128-byte swizzle; box_inner <= 32).
bool make_tmap_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer);

// Host: number of SMs of the current device (cached per device).
int num_sms();

}  // namespace lime

namespace lime {
namespace sm100 {

// tcgen05.st of 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Issues the MMAs of one 128-row tile: D[128 x N] (+)= A[128 x K] * B[N x K]^T.
// A and B are K-major 128-byte-swizzled operands split into blocks of 64 K
// columns; a_blk / b_blk are the byte strides between those blocks and
// a_base / b_base may point into a block at a 32-byte multiple (a K slice).
__device__ __forceinline__ void mma_tile(uint32_t d_tmem, uint32_t a_base, uint32_t a_blk,
                                         uint32_t b_base, uint32_t b_blk, int N, int K,
                                         bool accumulate) {
  const uint32_t idesc = idesc_bf16(128, N);
  for (int k = 0; k < K / 16; ++k) {
    const uint32_t off = (uint32_t)(k & 3) * 32;
    mma_bf16(d_tmem, sdesc_sw128(a_base + (k >> 2) * a_blk + off),
             sdesc_sw128(b_base + (k >> 2) * b_blk + off), idesc, accumulate || k > 0);
  }
}

// mma_tile with fp16 operands (both A and B fp16).
__device__ __forceinline__ void mma_tile_f16(uint32_t d_tmem, uint32_t a_base, uint32_t a_blk,
                                             uint32_t b_base, uint32_t b_blk, int N, int K,
                                             bool accumulate) {
  const uint32_t idesc = idesc_f16(128, N);
  for (int k = 0; k < K / 16; ++k) {
    const uint32_t off = (uint32_t)(k & 3) * 32;
    mma_bf16(d_tmem, sdesc_sw128(a_base + (k >> 2) * a_blk + off),
             sdesc_sw128(b_base + (k >> 2) * b_blk + off), idesc, accumulate || k > 0);
  }
}

// Thread 0 commits the MMAs it issued to `bar`; every thread of the CTA then
// waits for them (bounded) and flips its phase bit.
__device__ __forceinline__ void cta_mma_wait(uint64_t* bar, uint32_t& phase, unsigned* status,
                                             volatile int* abort_flag) {
  if (threadIdx.x == 0) mma_commit(bar);
  mbar_wait(bar, phase, status, abort_flag);
  phase ^= 1u;
  tc_fence_after();
}

// Reads 8 bf16 (16 bytes) of row `row`, columns [c8*8, c8*8+8), of a K-major
// swizzled [rows x (64*nblk)] operand whose blocks are `blk` bytes apart.
__device__ __forceinline__ uint4 sw_ld16(const uint8_t* base, uint32_t blk, int row, int col) {
  return *reinterpret_cast<const uint4*>(base + (col >> 6) * blk + sw128_offset(row, col & 63));
}
__device__ __forceinline__ void sw_st16(uint8_t* base, uint32_t blk, int row, int col, uint4 v) {
  *reinterpret_cast<uint4*>(base + (col >> 6) * blk + sw128_offset(row, col & 63)) = v;
}

__device__ __forceinline__ void unpack8(uint4 v, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 v;
  v.x = pack_bf16(f[0], f[1]);
  v.y = pack_bf16(f[2], f[3]);
  v.z = pack_bf16(f[4], f[5]);
  v.w = pack_bf16(f[6], f[7]);
  return v;
}

}  // namespace sm100
}  // namespace lime

namespace lime {
namespace sm100 {

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled
// layout: each K row holds 64 MN elements in 128 bytes, 8 K rows form a
// 1024-byte atom (stride between 8-row groups 1024 bytes), and consecutive
// 64-wide MN blocks are `lbo` bytes apart.  This is the byte image of a
// row-major [K x MN] tile stored as [rows x 64] swizzled blocks; a K step of
// 16 rows advances the start address by 2048 bytes.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t addr, uint32_t lbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// D[128 x N] (+)= A[128 x K] (K-major) * B where B is stored MN-major as a
// row-major [K x N] tile (blocks of 64 N columns `b_lbo` bytes apart).
__device__ __forceinline__ void mma_tile_bmn(uint32_t d_tmem, uint32_t a_base, uint32_t a_blk,
                                             uint32_t b_base, uint32_t b_lbo, int N, int K,
                                             bool accumulate) {
  const uint32_t idesc = idesc_bf16(128, N) | (1u << 16);   // B is MN-major
  for (int k = 0; k < K / 16; ++k) {
    const uint32_t off = (uint32_t)(k & 3) * 32;
    mma_bf16(d_tmem, sdesc_sw128(a_base + (k >> 2) * a_blk + off),
             sdesc_sw128_mn(b_base + (uint32_t)k * 2048, b_lbo), idesc, accumulate || k > 0);
  }
}

// ------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
// Bulk copy from this CTA's shared memory to another CTA's (dst and mbar are
// cluster addresses from cluster_map); completes `bytes` on that CTA's
// mbarrier.  Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_push_cluster(uint32_t dst, const void* src, uint32_t bytes,
                                                  uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "r"(smem_u32(src)), "r"(bytes), "r"(mbar)
      : "memory");
}
// Every thread of every CTA of the cluster: release this CTA's shared-memory
// writes and acquire the others'.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// The two halves of cluster_sync, for overlapping the barrier with work that
// neither needs the other CTAs nor is needed by them.  Every thread calls
// them alternately (arrive, wait, arrive, wait, ...), converged per warp.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Cooperative, coalesced store of the first `nv` rows of a [128 x 128] bf16
// tile held in the swizzled layout (2 blocks of [128 x 64]) to row-major
// global rows (any multiple of 32 threads; a warp writes two whole 256-byte
// rows per step).
__device__ __forceinline__ void tile_store_rows(const uint8_t* tile, bf16* dst, int nv) {
#pragma unroll 4
  for (int idx = (int)threadIdx.x; idx < 2048; idx += (int)blockDim.x) {
    const int r = idx >> 4, cc = idx & 15;
    if (r < nv) reinterpret_cast<uint4*>(dst + (int64_t)r * 128)[cc] = sw_ld16(tile, 128 * 128, r, cc * 8);
  }
}

// 8 fp16 -> 8 floats (exact).
__device__ __forceinline__ void unpack8_f16(uint4 v, float* f) {
  const __half2* p = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// 8 floats -> 8 fp16 (round to nearest even).
__device__ __forceinline__ uint4 pack8_f16(const float* f) {
  uint4 v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2 h = __floats2half2_rn(f[2 * j], f[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return v;
}

}  // namespace sm100
}  // namespace lime
