// Shared device helpers for liblime: element conversions, the sticky status
// word, and clamped access to jagged offsets.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lime.h"

namespace lime {

typedef __nv_bfloat16 bf16;

// Adds n to the process-wide count of kernels the library has launched.
void note_launches(int n);

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ void raise_flag(unsigned* status, unsigned f) {
  atomicOr(status, f);
}

// User u's row range [a, b) of a packed tensor with `total` rows, clamped so
// that garbage offsets never produce an out-of-bounds access.  A violated
// invariant (off[0] != 0, off[u] > off[u+1], off[B] != total) sets
// LIME_FLAG_BAD_OFFSETS.
__device__ __forceinline__ void user_range(const int64_t* off, int64_t u, int64_t B,
                                           int64_t total, int64_t* a, int64_t* b,
                                           unsigned* status) {
  int64_t x = off[u], y = off[u + 1];
  bool bad = (x > y) || (x < 0) || (y > total) || (u == 0 && x != 0) ||
             (u == B - 1 && y != total);
  if (bad) raise_flag(status, LIME_FLAG_BAD_OFFSETS);
  x = x < 0 ? 0 : (x > total ? total : x);
  y = y < x ? x : (y > total ? total : y);
  *a = x;
  *b = y;
}

// The user owning packed row r: the largest u with off[u] <= r, clamped to
// [0, B-1] (binary search over the B+1 offsets).
__device__ __forceinline__ int64_t owner_of(const int64_t* off, int64_t B, int64_t r) {
  int64_t lo = 0, hi = B;  // invariant: answer in [lo, hi)
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace lime
