// common.cuh - shared device helpers of the hs2 kernels: problem geometry,
// error recording, the balanced key-range split and small block-level scans.
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "hs2.h"

namespace hs2 {

constexpr int kD = 128;  // head dimension the kernels are built for

typedef __nv_bfloat16 bf16;

// Records the first error code of a launch sequence into the device error word.
__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Index b in [0, n) of the last entry with off[b] <= x (off ascending, off[0] <= x).
__device__ __forceinline__ int last_le(const int64_t* off, int n, int64_t x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(off + mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Geometry of a query row: its sequence, its absolute position t and the
// start of its sequence in the packed KV arrays.
struct QueryRow {
  int b;
  int64_t t;
  int64_t kv_start;
  int64_t kv_len;
};

__device__ __forceinline__ QueryRow query_row(const int64_t* qoff, const int64_t* kvoff, int B,
                                              int64_t qi) {
  QueryRow r;
  r.b = last_le(qoff, B, qi);  // the last of equal offsets: empty sequences are skipped
  const int64_t q0 = __ldg(qoff + r.b), q1 = __ldg(qoff + r.b + 1);
  r.kv_start = __ldg(kvoff + r.b);
  r.kv_len = __ldg(kvoff + r.b + 1) - r.kv_start;
  r.t = r.kv_len - (q1 - q0) + (qi - q0);
  return r;
}

// query_row for a whole CTA (every thread calls it, with the same qi): the
// sequence is the number of b' in [1, B] with qoff[b'] <= qi (offsets
// ascending from qoff[0] = 0), at most B - 1, found with one load per thread
// and a barrier count instead of a binary search of dependent loads.  Falls
// back to query_row when B exceeds the CTA.
__device__ __forceinline__ QueryRow query_row_block(const int64_t* qoff, const int64_t* kvoff, int B,
                                                    int64_t qi) {
  if (B > (int)blockDim.x) return query_row(qoff, kvoff, B, qi);
  const int b1 = (int)threadIdx.x + 1;
  const int c = __syncthreads_count(b1 <= B && __ldg(qoff + b1) <= qi);
  QueryRow r;
  r.b = c < B ? c : B - 1;
  const int64_t q0 = __ldg(qoff + r.b), q1 = __ldg(qoff + r.b + 1);
  r.kv_start = __ldg(kvoff + r.b);
  r.kv_len = __ldg(kvoff + r.b + 1) - r.kv_start;
  r.t = r.kv_len - (q1 - q0) + (qi - q0);
  return r;
}

// floor(a / b) for 0 <= a < 2^53 and 0 < b < 2^31, by one fp64 division.  Exact:
// a non-integer quotient q (< 2^53 / b) lies at least 1/b below the next
// integer, more than the division's rounding error q * 2^-53.  (The keys and
// CTA counts here keep a below 2^48.)
__device__ __forceinline__ int64_t floor_div_f64(int64_t a, int64_t b) {
  return (int64_t)floor((double)a / (double)b);
}

// Balanced split of W keys over P CTAs: CTA p owns keys [W*p/P, W*(p+1)/P).
__device__ __forceinline__ int64_t split_lo(int64_t W, int P, int p) {
  return floor_div_f64(W * (int64_t)p, P);
}
// The CTA that owns key x (0 <= x < W): the largest p with split_lo(p) <= x,
// i.e. W p < (x + 1) P, p = floor(((x + 1) P - 1) / W), within [0, P - 1].
__device__ __forceinline__ int split_owner(int64_t W, int P, int64_t x) {
  const int64_t q = floor_div_f64((x + 1) * (int64_t)P - 1, W);
  return (int)(q < 0 ? 0 : (q > P - 1 ? P - 1 : q));
}

// Order-preserving 32-bit key of a float score: larger score -> larger key,
// -0.0 and +0.0 map to the same key.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one value per thread (blockDim.x <= 1024,
// multiple of 32).  ``sh`` needs blockDim.x/32 + 1 ints.  Returns the exclusive
// prefix; *total gets the block sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sh[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp ? sh[warp - 1] : 0) + x - v;
  *total = sh[nw - 1];
  __syncthreads();
  return before;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// exp(x - m) with exp(-inf) = 0 and a row that has seen nothing (m = -inf) kept at 0.
__device__ __forceinline__ float exp_shift(float x, float m) {
  return (x == -INFINITY) ? 0.f : expf(x - m);
}

}  // namespace hs2
