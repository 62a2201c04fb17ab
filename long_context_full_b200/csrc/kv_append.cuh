// kv_append.cuh - writes the K/V rows of a step's new tokens into the shared
// KV cache of a Hybrid Block, at the positions the attention calls read them.
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
// "Two-Level KV Sharing" (the full-attention layer of a Hybrid Block produces
// the KV cache that its sparse layers reuse) and "Xiaomi Releases HySparse2,
// Targeting Long-Horizon Reasoning for Agents", section "From Hybrid SWA to
// HySparse2 ..." (decoding reads the cache a token at a time).  Positions
// follow the path's convention: query i of a sequence with cache length N and
// Tq new tokens sits at t = N - Tq + i, and its own key is cache row t.
//
// One warp per (new token, KV head), 16-byte loads and stores (bf16 rows of
// 256 bytes: lanes 0-15; fp32 rows of 512 bytes: all 32 lanes).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

constexpr int kAppendThreads = 256;

template <int ROW_BYTES>
__global__ void __launch_bounds__(kAppendThreads) k_kv_append(const uint8_t* Kn, const uint8_t* Vn,
                                                              uint8_t* K, uint8_t* V, const int64_t* qoff,
                                                              const int64_t* kvoff, int B, int Hkv,
                                                              int64_t total_q, int64_t total_kv, int* err) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int64_t w = ((int64_t)blockIdx.x * kAppendThreads + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (w >= total_q * Hkv) return;
  const int64_t qi = w / Hkv;
  const int g = (int)(w % Hkv);
  const QueryRow q = query_row(qoff, kvoff, B, qi);
  const int64_t row = q.kv_start + q.t;  // the token's own cache row
  if (q.t < 0 || q.kv_start < 0 || row >= total_kv) {
    if (lane == 0) record_error(err, HS2_ERR_DEVICE_INPUT);
    return;
  }
  const int64_t src = (qi * Hkv + g) * (int64_t)ROW_BYTES;
  const int64_t dst = (row * Hkv + g) * (int64_t)ROW_BYTES;
  // 16-byte pieces: lane l copies bytes 16l, 16l + 512, ... of the row
#pragma unroll
  for (int off = lane * 16; off < ROW_BYTES; off += 32 * 16) {
    const uint4 k = __ldg(reinterpret_cast<const uint4*>(Kn + src + off));
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(Vn + src + off));
    *reinterpret_cast<uint4*>(K + dst + off) = k;
    *reinterpret_cast<uint4*>(V + dst + off) = x;
  }
}

}  // namespace hs2
