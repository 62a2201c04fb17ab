// bridge.cuh - KV Bridging: the KV cache of a Cross-Decoder full-attention
// layer built from the hidden states of the corresponding Self-Decoder layer,
// K = H W_K and V = H W_V, as one GEMM on the fifth-generation tensor cores.
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
// "Two-Level KV Sharing" (KV Bridging: each Full Attention layer of the
// Cross-Decoder builds its KV cache from the hidden states of the matching
// Full Attention layer of the Self-Decoder, so the cache is ready without
// running the layers in between).  The pages give neither the hidden size nor
// the weights: both are inputs here.
//
// A CTA computes a tile of 128 tokens x NT output columns of K or V.  Warp 4
// issues TMA loads of H [128 x 64] and W^T [NT x 64] per stage (128-byte
// swizzle) into a kBrStages-deep ring; warp 5 issues tcgen05.mma (M128 N NT
// K16, both operands K-major, fp32 accumulators in NT tensor-memory columns);
// warps 0-3 read the accumulators back (row = lane), round to bf16 and write
// the cache rows.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

constexpr int kBrRows = 128;   // tokens per tile = tensor-memory lanes
constexpr int kBrKC = 64;      // hidden elements per stage (one 128-byte swizzled row)
constexpr int kBrStages = 4;
constexpr int kBrThreads = 32 * 6;

template <int NT>
constexpr size_t bridge_smem() {
  return 1024 + (size_t)kBrStages * (kBrRows + NT) * kBrKC * 2;
}

struct BridgeArgs {
  int64_t rows;   // tokens (cache rows)
  int hidden;     // multiple of kBrKC
  int ncols;      // Hkv * D, multiple of NT
  bf16* K;        // [rows, ncols]
  bf16* V;
  int* err;
};

template <int NT>
__global__ void __launch_bounds__(kBrThreads, 1)
    k_kv_bridge(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmWk,
                const __grid_constant__ CUtensorMap tmWv, const __grid_constant__ BridgeArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  constexpr int kABytes = kBrRows * kBrKC * 2, kBBytes = NT * kBrKC * 2;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full[kBrStages], empty[kBrStages], acc_full;
  __shared__ uint32_t tmem_base_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per = a.ncols / NT;
  const bool is_v = (int)blockIdx.x >= tiles_per;
  const int n0 = ((int)blockIdx.x % tiles_per) * NT;
  const int64_t m0 = (int64_t)blockIdx.y * kBrRows;
  const int nk = a.hidden / kBrKC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBrStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, NT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 4) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      const CUtensorMap* wmap = is_v ? &tmWv : &tmWk;
      int f = 0;
      for (; f < nk && ok; ++f) {
        const int st = f % kBrStages;
        if (!(ok = mbar_wait(&empty[st], ((uint32_t)(f / kBrStages) & 1u) ^ 1u))) break;
        uint8_t* sa = base + st * (kABytes + kBBytes);
        mbar_arrive_expect_tx(&full[st], kABytes + kBBytes);
        tma_load_2d(sa, &tmH, &full[st], f * kBrKC, (int)m0);
        tma_load_2d(sa + kABytes, wmap, &full[st], f * kBrKC, n0);
      }
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
      // before the CTA exits: the fills issued have landed and their stages
      // have been released
      for (int g = f - kBrStages; g < f; ++g) {
        if (g < 0) continue;
        const uint32_t ph = (uint32_t)(g / kBrStages) & 1u;
        if (!mbar_wait(&full[g % kBrStages], ph)) record_error(a.err, HS2_ERR_TIMEOUT);
        if (ok && !mbar_wait(&empty[g % kBrStages], ph)) record_error(a.err, HS2_ERR_TIMEOUT);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBrRows, NT, 0, 0);
      bool ok = true;
      for (int f = 0; f < nk && ok; ++f) {
        const int st = f % kBrStages;
        if (!(ok = mbar_wait(&full[st], (uint32_t)(f / kBrStages) & 1u))) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(base + st * (kABytes + kBBytes));
#pragma unroll
        for (int kk = 0; kk < kBrKC / 16; ++kk)
          umma_ss(tmem, umma_desc_sw128(sa + kk * 32, 16, 1024), umma_desc_sw128(sa + kABytes + kk * 32, 16, 1024),
                  idesc, (f > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      umma_commit(&acc_full);
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    bool ok = mbar_wait(&acc_full, 0);
    if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const int row = warp * 32 + lane;
    const bool rv = m0 + row < a.rows;
    bf16* out = (is_v ? a.V : a.K) + (m0 + row) * (int64_t)a.ncols + n0;
#pragma unroll 1
    for (int ch = 0; ch < NT / 32 && ok; ++ch) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, r);
      tmem_wait_ld();
      if (rv) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(out + ch * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NT);
  }
}

}  // namespace hs2
