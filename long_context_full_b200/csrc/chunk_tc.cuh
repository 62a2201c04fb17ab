// chunk_tc.cuh - Full Attention layer for a chunk of new query tokens (agent
// turns appended to a cached context), causal, on the fifth-generation tensor
// cores: tcgen05.mma with operands in shared memory (TMA, 128-byte swizzle) or
// tensor memory, accumulators in tensor memory.
//
// Source: "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
// Agents", sections "From Hybrid SWA to HySparse2 ..." (the full-attention layer
// builds the cache and judges token importance) and "Two-Level KV Sharing: ..."
// (prefill is dominated by large matrix products).
//
// A CTA owns 128 (query, head) rows: 128/G query tokens x the G query heads of
// one KV group, which share every K/V tile.  Two passes over the visible keys:
//   pass A (STATS): S = Q K^T per 128-key tile into tensor memory; the softmax
//                   warps keep each row's running max m and sum l.
//   pass B (OUT):   S = Q K^T again; P = exp(S - m) / l is exact (no online
//                   rescaling of O is ever needed); the selection scores (sum of
//                   P over the G heads of each query) are written; P goes back
//                   into tensor memory as bf16 and O += P V runs with A read
//                   from tensor memory.  O is final when the last tile is done.
// Roles: warps 0-7 softmax (warp w reads tensor-memory lanes 32(w%4).. + 31,
// one row per thread, and columns 64(w/4)..+63 of each tile), warp 8 TMA
// producer, warp 9 issues the MMAs (one thread).  Tensor memory: S double
// buffer at columns 0-255, O at 256-383, P (bf16) double buffer at 384-511.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"
#include "chunk_attn.cuh"

namespace hs2 {

constexpr int kTcRows = 128;                     // rows per CTA = tensor-memory lanes
constexpr int kTcKeys = 128;                     // keys per tile
constexpr int kTcStages = 2;                     // K/V ring depth
constexpr int kTcTileBytes = kTcKeys * kD * 2;   // a K or V tile: two swizzled [128][64] halves
constexpr int kTcQBytes = kTcRows * kD * 2;
constexpr int kTcSoftWarps = 8;   // two warpgroups: column halves of every tile
constexpr int kTcThreads = 32 * (kTcSoftWarps + 2);

template <bool OUT>
constexpr size_t chunk_tc_smem() {
  return 1024 + kTcQBytes + (size_t)kTcStages * (OUT ? 2 : 1) * kTcTileBytes;
}

template <bool OUT, int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_chunk_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ ChunkArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  constexpr int kStage = (OUT ? 2 : 1) * kTcTileBytes;
  constexpr uint32_t kCols = OUT ? 512 : 256;  // S double buffer (+ O and P)
  constexpr uint32_t kColO = 2 * kTcKeys, kColP = 3 * kTcKeys;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t kv_full[kTcStages], kv_empty[kTcStages];
  __shared__ __align__(8) uint64_t s_full[2], s_free[2], p_full[2];
  __shared__ __align__(8) uint64_t o_full;
  __shared__ uint32_t tmem_base_sh;

  ChTile c;
  if (!chunk_tile(a, c)) return;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sKV = base + kTcQBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int64_t nkeys = c.t0 + c.nq;  // keys [0, t_last] are visible to some row
  const int ntiles = (int)((nkeys + kTcKeys - 1) / kTcKeys);

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], OUT ? 1 : kTcSoftWarps);  // PV done (commit) / softmax warps read S
      mbar_init(&p_full[b], kTcSoftWarps);
    }
    mbar_init(&o_full, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kTcSoftWarps) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&q_full, kTcQBytes);
      tma_load_3d(sQ, &tmQ, &q_full, 0, g * G, (int)c.q0);
      tma_load_3d(sQ + kTcQBytes / 2, &tmQ, &q_full, 64, g * G, (int)c.q0);
      uint32_t issued = 0, last_phase = 0;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int st = j % kTcStages;
        const uint32_t ph = (uint32_t)(j / kTcStages) & 1u;
        if (!mbar_wait(&kv_empty[st], ph ^ 1u)) {
          record_error(a.err, HS2_ERR_TIMEOUT);
          ok = false;
          break;
        }
        uint8_t* sk = sKV + st * kStage;
        const int key = (int)(c.kv0 + (int64_t)j * kTcKeys);
        mbar_arrive_expect_tx(&kv_full[st], kStage);
        tma_load_3d(sk, &tmK, &kv_full[st], 0, g, key);
        tma_load_3d(sk + kTcTileBytes / 2, &tmK, &kv_full[st], 64, g, key);
        if (OUT) {
          tma_load_3d(sk + kTcTileBytes, &tmV, &kv_full[st], 0, g, key);
          tma_load_3d(sk + kTcTileBytes + kTcTileBytes / 2, &tmV, &kv_full[st], 64, g, key);
        }
        issued |= 1u << st;
        last_phase = (last_phase & ~(1u << st)) | (ph << st);
      }
      // before the CTA exits: every fill issued here has landed, and every
      // release of a stage (an MMA commit) has arrived
      if (!mbar_wait(&q_full, 0)) record_error(a.err, HS2_ERR_TIMEOUT);
      for (int s = 0; s < kTcStages; ++s)
        if ((issued >> s) & 1u) {
          if (!mbar_wait(&kv_full[s], (last_phase >> s) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
          if (ok && !mbar_wait(&kv_empty[s], (last_phase >> s) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
        }
    }
  } else if (warp == kTcSoftWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kTcRows, kTcKeys, 0, 0);  // Q K^T: both K-major
      constexpr uint32_t idesc_o = umma_idesc_bf16(kTcRows, kD, 0, 1);       // P V: V is MN-major
      bool ok = mbar_wait(&q_full, 0);
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
      tc_fence_after();
      const uint32_t qa = smem_u32(sQ);
      auto issue_s = [&](int j) -> bool {
        const int st = j % kTcStages, b = j & 1;
        if (!mbar_wait(&kv_full[st], (uint32_t)(j / kTcStages) & 1u)) return false;
        if (!mbar_wait(&s_free[b], ((uint32_t)(j >> 1) & 1u) ^ 1u)) return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(sKV + st * kStage);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32;
          umma_ss(tmem + b * kTcKeys, umma_desc_sw128(qa + off, 16, 1024),
                  umma_desc_sw128(kb + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&s_full[b]);
        if (!OUT) umma_commit(&kv_empty[st]);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int j = 0; j < ntiles && ok; ++j) {
        if (j + 1 < ntiles && !(ok = issue_s(j + 1))) break;
        if (OUT) {
          const int st = j % kTcStages, b = j & 1;
          if (!(ok = mbar_wait(&p_full[b], (uint32_t)(j >> 1) & 1u))) break;
          tc_fence_after();
          const uint32_t vb = smem_u32(sKV + st * kStage + kTcTileBytes);
#pragma unroll
          for (int kk = 0; kk < kTcKeys / 16; ++kk)
            umma_ts(tmem + kColO, tmem + kColP + b * (kTcKeys / 2) + kk * 8,
                    umma_desc_sw128(vb + kk * 2048, kTcTileBytes / 2, 1024), idesc_o,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&s_free[b]);
          umma_commit(&kv_empty[st]);
        }
      }
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
      if (OUT) {
        umma_commit(&o_full);
        // the commits that free the S buffers have arrived before the CTA exits
        for (int j = (ntiles > 2 ? ntiles - 2 : 0); ok && j < ntiles; ++j)
          if (!mbar_wait(&s_free[j & 1], (uint32_t)(j >> 1) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
      }
    }
  } else {
    // --------------------------------------------------------- softmax warps
    __shared__ float half_ml[2][kTcRows];  // STATS: the upper half's (m, l) per row
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int qr = row / G, hr = row % G;
    const bool rv = qr < c.nq;
    const int64_t t = c.t0 + qr;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t hrow = (c.q0 + qr) * a.Hq + (int64_t)g * G + hr;
    const int64_t t_min = c.t0;  // every row sees at least keys [0, t0]
    // Softmax in base 2: with c2 = scale * log2(e), exp(scale*s - m) = 2^(c2*s - m2)
    // where m2 = m * log2(e); the row statistics (m2, l) are kept in that form.
    // Pass B folds the normalisation into the exponent: P = 2^(c2*s - (m2 + log2 l)).
    const float c2 = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f, mb = 0.f;
    if (OUT && rv) {
      m = a.ml[hrow * 2];
      l = a.ml[hrow * 2 + 1];
      mb = m + log2f(l);  // l >= 1: the row's largest logit contributes 1
    }
    float* srow = a.scores + ((c.q0 + qr) * a.Hkv + g) * a.stride;
    const bool v4 = ((reinterpret_cast<uintptr_t>(a.scores) | ((uintptr_t)a.stride * 4)) & 15) == 0;
    // Every tcgen05.ld/st and full-mask shuffle below must be reached by the
    // whole warp: the branches around them use warp-uniform conditions only.
    const bool all_rv = __all_sync(0xffffffffu, rv);
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      if (ok && !mbar_wait(&s_full[b], (uint32_t)(j >> 1) & 1u)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) {
        // this warp's 64 keys of the tile: k0 .. k0+63
        const int64_t k0 = (int64_t)j * kTcKeys + half * 64;
        uint32_t r[2][32];
        tmem_ld32(trow + b * kTcKeys + half * 64, r[0]);
        tmem_ld32(trow + b * kTcKeys + half * 64 + 32, r[1]);
        tmem_wait_ld();
        auto S = [&](int i) { return __uint_as_float(r[i >> 5][i & 31]); };
        // MASKED: some key of the 64 lies past some row's position (or rows past the chunk)
        auto body = [&](auto masked_c) {
          constexpr bool MASKED = decltype(masked_c)::value;
          // keys k0 .. k0+nv-1 are visible to this row
          const int nv = MASKED ? (rv ? (int)max((int64_t)0, min((int64_t)64, t - k0 + 1)) : 0) : 64;
          auto valid = [nv](int i) { return !MASKED || i < nv; };
          if (!OUT) {
            float mx[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
#pragma unroll
            for (int i = 0; i < 64; ++i)
              mx[i & 7] = fmaxf(mx[i & 7], valid(i) ? S(i) : -INFINITY);
            const float cm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            if (cm != -INFINITY) {
              const float mn = fmaxf(m, cm * c2);
              float sm[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) sm[u] = 0.f;
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const float e = ex2_approx(fmaf(S(i), c2, -mn));
                sm[i & 7] += valid(i) ? e : 0.f;
              }
              l = l * ex2_approx(m - mn) +
                  (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
              m = mn;
            }
          } else {
            float p[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float e = ex2_approx(fmaf(S(i), c2, -mb));
              p[i] = valid(i) ? e : 0.f;
            }
            // P (bf16) into this tile's P buffer: 64 keys -> 32 packed columns
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(p[32 * cc + 2 * i], p[32 * cc + 2 * i + 1]);
              tmem_st16(trow + kColP + b * (kTcKeys / 2) + half * 32 + cc * 16, pk);
            }
            // scores: sum over the G rows of each query (consecutive lanes) by a
            // reduce-scatter butterfly on both 32-key chunks; each lane ends with
            // 32/G consecutive keys of each chunk, at offset ``off``
            int off = 0, n = 32;
#pragma unroll
            for (int msk = G / 2; msk >= 1; msk >>= 1) {
              const bool up = (lane & msk) != 0;
              n >>= 1;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                  if (i < n) {
                    float* q = p + 32 * cc;
                    const float send = up ? q[i] : q[i + n];
                    const float keep = up ? q[i + n] : q[i];
                    q[i] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
                  }
                }
              }
              if (up) off += n;
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int64_t kc = k0 + 32 * cc + off;
              if (!MASKED && v4) {
                float4* dst = reinterpret_cast<float4*>(srow + kc);
#pragma unroll
                for (int i = 0; i < 32 / G / 4; ++i)
                  dst[i] = make_float4(p[32 * cc + 4 * i], p[32 * cc + 4 * i + 1],
                                       p[32 * cc + 4 * i + 2], p[32 * cc + 4 * i + 3]);
              } else if (rv) {
#pragma unroll
                for (int i = 0; i < 32 / G; ++i)
                  if (kc + i <= t) srow[kc + i] = p[32 * cc + i];
              }
            }
          }
        };
        if (all_rv && k0 + 63 <= t_min) body(std::false_type{});
        else body(std::true_type{});
      }
      if (OUT) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(OUT ? &p_full[b] : &s_free[b]);
    }
    if (!OUT) {
      // merge the two column halves' running (m, l) of each row
      if (half == 1) {
        half_ml[0][row] = m;
        half_ml[1][row] = l;
      }
      named_barrier_sync(1, 32 * kTcSoftWarps);
      if (half == 0 && rv) {
        const float m2 = half_ml[0][row], l2 = half_ml[1][row];
        const float mm = fmaxf(m, m2);
        const float ll = (mm == -INFINITY) ? 0.f : l * ex2_approx(m - mm) + l2 * ex2_approx(m2 - mm);
        a.ml[hrow * 2] = mm;
        a.ml[hrow * 2 + 1] = ll;
      }
    } else {
      if (ok && !mbar_wait(&o_full, 0)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      bf16* O = static_cast<bf16*>(a.O);
#pragma unroll 1
      for (int cc = 0; cc < 2 && ok; ++cc) {
        const int ch = half * 2 + cc;
        uint32_t r[32];
        tmem_ld32(trow + kColO + ch * 32, r);
        tmem_wait_ld();
        if (rv) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(O + hrow * kD + ch * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

}  // namespace hs2
