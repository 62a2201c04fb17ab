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
// A CTA owns two Q tiles of 128 (query, head) rows each: 128/G query tokens x
// the G query heads of one KV group per tile, 256/G consecutive queries in all.
// Every K/V tile it loads feeds both Q tiles.  One kernel, two passes over the
// visible keys:
//   pass A: S_t = Q_t K^T per 128-key tile into tensor memory (four S buffers:
//           two per Q tile); softmax warpgroup t keeps each row's running max
//           and sum, in registers.
//   pass B: S_t = Q_t K^T again; P = exp(S - m) / l is exact, so O never needs
//           rescaling; the selection scores (sum of P over the G heads of each
//           query) are written; P goes back into the S columns as bf16 (two
//           keys per column, written behind the columns already read) and
//           O_t += P V runs with A read from tensor memory.
// Roles: warpgroup t (warps 4t .. 4t+3) does the softmax of Q tile t, one row
// per thread (warp w reads tensor-memory lanes 32(w%4) .. +31); warp 8 issues
// the TMA loads (Q once; K and V through separate rings of two and three
// stages); warp 9
// issues the MMAs from one thread.  Tensor memory (512 columns): pass A, the S
// buffers (tile t, buffer b) at 256t + 128b; pass B, S_t/P_t at 128t and O_t
// at 256 + 128t.  S_t of the next key tile is issued right after the
// O_t += P_t V that reads P_t: tcgen05.mma from one thread execute in order.
//
// Key split (a.ksplit > 1): the query tiles alone leave the last wave of CTAs
// part-empty (256 tiles on 148 SMs run in 2 waves, the second 73 % full), so
// the visible key tiles are cut into ksplit contiguous ranges, one CTA each,
// in two launches: mode 1 runs pass A over its range and writes each row's
// (max, sum); mode 2 merges the ranges' (max, sum) into the row's exact
// statistics, runs pass B over its range (P is then exact, so the scores of its
// keys are final and its share of O needs no rescaling) and writes that share
// in float32; k_chunk_o_sum adds the shares in a fixed order.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"
#include "chunk_attn.cuh"

namespace hs2 {

constexpr int kTcRows = 128;                     // rows per Q tile = tensor-memory lanes
constexpr int kTcQTiles = 2;                     // Q tiles per CTA
constexpr int kTcKeys = 128;                     // keys per K/V tile
constexpr int kTcKStages = 2;                    // depth of the K ring
constexpr int kTcVStages = 3;                    // depth of the V ring (V is needed later than K)
constexpr int kTcTileBytes = kTcKeys * kD * 2;   // a K or V tile: two swizzled [128][64] halves
constexpr int kTcQBytes = kTcRows * kD * 2;      // one Q tile
constexpr int kTcThreads = 32 * 10;              // 2 softmax warpgroups, TMA warp, MMA warp

constexpr size_t chunk_tc_smem() {
  return 1024 + (size_t)kTcQTiles * kTcQBytes + (size_t)(kTcKStages + kTcVStages) * kTcTileBytes;
}

template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_chunk_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ ChunkArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  constexpr int QT1 = kTcRows / G;  // queries per Q tile
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t k_full[kTcKStages], k_empty[kTcKStages];
  __shared__ __align__(8) uint64_t v_full[kTcVStages], v_empty[kTcVStages];
  __shared__ __align__(8) uint64_t sa_full[2][2], sa_free[2][2];  // pass A: [Q tile][S buffer]
  __shared__ __align__(8) uint64_t sb_full[2], pb_full[2], o_full;  // pass B: [Q tile]
  __shared__ uint32_t tmem_base_sh;

  const int ks = a.ksplit > 0 ? a.ksplit : 1;
  const int split = (int)blockIdx.z % ks;
  ChTile c;
  if (!chunk_tile(a, (int)blockIdx.z / ks, c)) return;
  const bool doA = a.mode != 2, doB = a.mode != 1;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = base + kTcQTiles * kTcQBytes;
  uint8_t* sV = sK + kTcKStages * kTcTileBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int64_t nkeys = c.t0 + c.nq;  // keys [0, t_last] are visible to some row
  const int ntot = (int)((nkeys + kTcKeys - 1) / kTcKeys);
  // this CTA's key tiles [j0, j0 + n)
  const int j0 = (int)((int64_t)ntot * split / ks);
  const int n = (int)((int64_t)ntot * (split + 1) / ks) - j0;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kTcKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kTcVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sa_full[t][b], 1);
        mbar_init(&sa_free[t][b], 4);  // the four warps of warpgroup t
      }
      mbar_init(&sb_full[t], 1);
      mbar_init(&pb_full[t], 4);
    }
    mbar_init(&o_full, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&q_full, kTcQTiles * kTcQBytes);
      for (int t = 0; t < kTcQTiles; ++t) {
        tma_load_3d(sQ + t * kTcQBytes, &tmQ, &q_full, 0, g * G, (int)(c.q0 + t * QT1));
        tma_load_3d(sQ + t * kTcQBytes + kTcQBytes / 2, &tmQ, &q_full, 64, g * G, (int)(c.q0 + t * QT1));
      }
      const uint64_t keep = policy_evict_last();
      // K fills 0 .. 2n-1 (pass A tiles, then pass B tiles); V fills 0 .. n-1
      auto fill = [&](uint64_t* full, uint64_t* empty, uint8_t* ring, int nst, const CUtensorMap* map,
                      int f, int j) -> bool {
        const int st = f % nst;
        if (!mbar_wait(&empty[st], ((uint32_t)(f / nst) & 1u) ^ 1u)) return false;
        const int key = (int)(c.kv0 + (int64_t)j * kTcKeys);
        uint8_t* dst = ring + st * kTcTileBytes;
        mbar_arrive_expect_tx(&full[st], kTcTileBytes);
        // every CTA of the KV group reads this tile, twice for K: keep it in L2
        tma_load_3d_hint(dst, map, &full[st], 0, g, key, keep);
        tma_load_3d_hint(dst + kTcTileBytes / 2, map, &full[st], 64, g, key, keep);
        return true;
      };
      int kf = 0, vf = 0;
      for (int j = 0; j < n && ok && doA; ++j) {
        if ((ok = fill(k_full, k_empty, sK, kTcKStages, &tmK, kf, j0 + j))) ++kf;
      }
      for (int j = 0; j < n && ok && doB; ++j) {
        if (!(ok = fill(k_full, k_empty, sK, kTcKStages, &tmK, kf, j0 + j))) break;
        ++kf;
        if (!(ok = fill(v_full, v_empty, sV, kTcVStages, &tmV, vf, j0 + j))) break;
        ++vf;
      }
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
      // before the CTA exits: every fill issued here has landed, and every
      // release of a stage (an MMA commit) has arrived
      if (!mbar_wait(&q_full, 0)) record_error(a.err, HS2_ERR_TIMEOUT);
      auto drain = [&](uint64_t* full, uint64_t* empty, int nst, int nf) {
        for (int f = nf - nst; f < nf; ++f) {
          if (f < 0) continue;
          const uint32_t ph = (uint32_t)(f / nst) & 1u;
          if (!mbar_wait(&full[f % nst], ph)) record_error(a.err, HS2_ERR_TIMEOUT);
          if (ok && !mbar_wait(&empty[f % nst], ph)) record_error(a.err, HS2_ERR_TIMEOUT);
        }
      };
      drain(k_full, k_empty, kTcKStages, kf);
      drain(v_full, v_empty, kTcVStages, vf);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kTcRows, kTcKeys, 0, 0);  // Q K^T: both K-major
      constexpr uint32_t idesc_o = umma_idesc_bf16(kTcRows, kD, 0, 1);       // P V: V is MN-major
      bool ok = mbar_wait(&q_full, 0);
      tc_fence_after();
      const uint32_t qa0 = smem_u32(sQ);
      // S (128 x 128) = Q_t K^T into tensor columns d_col
      // base descriptors once; per 16-wide k step only the start address moves
      const uint64_t qd[2] = {umma_desc_sw128(qa0, 16, 1024), umma_desc_sw128(qa0 + kTcQBytes, 16, 1024)};
      const uint64_t kd0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      auto mma_s = [&](uint32_t d_col, int t, int kst) {
        const uint64_t kd = umma_desc_add(kd0, kst * kTcTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kTcTileBytes / 2) + (kk & 3) * 32;
          umma_ss(tmem + d_col, umma_desc_add(qd[t], off), umma_desc_add(kd, off), idesc_s, kk > 0);
        }
      };
      auto kwait = [&](int f) { return mbar_wait(&k_full[f % kTcKStages], (uint32_t)(f / kTcKStages) & 1u); };
      // ---- pass A (local tile j = key tile j0 + j)
      for (int j = 0; j < n && ok && doA; ++j) {
        if (!(ok = kwait(j))) break;
        const int b = j & 1;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = mbar_wait(&sa_free[t][b], ((uint32_t)(j >> 1) & 1u) ^ 1u))) break;
          tc_fence_after();
          mma_s(256 * t + 128 * b, t, j % kTcKStages);
          umma_commit(&sa_full[t][b]);
        }
        umma_commit(&k_empty[j % kTcKStages]);
      }
      // every S buffer of pass A has been read before pass B reuses the columns
      for (int j = (n > 2 ? n - 2 : 0); j < n && ok && doA; ++j)
        for (int t = 0; t < 2 && ok; ++t) ok = mbar_wait(&sa_free[t][j & 1], (uint32_t)(j >> 1) & 1u);
      tc_fence_after();
      // ---- pass B (its K fills follow pass A's)
      const int kb = doA ? n : 0;
      if (doB && ok && n > 0 && (ok = kwait(kb))) {
        tc_fence_after();
        mma_s(0, 0, kb % kTcKStages);
        umma_commit(&sb_full[0]);
        mma_s(128, 1, kb % kTcKStages);
        umma_commit(&sb_full[1]);
        umma_commit(&k_empty[kb % kTcKStages]);
      }
      for (int j = 0; j < n && ok && doB; ++j) {
        const int vst = j % kTcVStages;
        if (!(ok = mbar_wait(&v_full[vst], (uint32_t)(j / kTcVStages) & 1u))) break;
        const uint64_t vd = umma_desc_sw128(smem_u32(sV + vst * kTcTileBytes), kTcTileBytes / 2, 1024);
        const int kf = kb + j + 1;  // the K fill of local tile j + 1
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = mbar_wait(&pb_full[t], (uint32_t)j & 1u))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTcKeys / 16; ++kk)
            umma_ts(tmem + 256 + 128 * t, tmem + 128 * t + kk * 8, umma_desc_add(vd, kk * 2048), idesc_o,
                    (j > 0 || kk > 0) ? 1u : 0u);
          if (t == 1) umma_commit(&v_empty[vst]);
          if (j + 1 < n) {
            // S_t of the next tile overwrites P_t, which the MMAs just issued
            // read: tcgen05.mma from one thread execute in issue order
            if (t == 0 && !(ok = kwait(kf))) break;
            tc_fence_after();
            mma_s(128 * t, t, kf % kTcKStages);
            umma_commit(&sb_full[t]);
            if (t == 1) umma_commit(&k_empty[kf % kTcKStages]);
          }
        }
      }
      umma_commit(&o_full);  // every MMA of the CTA (the softmax warps wait for it)
      if (!ok) record_error(a.err, HS2_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------- softmax warpgroup of Q tile tq
    const int tq = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;              // row of the Q tile = tensor-memory lane
    const int qr = tq * QT1 + row / G, hr = row % G;  // query of the CTA, head of the group
    const bool rv = qr < c.nq;
    const int64_t t = c.t0 + qr;
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t hrow = (c.q0 + qr) * a.Hq + (int64_t)g * G + hr;
    const int64_t t_min = c.t0;  // every row sees at least keys [0, t0]
    float* srow = a.scores + ((c.q0 + qr) * a.Hkv + g) * a.stride;
    const bool v4 = ((reinterpret_cast<uintptr_t>(a.scores) | ((uintptr_t)a.stride * 4)) & 15) == 0;
    // Every tcgen05.ld/st and full-mask shuffle below is reached by the whole
    // warp: the branches around them use warp-uniform conditions only.
    const bool all_rv = __all_sync(0xffffffffu, rv);
    // Softmax in base 2: with c2 = scale * log2(e), exp(scale*s - m) = 2^(c2*s - m2)
    // where m2 = m * log2(e); pass B folds the normalisation into the exponent:
    // P = 2^(c2*s - (m2 + log2 l)).
    const float c2 = a.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // ---- pass A: running max and sum
    for (int j = 0; j < n && doA; ++j) {
      const int b = j & 1;
      if (ok && !mbar_wait(&sa_full[tq][b], (uint32_t)(j >> 1) & 1u)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) {
        // the whole 128-key row of S at once: one wait, 128-wide independent work
        const int64_t k0 = (int64_t)(j0 + j) * kTcKeys;
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(trow + 256 * tq + 128 * b + 32 * q, r[q]);
        tmem_wait_ld();
        auto S = [&](int i) { return __uint_as_float(r[i >> 5][i & 31]); };
        auto body = [&](auto masked_c) {
          constexpr bool MASKED = decltype(masked_c)::value;
          // keys k0 .. k0+nv-1 are visible to this row
          const int nv = MASKED ? (rv ? (int)max((int64_t)0, min((int64_t)kTcKeys, t - k0 + 1)) : 0) : kTcKeys;
          auto valid = [nv](int i) { return !MASKED || i < nv; };
          float mx[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
#pragma unroll
          for (int i = 0; i < kTcKeys; ++i) mx[i & 7] = fmaxf(mx[i & 7], valid(i) ? S(i) : -INFINITY);
          const float cm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
          if (cm != -INFINITY) {
            const float mn = fmaxf(m, cm * c2);
            float sm[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) sm[u] = 0.f;
#pragma unroll
            for (int i = 0; i < kTcKeys; ++i) {
              const float e = ex2_approx(fmaf(S(i), c2, -mn));
              sm[i & 7] += valid(i) ? e : 0.f;
            }
            l = l * ex2_approx(m - mn) +
                (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
            m = mn;
          }
        };
        if (all_rv && k0 + kTcKeys - 1 <= t_min) body(std::false_type{});
        else body(std::true_type{});
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sa_free[tq][b]);
    }
    const int64_t nrows = a.total_q * a.Hq;
    if (a.mode == 1) {  // statistics of this key range only (m = -inf, l = 0 if it has none)
      if (rv) {
        a.part_ml[((int64_t)split * nrows + hrow) * 2] = m;
        a.part_ml[((int64_t)split * nrows + hrow) * 2 + 1] = l;
      }
    }
    if (a.mode == 2 && rv) {  // the row's statistics over all ranges, in range order
      float M = -INFINITY;
      for (int q = 0; q < ks; ++q) M = fmaxf(M, a.part_ml[((int64_t)q * nrows + hrow) * 2]);
      float L = 0.f;
      for (int q = 0; q < ks; ++q) {
        const float mq = a.part_ml[((int64_t)q * nrows + hrow) * 2];
        if (mq != -INFINITY) L += a.part_ml[((int64_t)q * nrows + hrow) * 2 + 1] * exp2f(mq - M);
      }
      m = M;
      l = L;
    }
    const float mb = (rv && l > 0.f) ? m + log2f(l) : 0.f;  // l >= 1 for a visible row
    // ---- pass B: P (handed to the MMA warp first), then the scores
    for (int j = 0; j < n && doB; ++j) {
      if (ok && !mbar_wait(&sb_full[tq], (uint32_t)j & 1u)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int64_t k0 = (int64_t)(j0 + j) * kTcKeys;
      const bool full = all_rv && k0 + kTcKeys - 1 <= t_min;  // no key of the tile is masked
      // keys k0 .. k0+nv-1 are visible to this row
      const int nv = full ? kTcKeys : (rv ? (int)max((int64_t)0, min((int64_t)kTcKeys, t - k0 + 1)) : 0);
      float p[4][32];
      if (ok) {
        // the whole 128-key row of S at once, then P (bf16) into the first 64
        // columns, which have been read
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(trow + 128 * tq + 32 * q, r[q]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float e = ex2_approx(fmaf(__uint_as_float(r[q][i]), c2, -mb));
            p[q][i] = (full || 32 * q + i < nv) ? e : 0.f;
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(p[q][2 * i], p[q][2 * i + 1]);
          tmem_st16(trow + 128 * tq + 16 * q, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pb_full[tq]);
      if (ok) {
        // scores: sum over the G rows of each query (consecutive lanes) by a
        // reduce-scatter butterfly, two 32-key chunks at a time; each lane ends
        // with 32/G consecutive keys of each chunk, at offset ``off``
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          int off = 0, nn = 32;
#pragma unroll
          for (int msk = G / 2; msk >= 1; msk >>= 1) {
            const bool up = (lane & msk) != 0;
            nn >>= 1;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                if (i < nn) {
                  float* q = p[2 * hh + cc];
                  const float send = up ? q[i] : q[i + nn];
                  const float keep = up ? q[i + nn] : q[i];
                  q[i] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
                }
              }
            }
            if (up) off += nn;
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const float* q = p[2 * hh + cc];
            const int64_t ks = k0 + 64 * hh + 32 * cc + off;
            if (full && v4) {
              float4* dst = reinterpret_cast<float4*>(srow + ks);
              // scores are read once, later, by the selection: stream them past L2
#pragma unroll
              for (int i = 0; i < 32 / G / 4; ++i)
                __stcs(dst + i, make_float4(q[4 * i], q[4 * i + 1], q[4 * i + 2], q[4 * i + 3]));
            } else if (rv) {
#pragma unroll
              for (int i = 0; i < 32 / G; ++i)
                if (ks + i <= t) srow[ks + i] = q[i];
            }
          }
        }
      }
    }
    // ---- O of this row: bf16 out of tensor memory (mode 2: this range's
    // float32 share, zero for a range with no key tile)
    if (ok && !mbar_wait(&o_full, 0)) {
      record_error(a.err, HS2_ERR_TIMEOUT);
      ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    bf16* O = static_cast<bf16*>(a.O);
#pragma unroll 1
    for (int ch = 0; ch < 4 && ok && a.mode == 2; ++ch) {
      uint32_t r[32];
      if (n > 0) {
        tmem_ld32(trow + 256 + 128 * tq + ch * 32, r);
        tmem_wait_ld();
      }
      if (rv) {
        float4* dst = reinterpret_cast<float4*>(a.part_o + ((int64_t)split * nrows + hrow) * kD + ch * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = n > 0 ? make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                       __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll 1
    for (int ch = 0; ch < 4 && ok && a.mode == 0; ++ch) {
      uint32_t r[32];
      tmem_ld32(trow + 256 + 128 * tq + ch * 32, r);
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
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// O of a key-split chunk: the ranges' float32 shares added in range order,
// written as bf16.  One thread per 4 columns of a row.
__global__ void __launch_bounds__(256) k_chunk_o_sum(const float* part_o, int ks, int64_t nrows, bf16* O) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // float4 index
  if (i >= nrows * (kD / 4)) return;
  float4 acc = reinterpret_cast<const float4*>(part_o)[i];
  for (int q = 1; q < ks; ++q) {
    const float4 v = reinterpret_cast<const float4*>(part_o)[(int64_t)q * nrows * (kD / 4) + i];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  uint2 pk;
  pk.x = pack_bf16(acc.x, acc.y);
  pk.y = pack_bf16(acc.z, acc.w);
  reinterpret_cast<uint2*>(O)[i] = pk;
}

}  // namespace hs2
