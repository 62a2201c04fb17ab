// chunk_attn.cuh - Full Attention layer of a Hybrid Block for a chunk of new
// query tokens appended to a cached context (agent turns), causal, with the
// per-key selection scores of every query token.
//
// Source: "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
// Agents", section "From Hybrid SWA to HySparse2 ..." (one full-attention layer
// per Hybrid Block builds the cache and judges token importance) and section
// "Two-Level KV Sharing: ..." (prefill is dominated by large matrix products).
//
// Storing per-head logits is out of the question here (Tq x N x Hq floats), so
// the scores take a second pass that recomputes Q K^T with the final softmax
// statistics of the first pass:
//   pass 1  k_chunk_fwd_*:    O and (m_h, l_h) per (query, head), online softmax
//   pass 2  k_chunk_scores_*: s_g[j] = sum_{h in g} exp(x_hj - m_h) / l_h
// bf16 tiles: 128 rows = (128 / G) query tokens x G heads of one KV group share
// every K/V tile (GQA), 64 keys per tile, 8 warps of 16 rows on mma.sync.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

constexpr int kChRows = 128;      // (query, head) rows per CTA
constexpr int kChWarps = 8;       // consumer warps, 16 rows each
constexpr int kChTile = 64;       // keys per stage
constexpr int kChStages = 3;
constexpr int kChKBytes = 2 * 8192;  // one K (or V) tile: two swizzled 64-column halves

struct ChunkArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hq, Hkv, G, QT;  // QT: query tokens per CTA (= 128 / G for bf16)
  int64_t total_q, total_kv;
  float scale;
  void* O;
  float* ml;              // [total_q, Hq, 2]
  float* scores;
  int64_t stride;
  int* err;
};

// Sequence-level geometry of CTA (blockIdx.x = query tile, blockIdx.z = sequence).
struct ChTile {
  int64_t q0;       // first query row (packed index) of the tile
  int nq;           // query tokens in the tile
  int64_t kv0;      // first key of the sequence (packed index)
  int64_t N;        // keys of the sequence
  int64_t t0;       // position of the tile's first query
};
__device__ __forceinline__ bool chunk_tile(const ChunkArgs& a, ChTile& c) {
  const int b = blockIdx.z;
  const int64_t qs = __ldg(a.qoff + b), qe = __ldg(a.qoff + b + 1);
  c.kv0 = __ldg(a.kvoff + b);
  c.N = __ldg(a.kvoff + b + 1) - c.kv0;
  const int64_t Tq = qe - qs;
  const int64_t i0 = (int64_t)blockIdx.x * a.QT;
  if (i0 >= Tq) return false;
  if (qs < 0 || qe > a.total_q || c.kv0 < 0 || c.kv0 + c.N > a.total_kv || Tq > c.N ||
      c.N > a.stride) {
    if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    return false;
  }
  c.q0 = qs + i0;
  c.nq = (int)(Tq - i0 < a.QT ? Tq - i0 : a.QT);
  c.t0 = c.N - Tq + i0;
  return true;
}

// ----------------------------------------------------------------------------
// bf16 tiles on mma.sync.  Warp w owns rows 16w..16w+15; row -> (query r / G,
// head r % G).  S = Q K^T (16 x 64 per warp) from ldmatrix'ed K, P re-used as
// the A operand of P V straight from the S accumulators.
// ----------------------------------------------------------------------------
template <bool SCORES>
__global__ void __launch_bounds__(32 * (kChWarps + 1))
    k_chunk_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ ChunkArgs a) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kChStages];
  __shared__ __align__(8) uint64_t empty_bar[kChStages];
  ChTile c;
  if (!chunk_tile(a, c)) return;
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  constexpr int kStage = SCORES ? kChKBytes : 2 * kChKBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  // keys [0, t_last] are visible to some query of the tile
  const int64_t t_last = c.t0 + c.nq - 1;
  const int64_t nkeys = t_last + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kChStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kChWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kChWarps) {
    if (lane != 0) return;
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    for (int64_t k0 = 0; k0 < nkeys; k0 += kChTile) {
      if (!mbar_wait(&empty_bar[stage], phase ^ 1)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        break;
      }
      mbar_arrive_expect_tx(&full_bar[stage], kStage);
      uint8_t* sk = ring + stage * kStage;
      const int key = (int)(c.kv0 + k0);
      tma_load_3d(sk, &tmK, &full_bar[stage], 0, g, key);
      tma_load_3d(sk + 8192, &tmK, &full_bar[stage], 64, g, key);
      if (!SCORES) {
        tma_load_3d(sk + kChKBytes, &tmV, &full_bar[stage], 0, g, key);
        tma_load_3d(sk + kChKBytes + 8192, &tmV, &full_bar[stage], 64, g, key);
      }
      issued |= 1u << stage;
      last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == kChStages) { stage = 0; phase ^= 1; }
    }
    for (int s = 0; s < kChStages; ++s)
      if ((issued >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
    return;
  }

  const int r = lane >> 2, qd = lane & 3;
  const bf16* Q = static_cast<const bf16*>(a.Q);
  // this thread's two rows
  const int rowA = warp * 16 + r, rowB = rowA + 8;
  const int qA = rowA / a.G, qB = rowB / a.G;
  const bool okA = rowA < a.QT * a.G && qA < c.nq, okB = rowB < a.QT * a.G && qB < c.nq;
  const int64_t tA = c.t0 + qA, tB = c.t0 + qB;
  // A fragments of Q (16 rows x 128 d) for 8 k-steps
  uint32_t qa[8][4];
  {
    const bf16* pa = Q + ((c.q0 + qA) * a.Hq + (int64_t)g * a.G + rowA % a.G) * kD;
    const bf16* pb = Q + ((c.q0 + qB) * a.Hq + (int64_t)g * a.G + rowB % a.G) * kD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int d = kk * 16 + 2 * qd;
      qa[kk][0] = okA ? *reinterpret_cast<const uint32_t*>(pa + d) : 0u;
      qa[kk][1] = okB ? *reinterpret_cast<const uint32_t*>(pb + d) : 0u;
      qa[kk][2] = okA ? *reinterpret_cast<const uint32_t*>(pa + d + 8) : 0u;
      qa[kk][3] = okB ? *reinterpret_cast<const uint32_t*>(pb + d + 8) : 0u;
    }
  }
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
  if (SCORES) {
    if (okA) { mA = a.ml[((c.q0 + qA) * a.Hq + (int64_t)g * a.G + rowA % a.G) * 2]; lA = a.ml[((c.q0 + qA) * a.Hq + (int64_t)g * a.G + rowA % a.G) * 2 + 1]; }
    if (okB) { mB = a.ml[((c.q0 + qB) * a.Hq + (int64_t)g * a.G + rowB % a.G) * 2]; lB = a.ml[((c.q0 + qB) * a.Hq + (int64_t)g * a.G + rowB % a.G) * 2 + 1]; }
  }
  const float ilA = lA > 0.f ? 1.f / lA : 0.f, ilB = lB > 0.f ? 1.f / lB : 0.f;
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int64_t k0 = 0; k0 < nkeys; k0 += kChTile) {
    if (ok && !mbar_wait(&full_bar[stage], phase)) {
      record_error(a.err, HS2_ERR_TIMEOUT);
      ok = false;
    }
    if (ok) {
      const uint32_t skb = smem_u32(ring + stage * kStage);
      float s[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
      // S = Q K^T: B fragments from K rows (key = n*8 + lane%8), 4 chunks per x4
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int key = n * 8 + (lane & 7);
#pragma unroll
        for (int kk2 = 0; kk2 < 4; ++kk2) {
          const int chunk = kk2 * 4 + (lane >> 3);  // 16-byte chunk 0..15 of the row
          const uint32_t addr = skb + (chunk >> 3) * 8192 + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3, addr);
          mma_bf16(s[n], qa[2 * kk2][0], qa[2 * kk2][1], qa[2 * kk2][2], qa[2 * kk2][3], b0, b1);
          mma_bf16(s[n], qa[2 * kk2 + 1][0], qa[2 * kk2 + 1][1], qa[2 * kk2 + 1][2], qa[2 * kk2 + 1][3], b2, b3);
        }
      }
      // scale + causal mask
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int64_t j0 = k0 + n * 8 + 2 * qd;
        s[n][0] = (okA && j0 <= tA) ? s[n][0] * a.scale : -INFINITY;
        s[n][1] = (okA && j0 + 1 <= tA) ? s[n][1] * a.scale : -INFINITY;
        s[n][2] = (okB && j0 <= tB) ? s[n][2] * a.scale : -INFINITY;
        s[n][3] = (okB && j0 + 1 <= tB) ? s[n][3] * a.scale : -INFINITY;
      }
      if (SCORES) {
        // p = exp(x - m) / l, summed over the G heads of each query token
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          float v0 = exp_shift(s[n][0], mA) * ilA, v1 = exp_shift(s[n][1], mA) * ilA;
          float v2 = exp_shift(s[n][2], mB) * ilB, v3 = exp_shift(s[n][3], mB) * ilB;
          for (int off = 4; off < 4 * a.G; off <<= 1) {
            v0 += __shfl_xor_sync(0xffffffffu, v0, off);
            v1 += __shfl_xor_sync(0xffffffffu, v1, off);
            v2 += __shfl_xor_sync(0xffffffffu, v2, off);
            v3 += __shfl_xor_sync(0xffffffffu, v3, off);
          }
          if (rowA % a.G == 0) {
            const int64_t j = k0 + n * 8 + 2 * qd;
            float* dstA = a.scores + ((c.q0 + qA) * a.Hkv + g) * a.stride;
            float* dstB = a.scores + ((c.q0 + qB) * a.Hkv + g) * a.stride;
            if (okA && j <= tA) dstA[j] = v0;
            if (okA && j + 1 <= tA) dstA[j + 1] = v1;
            if (okB && j <= tB) dstB[j] = v2;
            if (okB && j + 1 <= tB) dstB[j + 1] = v3;
          }
        }
      } else {
        float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          mxA = fmaxf(mxA, fmaxf(s[n][0], s[n][1]));
          mxB = fmaxf(mxB, fmaxf(s[n][2], s[n][3]));
        }
        mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
        mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
        const float mnA = fmaxf(mA, mxA), mnB = fmaxf(mB, mxB);
        const float alA = (mnA == -INFINITY) ? 1.f : exp_shift(mA, mnA);
        const float alB = (mnB == -INFINITY) ? 1.f : exp_shift(mB, mnB);
        float sumA = 0.f, sumB = 0.f;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          s[n][0] = exp_shift(s[n][0], mnA); s[n][1] = exp_shift(s[n][1], mnA);
          s[n][2] = exp_shift(s[n][2], mnB); s[n][3] = exp_shift(s[n][3], mnB);
          sumA += s[n][0] + s[n][1];
          sumB += s[n][2] + s[n][3];
        }
        lA = lA * alA + sumA;
        lB = lB * alB + sumB;
        mA = mnA;
        mB = mnB;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          o[i][0] *= alA; o[i][1] *= alA; o[i][2] *= alB; o[i][3] *= alB;
        }
        const uint32_t svb = skb + kChKBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 keys per k-step
          const uint32_t a0 = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
          const uint32_t a1 = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
          const uint32_t a2 = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
          const uint32_t a3 = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
          const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
          for (int n2 = 0; n2 < 8; ++n2) {  // pairs of 8-column d tiles
            const int chunk = n2 * 2 + (lane >> 4);
            const uint32_t addr = svb + (chunk >> 3) * 8192 + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(b0, b1, b2, b3, addr);
            mma_bf16(o[2 * n2], a0, a1, a2, a3, b0, b1);
            mma_bf16(o[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[stage]);
    if (++stage == kChStages) { stage = 0; phase ^= 1; }
  }
  if (!SCORES) {
    lA += __shfl_xor_sync(0xffffffffu, lA, 1);
    lA += __shfl_xor_sync(0xffffffffu, lA, 2);
    lB += __shfl_xor_sync(0xffffffffu, lB, 1);
    lB += __shfl_xor_sync(0xffffffffu, lB, 2);
    bf16* O = static_cast<bf16*>(a.O);
    const float iA = lA > 0.f ? 1.f / lA : 0.f, iB = lB > 0.f ? 1.f / lB : 0.f;
    const int64_t hrA = (c.q0 + qA) * a.Hq + (int64_t)g * a.G + rowA % a.G;
    const int64_t hrB = (c.q0 + qB) * a.Hq + (int64_t)g * a.G + rowB % a.G;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int d = i * 8 + 2 * qd;
      if (okA) *reinterpret_cast<uint32_t*>(O + hrA * kD + d) = pack_bf16(o[i][0] * iA, o[i][1] * iA);
      if (okB) *reinterpret_cast<uint32_t*>(O + hrB * kD + d) = pack_bf16(o[i][2] * iB, o[i][3] * iB);
    }
    if (qd == 0) {
      if (okA) { a.ml[hrA * 2] = mA; a.ml[hrA * 2 + 1] = lA; }
      if (okB) { a.ml[hrB * 2] = mB; a.ml[hrB * 2 + 1] = lB; }
    }
  }
}

// ----------------------------------------------------------------------------
// float32 chunk path on the CUDA cores (exact fp32 arithmetic).
// Pass 1: one CTA per (query row, KV group); warp w takes every 4th key.
// ----------------------------------------------------------------------------
template <int GP>
__global__ void __launch_bounds__(128) k_chunk_fwd_f32(const __grid_constant__ ChunkArgs a) {
  const int64_t qi = blockIdx.x;
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const QueryRow qr = query_row(a.qoff, a.kvoff, a.B, qi);
  const float* Q = static_cast<const float*>(a.Q);
  const float* K = static_cast<const float*>(a.K);
  const float* V = static_cast<const float*>(a.V);
  __shared__ float sm[4][GP], sl[4][GP];
  __shared__ float so[4][GP][kD];
  float4 q[GP], o[GP];
  float m[GP], l[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    q[h] = (h < a.G) ? *reinterpret_cast<const float4*>(Q + (qi * a.Hq + (int64_t)g * a.G + h) * kD + lane * 4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    o[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    m[h] = -INFINITY;
    l[h] = 0.f;
  }
  const bool good = qr.kv_start >= 0 && qr.kv_start + qr.kv_len <= a.total_kv && qr.t < qr.kv_len;
  if (!good && threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
  for (int64_t j = warp; good && j <= qr.t; j += 4) {
    const int64_t row = (qr.kv_start + j) * a.Hkv + g;
    const float4 kv = *reinterpret_cast<const float4*>(K + row * kD + lane * 4);
    const float4 vv = *reinterpret_cast<const float4*>(V + row * kD + lane * 4);
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      if (h >= a.G) break;
      float dot = q[h].x * kv.x;
      dot = fmaf(q[h].y, kv.y, dot);
      dot = fmaf(q[h].z, kv.z, dot);
      dot = fmaf(q[h].w, kv.w, dot);
      const float x = warp_sum(dot) * a.scale;
      const float mn = fmaxf(m[h], x);
      const float al = exp_shift(m[h], mn);
      const float pr = expf(x - mn);
      l[h] = l[h] * al + pr;
      o[h].x = fmaf(pr, vv.x, o[h].x * al);
      o[h].y = fmaf(pr, vv.y, o[h].y * al);
      o[h].z = fmaf(pr, vv.z, o[h].z * al);
      o[h].w = fmaf(pr, vv.w, o[h].w * al);
      m[h] = mn;
    }
  }
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    if (lane == 0) { sm[warp][h] = m[h]; sl[warp][h] = l[h]; }
    *reinterpret_cast<float4*>(&so[warp][h][lane * 4]) = o[h];
  }
  __syncthreads();
  float* O = static_cast<float*>(a.O);
  for (int i = threadIdx.x; i < a.G * kD; i += blockDim.x) {
    const int h = i / kD, d = i % kD;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w][h]);
    float L = 0.f, acc = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float wt = exp_shift(sm[w][h], M);
      L = fmaf(sl[w][h], wt, L);
      acc = fmaf(so[w][h][d], wt, acc);
    }
    const int64_t hr = qi * a.Hq + (int64_t)g * a.G + h;
    O[hr * kD + d] = L > 0.f ? acc / L : 0.f;
    if (d == 0) { a.ml[hr * 2] = M; a.ml[hr * 2 + 1] = L; }
  }
}

// Pass 2 (fp32): CTA (key block of 32, KV group, query row); warp w scores keys
// 8w..8w+7 of the block: recomputed logits, normalised, summed over the group.
template <int GP>
__global__ void __launch_bounds__(128) k_chunk_scores_f32(const __grid_constant__ ChunkArgs a) {
  const int64_t qi = blockIdx.z;
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const QueryRow qr = query_row(a.qoff, a.kvoff, a.B, qi);
  if (qr.kv_start < 0 || qr.kv_start + qr.kv_len > a.total_kv || qr.t >= qr.kv_len) return;
  if (qr.t >= a.stride) { if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT); return; }
  const float* Q = static_cast<const float*>(a.Q);
  const float* K = static_cast<const float*>(a.K);
  float4 q[GP];
  float m[GP], lh[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    const int64_t hr = qi * a.Hq + (int64_t)g * a.G + h;
    q[h] = (h < a.G) ? *reinterpret_cast<const float4*>(Q + hr * kD + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    m[h] = (h < a.G) ? a.ml[hr * 2] : 0.f;
    lh[h] = (h < a.G) ? a.ml[hr * 2 + 1] : 1.f;
  }
  for (int i = 0; i < 8; ++i) {
    const int64_t j = (int64_t)blockIdx.x * 32 + warp * 8 + i;
    if (j > qr.t) break;
    const float4 kv = *reinterpret_cast<const float4*>(K + ((qr.kv_start + j) * a.Hkv + g) * kD + lane * 4);
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      if (h >= a.G) break;
      float dot = q[h].x * kv.x;
      dot = fmaf(q[h].y, kv.y, dot);
      dot = fmaf(q[h].z, kv.z, dot);
      dot = fmaf(q[h].w, kv.w, dot);
      const float x = warp_sum(dot) * a.scale;
      sc += expf(x - m[h]) / lh[h];
    }
    if (lane == 0) a.scores[(qi * a.Hkv + g) * a.stride + j] = sc;
  }
}

}  // namespace hs2
