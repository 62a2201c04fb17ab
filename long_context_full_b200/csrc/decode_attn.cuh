// decode_attn.cuh - Full Attention layer of a Hybrid Block for decode (one query
// token per sequence), which also emits the per-key selection scores.
//
// Source: "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
// Agents", section "From Hybrid SWA to HySparse2 ..." (the full-attention layer
// builds the KV cache and decides which tokens are important) and "Xiaomi
// Unveils HySparse2 for Faster Long-Context AI", section "Two-Level KV Sharing".
//
// Three launches:
//   1. k_decode_bf16 / k_decode_f32: split-context pass.  The packed key space
//      of every KV head is cut into P balanced ranges, one per CTA, regardless
//      of sequence boundaries (ragged batches stay balanced).  A CTA streams its
//      K/V rows once, writes the scaled logits x_hj of its keys, and keeps an
//      online-softmax partial (m, l, O) per warp and per sequence piece.
//   2. k_decode_combine: merges the partials of each (sequence, head) into the
//      output O and the final softmax statistics (m_h, l_h).
//   3. k_finalize_scores: s_g[j] = sum_{h in g} exp(x_hj - m_h) / l_h.
// The per-head logits must be stored because the score needs each head's final
// statistics, which are only known after the whole cache has been read; storing
// them (32 B per key and KV head at G = 8) is far cheaper than reading K twice.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

constexpr int kDecTile = 64;        // keys per pipeline stage
constexpr int kDecWarps = 4;        // consumer warps, 16 keys of each tile each
constexpr int kDecStageBytes = 4 * 8192;  // K and V, two 64-column swizzled halves each

struct DecodeArgs {
  const void* Q;          // [total_q, Hq, D]
  const void* K;          // [total_kv, Hkv, D] (CUDA-core path)
  const void* V;
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hq, Hkv, G, P;   // P: CTAs per KV head
  int64_t total_q, total_kv;
  float scale;
  float* logits;          // [total_kv, Hq]
  float* pm;              // [(P+B), Hkv, kDecWarps, G]
  float* pl;
  float* po;              // [(P+B), Hkv, kDecWarps, G, D]
  int* err;
};

// Walks the pieces (sequence b, key range [s, e)) of CTA p's key range; for
// each piece whose sequence has a query row, calls f(b, s, e, q0).
template <typename F>
__device__ __forceinline__ void for_each_piece(const DecodeArgs& a, int p, F f) {
  const int64_t W = a.total_kv;
  const int64_t lo = split_lo(W, a.P, p), hi = split_lo(W, a.P, p + 1);
  if (lo >= hi) return;
  for (int b = last_le(a.kvoff, a.B, lo); b < a.B; ++b) {
    const int64_t kb = __ldg(a.kvoff + b), ke = __ldg(a.kvoff + b + 1);
    if (kb >= hi) break;
    const int64_t s = kb > lo ? kb : lo, e = ke < hi ? ke : hi;
    if (s >= e) continue;
    const int64_t q0 = __ldg(a.qoff + b), qn = __ldg(a.qoff + b + 1) - q0;
    if (qn < 1) continue;
    if (q0 < 0 || q0 >= a.total_q) continue;  // inconsistent offsets: reported by the combine
    f(b, s, e, q0);
  }
}

// ----------------------------------------------------------------------------
// bf16 split-context pass on the tensor cores (mma.sync m16n8k16).
// Per warp and 16-key slice of a tile:  S^T[16 keys x 8 heads] = K Q^T, then
// O^T[128 x 8] += V^T P^T, with P^T obtained from the S^T accumulator by one
// register transpose (movmatrix), so no shared-memory round trip for P.
// Warp 4 is the producer: one lane issues TMA loads into an NST-deep ring.
// ----------------------------------------------------------------------------
template <int NST>
__global__ void __launch_bounds__(32 * (kDecWarps + 1))
    k_decode_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ DecodeArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[NST];
  __shared__ __align__(8) uint64_t empty_bar[NST];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x, g = blockIdx.y;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kDecWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;  // bit s: stage s has a fill in flight or unconsumed
    uint32_t last_phase = 0;
    bool ok = true;
    for_each_piece(a, p, [&](int b, int64_t s, int64_t e, int64_t q0) {
      for (int64_t k0 = s; k0 < e && ok; k0 += kDecTile) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1)) {
          record_error(a.err, HS2_ERR_TIMEOUT);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[stage], kDecStageBytes);
        uint8_t* sk = ring + stage * kDecStageBytes;
        uint8_t* sv = sk + 2 * 8192;
        const int key = static_cast<int>(k0);
        tma_load_3d_hint(sk, &tmK, &full_bar[stage], 0, g, key, pol);
        tma_load_3d_hint(sk + 8192, &tmK, &full_bar[stage], 64, g, key, pol);
        tma_load_3d_hint(sv, &tmV, &full_bar[stage], 0, g, key, pol);
        tma_load_3d_hint(sv + 8192, &tmV, &full_bar[stage], 64, g, key, pol);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == NST) { stage = 0; phase ^= 1; }
      }
    });
    // drain: every fill this thread issued has landed before the CTA can exit
    for (int s = 0; s < NST; ++s)
      if ((issued >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
    return;
  }

  // -------------------------------------------------------------- consumers
  const bf16* Q = static_cast<const bf16*>(a.Q);
  const uint64_t keep = policy_evict_last();
  const int r = lane >> 2, qd = lane & 3;
  const float NEG = -INFINITY;
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;

  for_each_piece(a, p, [&](int b, int64_t s, int64_t e, int64_t q0) {
    // query fragments: B operand of S^T = K Q^T, head n = r of the group
    uint32_t qf[8][2];
    const bf16* qrow = Q + ((q0 * a.Hq) + (int64_t)g * a.G + r) * kD;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      if (r < a.G) {
        qf[kk][0] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * qd);
        qf[kk][1] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * qd);
      } else {
        qf[kk][0] = qf[kk][1] = 0u;
      }
    }
    float m0 = NEG, m1 = NEG, l0 = 0.f, l1 = 0.f;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    const int h0 = 2 * qd, h1 = 2 * qd + 1;  // this thread's two heads
    float* lg = a.logits + (int64_t)g * a.G;

    for (int64_t k0 = s; k0 < e; k0 += kDecTile) {
      if (ok && !mbar_wait(&full_bar[stage], phase)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      if (ok) {
        const uint8_t* sk = ring + stage * kDecStageBytes;
        const uint8_t* sv = sk + 2 * 8192;
        const uint32_t skb = smem_u32(sk), svb = smem_u32(sv);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int row = warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int chunk = (kk & 3) * 2 + (lane >> 4);
            const uint32_t addr = skb + (kk >> 2) * 8192 + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a0, a1, a2, a3, addr);
            mma_bf16(c, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
          }
        }
        const int64_t klo = k0 + warp * 16 + r, khi = klo + 8;
        const bool vlo = klo < e, vhi = khi < e;
        const float x0 = vlo ? c[0] * a.scale : NEG, x1 = vlo ? c[1] * a.scale : NEG;
        const float x2 = vhi ? c[2] * a.scale : NEG, x3 = vhi ? c[3] * a.scale : NEG;
        // logits of the real heads
        // logits are read back by the score finalize right after this pass:
        // ask L2 to keep them (the K/V stream is loaded evict-first)
        if (h1 < a.G && (a.G & 1) == 0) {  // even G: the pair is 8-byte aligned
          if (vlo) st_hint_f2(lg + klo * a.Hq + h0, x0, x1, keep);
          if (vhi) st_hint_f2(lg + khi * a.Hq + h0, x2, x3, keep);
        } else {
          if (h0 < a.G) {
            if (vlo) st_hint_f1(lg + klo * a.Hq + h0, x0, keep);
            if (vhi) st_hint_f1(lg + khi * a.Hq + h0, x2, keep);
          }
          if (h1 < a.G) {
            if (vlo) st_hint_f1(lg + klo * a.Hq + h1, x1, keep);
            if (vhi) st_hint_f1(lg + khi * a.Hq + h1, x3, keep);
          }
        }
        // online softmax over the 16 keys of this warp, per head (column)
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = (mn0 == NEG) ? 1.f : exp_shift(m0, mn0);
        const float al1 = (mn1 == NEG) ? 1.f : exp_shift(m1, mn1);
        const float p0 = exp_shift(x0, mn0), p1 = exp_shift(x1, mn1);
        const float p2 = exp_shift(x2, mn0), p3 = exp_shift(x3, mn1);
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
        }
        const uint32_t b0 = movmatrix_t(pack_bf16(p0, p1));
        const uint32_t b1 = movmatrix_t(pack_bf16(p2, p3));
        {
          const int row = warp * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int chunk = (mt & 3) * 2 + ((lane >> 3) & 1);
            const uint32_t addr = svb + (mt >> 2) * 8192 + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(a0, a1, a2, a3, addr);
            mma_bf16(o[mt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[stage]);
      if (++stage == NST) { stage = 0; phase ^= 1; }
    }
    // per-warp partial of this piece
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int64_t slot = (int64_t)p + b;
    const int64_t base = ((slot * a.Hkv + g) * kDecWarps + warp) * a.G;
    if (r == 0) {
      if (h0 < a.G) { a.pm[base + h0] = m0; a.pl[base + h0] = l0; }
      if (h1 < a.G) { a.pm[base + h1] = m1; a.pl[base + h1] = l1; }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int d = mt * 16 + r;
      if (h0 < a.G) {
        a.po[(base + h0) * kD + d] = o[mt][0];
        a.po[(base + h0) * kD + d + 8] = o[mt][2];
      }
      if (h1 < a.G) {
        a.po[(base + h1) * kD + d] = o[mt][1];
        a.po[(base + h1) * kD + d + 8] = o[mt][3];
      }
    }
  });
}

// ----------------------------------------------------------------------------
// float32 split-context pass on the CUDA cores (exact fp32 products and sums).
// Each warp takes every 4th key of the CTA's pieces; lane i holds dims
// 4i..4i+3.  GP >= G is the compile-time head bound.
// ----------------------------------------------------------------------------
template <int GP>
__global__ void __launch_bounds__(32 * kDecWarps) k_decode_f32(const __grid_constant__ DecodeArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x, g = blockIdx.y;
  const float* Q = static_cast<const float*>(a.Q);
  const float* K = static_cast<const float*>(a.K);
  const float* V = static_cast<const float*>(a.V);
  for_each_piece(a, p, [&](int b, int64_t s, int64_t e, int64_t q0) {
    float4 q[GP];
    float m[GP], l[GP];
    float4 o[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      q[h] = (h < a.G) ? *reinterpret_cast<const float4*>(Q + ((q0 * a.Hq) + (int64_t)g * a.G + h) * kD + lane * 4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      m[h] = -INFINITY;
      l[h] = 0.f;
      o[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int64_t j = s + warp; j < e; j += kDecWarps) {
      const float4 kv = *reinterpret_cast<const float4*>(K + (j * a.Hkv + g) * kD + lane * 4);
      const float4 vv = *reinterpret_cast<const float4*>(V + (j * a.Hkv + g) * kD + lane * 4);
#pragma unroll
      for (int h = 0; h < GP; ++h) {
        if (h >= a.G) break;
        float dot = q[h].x * kv.x;
        dot = fmaf(q[h].y, kv.y, dot);
        dot = fmaf(q[h].z, kv.z, dot);
        dot = fmaf(q[h].w, kv.w, dot);
        const float x = warp_sum(dot) * a.scale;
        if (lane == 0) a.logits[j * a.Hq + (int64_t)g * a.G + h] = x;
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
    const int64_t slot = (int64_t)p + b;
    const int64_t base = ((slot * a.Hkv + g) * kDecWarps + warp) * a.G;
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      if (h >= a.G) break;
      if (lane == 0) { a.pm[base + h] = m[h]; a.pl[base + h] = l[h]; }
      *reinterpret_cast<float4*>(a.po + (base + h) * kD + lane * 4) = o[h];
    }
  });
}

// ----------------------------------------------------------------------------
// Combine: O and (m_h, 1/l_h) of each (sequence, head) from the per-warp partials
// of every CTA whose key range meets the sequence.  Grid (B, Hkv, G), D
// threads: thread i owns partial i for the max and the weights, then thread d
// sums dimension d over all partials (independent, coalesced loads).
// ----------------------------------------------------------------------------
constexpr int kCombStage = 64;  // partial rows staged in shared memory per round

template <typename OT>
__global__ void __launch_bounds__(kD) k_decode_combine(const __grid_constant__ DecodeArgs a, OT* O,
                                                       float* ml) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int b = blockIdx.x, g = blockIdx.y, hl = blockIdx.z, d = threadIdx.x;
  if (b == 0 && g == 0 && hl == 0 && d == 0) {
    if (__ldg(a.kvoff + a.B) != a.total_kv || __ldg(a.qoff + a.B) != a.total_q)
      record_error(a.err, HS2_ERR_DEVICE_INPUT);
  }
  const int64_t q0 = __ldg(a.qoff + b);
  const int64_t qn = __ldg(a.qoff + b + 1) - q0;
  if (qn < 1) return;
  if (qn > 1 || q0 < 0 || q0 >= a.total_q) {
    if (d == 0 && hl == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    return;
  }
  const int64_t W = a.total_kv;
  const int64_t kb = __ldg(a.kvoff + b), ke = __ldg(a.kvoff + b + 1);
  int pf = 0, np = 0;
  if (ke > kb) {
    pf = split_owner(W, a.P, kb);
    np = (split_owner(W, a.P, ke - 1) - pf + 1) * kDecWarps;
  }
  __shared__ __align__(16) float so[kCombStage][kD];
  __shared__ float sw[kCombStage], swl[kCombStage];
  __shared__ float red[kD / 32];
  // partial i = (CTA pf + i / warps, warp i % warps); CTAs with an empty range wrote nothing
  auto pidx = [&](int i, bool* valid) -> int64_t {
    const int p = pf + i / kDecWarps;
    *valid = split_lo(W, a.P, p) < split_lo(W, a.P, p + 1);
    return (((int64_t)(p + b) * a.Hkv + g) * kDecWarps + (i % kDecWarps)) * a.G + hl;
  };
  float M = -INFINITY;
  for (int i = d; i < np; i += kD) {
    bool v;
    const int64_t pi = pidx(i, &v);
    if (v) M = fmaxf(M, a.pm[pi]);
  }
  M = warp_max(M);
  if ((d & 31) == 0) red[d >> 5] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float L = 0.f, acc = 0.f;
  for (int c0 = 0; c0 < np; c0 += kCombStage) {
    const int n = min(kCombStage, np - c0);
    if (d < n) {
      bool v;
      const int64_t pi = pidx(c0 + d, &v);
      const float w = v ? exp_shift(a.pm[pi], M) : 0.f;
      sw[d] = w;
      swl[d] = w != 0.f ? w * a.pl[pi] : 0.f;
    }
    // the n partial O rows, all copies in flight at once (zero rows skipped)
    for (int e = d; e < n * (kD / 4); e += kD) {
      const int i = e / (kD / 4), c = e % (kD / 4);
      bool v;
      const int64_t pi = pidx(c0 + i, &v);
      cp_async16(&so[i][c * 4], a.po + pi * kD + c * 4, v ? 16 : 0);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      acc = fmaf(so[i][d], sw[i], acc);
      L += swl[i];
    }
    __syncthreads();
  }
  const int64_t row = q0 * a.Hq + (int64_t)g * a.G + hl;
  O[row * kD + d] = from_f<OT>(L > 0.f ? acc / L : 0.f);
  if (d == 0) {  // (m_h, 1 / l_h): the score finalize multiplies
    ml[row * 2] = M;
    ml[row * 2 + 1] = L > 0.f ? 1.f / L : 0.f;
  }
}

// ----------------------------------------------------------------------------
// Scores: s_g[j] = sum_{h in group g} exp(x_hj - m_h) / l_h, written to row
// (query, g) at column j.  Persistent grid: block i handles key tiles i,
// i + gridDim.x, ... of kFinKeys keys each (tile = (sequence, key block)).  A
// tile's logits [keys x Hq] are one contiguous span; they are copied into
// shared memory with 16-byte cp.async (row pitch Hq + 4 floats, so the per-key
// reads below are free of bank conflicts), double-buffered so that the copy of
// the next tile overlaps the exponentials of this one.  Thread j scores key j
// of the tile for every KV head; the writes are coalesced along j.
// ----------------------------------------------------------------------------
constexpr int kFinKeys = 128;
constexpr float kLog2e = 1.4426950408889634f;

// Tile -> (sequence, first key); tiles cover ceil(max_len / kFinKeys) blocks
// of every sequence, empty ones are skipped.
__device__ __forceinline__ bool fin_tile(const DecodeArgs& a, int64_t tile, int ntile_seq, int* b,
                                         int64_t* q0, int64_t* kb, int64_t* j0, int* nk) {
  *b = (int)(tile / ntile_seq);
  *j0 = (tile % ntile_seq) * kFinKeys;
  *q0 = __ldg(a.qoff + *b);
  if (__ldg(a.qoff + *b + 1) - *q0 < 1) return false;
  *kb = __ldg(a.kvoff + *b);
  const int64_t N = __ldg(a.kvoff + *b + 1) - *kb;
  if (*j0 >= N) return false;
  *nk = (int)(N - *j0 < kFinKeys ? N - *j0 : kFinKeys);
  return true;
}

__global__ void __launch_bounds__(kFinKeys) k_finalize_scores(const __grid_constant__ DecodeArgs a,
                                                              const float* ml, float* scores,
                                                              int64_t stride, int ntile_seq) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ __align__(16) float fsm[];  // 2 x [kFinKeys][Hq + 4] logits, [Hq][2] stats
  const int Hq = a.Hq, pitch = Hq + 4;
  const int64_t ntiles = (int64_t)a.B * ntile_seq;
  float* buf[2] = {fsm, fsm + (size_t)kFinKeys * pitch};
  float* fst = fsm + 2 * (size_t)kFinKeys * pitch;  // (m_h, 1 / l_h) of the tile's query
  const bool vec = (Hq & 3) == 0;
  const bool vec4 = vec && (a.G & 3) == 0;
  const uint64_t dead = policy_evict_first();  // each logit is read once

  // issue the copy of one tile into buffer k (all threads); a tile whose
  // offsets disagree with the totals copies nothing and is reported
  auto load_tile = [&](int64_t tile, int k) -> bool {
    int b, nk;
    int64_t q0, kb, j0;
    if (!fin_tile(a, tile, ntile_seq, &b, &q0, &kb, &j0, &nk)) return false;
    const int64_t N = __ldg(a.kvoff + b + 1) - kb;
    if (q0 < 0 || q0 >= a.total_q || kb < 0 || kb + N > a.total_kv || N > stride) {
      if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
      return false;
    }
    const float* src = a.logits + (kb + j0) * Hq;
    float* dst = buf[k];
    if (vec) {
      const int per_key = Hq / 4;
      for (int i = threadIdx.x; i < nk * per_key; i += kFinKeys) {
        const int key = i / per_key, c = i % per_key;
        cp_async16_hint(dst + key * pitch + c * 4, src + (int64_t)key * Hq + c * 4, dead);
      }
    } else {
      for (int i = threadIdx.x; i < nk * Hq; i += kFinKeys) dst[(i / Hq) * pitch + i % Hq] = __ldg(src + i);
    }
    return true;
  };

  int64_t tile = blockIdx.x;
  int cur = 0;
  bool have = tile < ntiles && load_tile(tile, 0);
  cp_async_commit();
  while (tile < ntiles) {
    const int64_t next = tile + gridDim.x;
    // next non-empty tile goes into the other buffer while this one is scored
    int64_t nt = next;
    bool nhave = false;
    while (nt < ntiles && !(nhave = load_tile(nt, cur ^ 1))) nt += gridDim.x;
    cp_async_commit();
    if (have) {
      int b, nk;
      int64_t q0, kb, j0;
      fin_tile(a, tile, ntile_seq, &b, &q0, &kb, &j0, &nk);  // checked by load_tile
      {
        // (m_h, 1/l_h) -> (m_h * log2 e, 1/l_h): exp(x - m) = 2^(x log2 e - m log2 e)
        for (int i = threadIdx.x; i < 2 * Hq; i += kFinKeys) {
          const float v = __ldg(ml + q0 * Hq * 2 + i);
          fst[i] = (i & 1) ? v : v * 1.4426950408889634f;
        }
        cp_async_wait_prev();  // this tile's copy has landed (the next may be in flight)
        __syncthreads();
        const int kj = threadIdx.x;
        if (kj < nk) {
          const float* x = buf[cur] + kj * pitch;
          for (int g = 0; g < a.Hkv; ++g) {
            float sc = 0.f;
            if (vec4) {  // 16-byte reads: the row pitch of 9 x 16 bytes spreads 8 lanes over all banks
              for (int h = g * a.G; h < (g + 1) * a.G; h += 4) {
                const float4 v = *reinterpret_cast<const float4*>(x + h);
                sc = fmaf(ex2_approx(fmaf(v.x, kLog2e, -fst[2 * h])), fst[2 * h + 1], sc);
                sc = fmaf(ex2_approx(fmaf(v.y, kLog2e, -fst[2 * h + 2])), fst[2 * h + 3], sc);
                sc = fmaf(ex2_approx(fmaf(v.z, kLog2e, -fst[2 * h + 4])), fst[2 * h + 5], sc);
                sc = fmaf(ex2_approx(fmaf(v.w, kLog2e, -fst[2 * h + 6])), fst[2 * h + 7], sc);
              }
            } else {
              for (int h = g * a.G; h < (g + 1) * a.G; ++h)
                sc = fmaf(ex2_approx(fmaf(x[h], kLog2e, -fst[2 * h])), fst[2 * h + 1], sc);
            }
            scores[(q0 * a.Hkv + g) * stride + j0 + kj] = sc;
          }
        }
      }
    }
    __syncthreads();  // buffer ``cur`` is free again
    tile = nt;
    have = nhave;
    cur ^= 1;
  }
  cp_async_wait_all_groups();
}

}  // namespace hs2
