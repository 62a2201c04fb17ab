// decode_attn.cuh - Full Attention layer of a Hybrid Block for decode (one query
// token per sequence), which also emits the per-key selection scores.
//
// Source: "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
// Agents", section "From Hybrid SWA to HySparse2 ..." (the full-attention layer
// builds the KV cache and decides which tokens are important) and "Xiaomi
// Unveils HySparse2 for Faster Long-Context AI", section "Two-Level KV Sharing".
//
// Two launches:
//   1. k_decode_bf16 / k_decode_f32: split-context pass.  The packed key space
//      of every KV head is cut into P balanced ranges, one per CTA, regardless
//      of sequence boundaries (ragged batches stay balanced).  A CTA streams its
//      K/V rows once, writes the scaled logits x_hj of its keys, and keeps an
//      online-softmax partial (m, l, O) per warp and sequence piece; the bf16
//      pass folds its warps' partials into one per piece before it ends.
//   2. k_finalize_scores: merges the partials of every (sequence, head) into
//      the output O, and computes s_g[j] = sum_{h in g} exp(x_hj - m_h) / l_h
//      over the same CTA ranges as the pass, newest keys first (the logits the
//      pass wrote last are the ones most likely still in L2), staged by bulk
//      copies while the merge runs.
// (k_decode_combine, the merge alone with float O and (m_h, 1/l_h) out, serves
// the context-parallel partial pass.)
// The per-head logits must be stored because the score needs each head's final
// statistics, which are only known after the whole cache has been read; storing
// them (32 B per key and KV head at G = 8) is far cheaper than reading K twice.
// Logits are laid out group-major, [Hkv][total_kv][Gp] with Gp = G rounded up to
// a multiple of 4, so a CTA's logits are one span and every key's row starts
// on a 16-byte boundary.
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
  float* logits;          // [Hkv, total_kv, Gp]
  int Gp;                 // G rounded up to a multiple of 4
  int nw;                 // warp partials per piece that hold data: 1 (bf16, folded) or kDecWarps
  float* pm;              // [(P+B), Hkv, kDecWarps, G]
  float* pl;
  float* po;              // [(P+B), Hkv, kDecWarps, G, D]
  int* err;
};

__host__ __device__ constexpr int logit_pitch(int G) { return (G + 3) & ~3; }

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

// A CTA whose key range is empty (more CTAs than keys) writes, for the
// sequence holding its start, partials that carry nothing (m = -inf, l = 0,
// O = 0), so that the merge of that sequence's CTAs [split_owner(kb),
// split_owner(ke - 1)] - which contains such a CTA only strictly inside a
// sequence - needs no check.  Warp ``w`` of the CTA writes its own slot.
__device__ __forceinline__ void empty_range_partials(const DecodeArgs& a, int p, int g, int w) {
  const int64_t lo = split_lo(a.total_kv, a.P, p), hi = split_lo(a.total_kv, a.P, p + 1);
  if (lo < hi || lo >= a.total_kv) return;
  const int b = last_le(a.kvoff, a.B, lo);
  const int64_t base = ((((int64_t)p + b) * a.Hkv + g) * kDecWarps + w) * a.G;
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < a.G * kD; i += 32) a.po[base * kD + i] = 0.f;
  if (lane < a.G) {
    a.pm[base + lane] = -INFINITY;
    a.pl[base + lane] = 0.f;
  }
}

// ----------------------------------------------------------------------------
// bf16 split-context pass on the tensor cores (mma.sync m16n8k16).
// Per warp and 16-key slice of a tile:  S^T[16 keys x 8 heads] = K Q^T, then
// O^T[128 x 8] += V^T P^T, with P^T obtained from the S^T accumulator by one
// register transpose (movmatrix), so no shared-memory round trip for P.
// Warp 4 is the producer: one lane issues TMA loads into an NST-deep ring.
// ----------------------------------------------------------------------------
// The streaming pass of one CTA (p, g): ``ring`` is the NST-stage K/V ring in
// dynamic shared memory, ``lg`` / ``kstride`` where key j's G logits of group
// g go (lg + j * kstride + head).  Every thread of the CTA calls it; it returns
// once this thread's part is done (the producer lane after its last fill has
// landed).  Returns false if a bounded wait ran out.
template <int NST>
__device__ __forceinline__ bool decode_stream_bf16(const CUtensorMap* tmK, const CUtensorMap* tmV,
                                                   const DecodeArgs& a, uint8_t* ring,
                                                   uint64_t* full_bar, uint64_t* empty_bar,
                                                   float* lg, int64_t kstride) {
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
    if (lane != 0) return true;
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
        tma_load_3d_hint(sk, tmK, &full_bar[stage], 0, g, key, pol);
        tma_load_3d_hint(sk + 8192, tmK, &full_bar[stage], 64, g, key, pol);
        tma_load_3d_hint(sv, tmV, &full_bar[stage], 0, g, key, pol);
        tma_load_3d_hint(sv + 8192, tmV, &full_bar[stage], 64, g, key, pol);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == NST) { stage = 0; phase ^= 1; }
      }
    });
    // drain: every fill this thread issued has landed before the CTA can exit
    for (int s = 0; s < NST; ++s)
      if ((issued >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) {
          record_error(a.err, HS2_ERR_TIMEOUT);
          ok = false;
        }
    return ok;
  }

  // -------------------------------------------------------------- consumers
  empty_range_partials(a, p, g, warp);
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
          if (vlo) st_hint_f2(lg + klo * kstride + h0, x0, x1, keep);
          if (vhi) st_hint_f2(lg + khi * kstride + h0, x2, x3, keep);
        } else {
          if (h0 < a.G) {
            if (vlo) st_hint_f1(lg + klo * kstride + h0, x0, keep);
            if (vhi) st_hint_f1(lg + khi * kstride + h0, x2, keep);
          }
          if (h1 < a.G) {
            if (vlo) st_hint_f1(lg + klo * kstride + h1, x1, keep);
            if (vhi) st_hint_f1(lg + khi * kstride + h1, x3, keep);
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
    // fold the four warps' partials of this piece into warp 0's slot: thread d
    // of the consumers takes dimension d of every head (4x fewer partials for
    // the combine to read)
    named_barrier_sync(1, 32 * kDecWarps);  // every consumer warp's partial is written
    {
      const int d = threadIdx.x;
      const int64_t w0 = (slot * a.Hkv + g) * kDecWarps * a.G;
      float acc[8], mm[8], ll[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        acc[h] = 0.f;
        mm[h] = NEG;
        ll[h] = 0.f;
        if (h < a.G) {
          float mw[kDecWarps];
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            mw[w] = a.pm[w0 + w * a.G + h];
            mm[h] = fmaxf(mm[h], mw[w]);
          }
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            const float f = exp_shift(mw[w], mm[h]);
            acc[h] = fmaf(f, a.po[(w0 + w * a.G + h) * kD + d], acc[h]);
            ll[h] = fmaf(f, a.pl[w0 + w * a.G + h], ll[h]);
          }
        }
      }
      named_barrier_sync(1, 32 * kDecWarps);  // every read of the four slots is done
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h < a.G) {
          a.po[(w0 + h) * kD + d] = acc[h];
          if (d == 0) {
            a.pm[w0 + h] = mm[h];
            a.pl[w0 + h] = ll[h];
          }
        }
      }
    }
  });
  return ok;
}

// Split-context pass as its own launch (the combine and the score finalize
// follow as separate kernels).
template <int NST>
__global__ void __launch_bounds__(32 * (kDecWarps + 1))
    k_decode_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ DecodeArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[NST];
  __shared__ __align__(8) uint64_t empty_bar[NST];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  decode_stream_bf16<NST>(&tmK, &tmV, a, ring, full_bar, empty_bar,
                          a.logits + (int64_t)blockIdx.y * a.total_kv * a.Gp, a.Gp);
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
  empty_range_partials(a, p, g, warp);
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
        if (lane == 0) a.logits[((int64_t)g * a.total_kv + j) * a.Gp + h] = x;
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
// Combine: O and (m_h, 1/l_h) of one (sequence, head) per CTA from the partials
// of every CTA whose key range meets the sequence (nw per CTA piece).  Eight
// warps: the partials' maxima and weights are computed lane-parallel and kept
// in shared memory, then warp w sums partials w, w + 8, ... with each lane on
// four dimensions (16-byte loads, several partials in flight per lane).
// ----------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombCap = 1024;  // partial weights staged per round

template <typename OT>
__global__ void __launch_bounds__(kCombThreads) k_decode_combine(const __grid_constant__ DecodeArgs a, OT* O,
                                                                 float* ml) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  __shared__ float wsh[kCombCap];
  __shared__ float red[kCombThreads / 32];
  __shared__ __align__(16) float4 osh[kCombThreads / 32][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kCombThreads / 32;
  const int64_t item = blockIdx.x;
  const int b = (int)(item / a.Hq), h = (int)(item % a.Hq);
  const int g = h / a.G, hl = h % a.G;
  if (item == 0 && threadIdx.x == 0) {
    if (__ldg(a.kvoff + a.B) != a.total_kv || __ldg(a.qoff + a.B) != a.total_q)
      record_error(a.err, HS2_ERR_DEVICE_INPUT);
  }
  const int64_t q0 = __ldg(a.qoff + b);
  const int64_t qn = __ldg(a.qoff + b + 1) - q0;
  if (qn < 1) return;
  if (qn > 1 || q0 < 0 || q0 >= a.total_q) {
    if (threadIdx.x == 0 && hl == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    return;
  }
  const int64_t W = a.total_kv;
  const int64_t kb = __ldg(a.kvoff + b), ke = __ldg(a.kvoff + b + 1);
  int pf = 0, np = 0;
  if (ke > kb) {
    pf = split_owner(W, a.P, kb);
    np = (split_owner(W, a.P, ke - 1) - pf + 1) * a.nw;
  }
  // partial i = (CTA pf + i / nw, warp i % nw); CTAs with an empty range wrote
  // neutral partials (empty_range_partials)
  auto pidx = [&](int i) -> int64_t {
    return (((int64_t)(pf + i / a.nw + b) * a.Hkv + g) * kDecWarps + (i % a.nw)) * a.G + hl;
  };
  // ---- the maximum over the partials
  float M = -INFINITY;
  for (int i = threadIdx.x; i < np; i += kCombThreads) M = fmaxf(M, __ldcg(a.pm + pidx(i)));
  M = warp_max(M);
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  // ---- per round of kCombCap partials: weights, then the weighted O rows
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < np; c0 += kCombCap) {
    const int n = min(kCombCap, np - c0);
    for (int i = threadIdx.x; i < n; i += kCombThreads) {
      const int64_t pi = pidx(c0 + i);
      const float w = exp_shift(__ldcg(a.pm + pi), M);
      L = fmaf(w, __ldcg(a.pl + pi), L);
      wsh[i] = w;
    }
    __syncthreads();
    constexpr int U = 4;
    for (int i0 = warp; i0 < n; i0 += NW * U) {
      float4 o[U];
      float wt[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * NW;
        wt[u] = i < n ? wsh[i] : 0.f;
        o[u] = wt[u] != 0.f ? __ldcg(reinterpret_cast<const float4*>(a.po + pidx(c0 + i) * kD) + lane)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        acc.x = fmaf(wt[u], o[u].x, acc.x);
        acc.y = fmaf(wt[u], o[u].y, acc.y);
        acc.z = fmaf(wt[u], o[u].z, acc.z);
        acc.w = fmaf(wt[u], o[u].w, acc.w);
      }
    }
    __syncthreads();  // wsh is refilled by the next round
  }
  L = warp_sum(L);
  osh[warp][lane] = acc;
  __syncthreads();  // red[] is free again: the maxima were read before the rounds
  if (lane == 0) red[warp] = L;
  __syncthreads();
  if (warp == 0) {
    float Lt = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      Lt += red[w];
      const float4 v = osh[w][lane];
      o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
    }
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    const int64_t row = q0 * a.Hq + h;
    OT* dst = O + row * kD + lane * 4;
    dst[0] = from_f<OT>(o.x * inv);
    dst[1] = from_f<OT>(o.y * inv);
    dst[2] = from_f<OT>(o.z * inv);
    dst[3] = from_f<OT>(o.w * inv);
    if (lane == 0) {  // (m_h, 1 / l_h): the score finalize multiplies
      ml[row * 2] = M;
      ml[row * 2 + 1] = inv;
    }
  }
}

// ----------------------------------------------------------------------------
// Finish of the decode call: the combine and the scores in one launch.
// Scores: s_g[j] = sum_{h in group g} exp(x_hj - m_h) / l_h, written to row
// (query, g) at column j.  Grid (P, Hkv): CTA (p, g) takes the key range of the
// pass's CTA (p, g), its pieces last first and each piece's keys from the top
// down, so the logits written last are read first.  Warp 8 (one lane) streams
// the logits into a ring of kFinStages stages of kFinChunk keys with untiled
// bulk copies (the TMA engine; a chunk's span is contiguous and starts on a
// 16-byte boundary since Gp is a multiple of 4), from the start of the kernel.
// Meanwhile warps 0-7:
//   1. (ml_in == null) merge the partials of the (sequence, head) items
//      c, c + P*Hkv, ... into O, as k_decode_combine does;
//   2. for each piece: the final (m_h, l_h) of the group's G heads, from the
//      partials (lane-parallel, one warp per head) or from ml_in;
//   3. score kFinChunk / 256 keys per thread per stage, the writes coalesced
//      along j.
// ----------------------------------------------------------------------------
constexpr int kFinChunk = 1024;
constexpr int kFinStages = 3;
constexpr int kFinWarps = 8;
constexpr int kFinThreads = 32 * (kFinWarps + 1);
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr size_t finalize_smem(int G) {
  return (size_t)kFinStages * kFinChunk * logit_pitch(G) * sizeof(float);
}

// Walks the pieces of CTA p's key range last first; f(b, s, e, q0) as for_each_piece.
template <typename F>
__device__ __forceinline__ void for_each_piece_rev(const DecodeArgs& a, int p, F f) {
  const int64_t W = a.total_kv;
  const int64_t lo = split_lo(W, a.P, p), hi = split_lo(W, a.P, p + 1);
  if (lo >= hi) return;
  for (int b = last_le(a.kvoff, a.B, hi - 1); b >= 0; --b) {
    const int64_t kb = __ldg(a.kvoff + b), ke = __ldg(a.kvoff + b + 1);
    if (ke <= lo) break;
    const int64_t s = kb > lo ? kb : lo, e = ke < hi ? ke : hi;
    if (s >= e) continue;
    const int64_t q0 = __ldg(a.qoff + b), qn = __ldg(a.qoff + b + 1) - q0;
    if (qn < 1) continue;
    if (q0 < 0 || q0 >= a.total_q) continue;  // inconsistent offsets: reported with the O items
    f(b, s, e, q0);
  }
}

// One untiled bulk copy global -> this CTA's shared memory with an L2 policy,
// completion counted on ``bar``; 16-byte aligned addresses, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                               uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// The CTAs whose key range meets sequence b: [*pf, *pf + *pn).
__device__ __forceinline__ void seq_owners(const DecodeArgs& a, int b, int* pf, int* pn) {
  const int64_t W = a.total_kv;
  const int64_t kb = __ldg(a.kvoff + b), ke = __ldg(a.kvoff + b + 1);
  *pf = 0;
  *pn = 0;
  if (ke > kb) {
    *pf = split_owner(W, a.P, kb);
    *pn = split_owner(W, a.P, ke - 1) - *pf + 1;
  }
}

// Index of partial i (= CTA pf + i / nw, warp i % nw) of (sequence b, KV head
// g, head hl).  A CTA with an empty key range wrote a neutral partial.
__device__ __forceinline__ int64_t partial_at(const DecodeArgs& a, int b, int g, int hl, int pf, int i) {
  const int p = pf + i / a.nw;
  return (((int64_t)(p + b) * a.Hkv + g) * kDecWarps + (i % a.nw)) * a.G + hl;
}

// Final (m, l) of one head from its np partials; one warp, every lane returns it.
__device__ __forceinline__ void head_stats(const DecodeArgs& a, int b, int g, int hl, int pf, int np,
                                           float* Mo, float* Lo) {
  const int lane = threadIdx.x & 31;
  constexpr int R = 4;  // partials a lane keeps in registers (np <= 128: one load each)
  float mv[R], lv[R];
  float M = -INFINITY;
#pragma unroll
  for (int u = 0; u < R; ++u) {
    const int i = u * 32 + lane;
    mv[u] = -INFINITY;
    lv[u] = 0.f;
    if (i < np) {
      const int64_t pi = partial_at(a, b, g, hl, pf, i);
      mv[u] = __ldcg(a.pm + pi);
      lv[u] = __ldcg(a.pl + pi);
    }
  }
  for (int i = R * 32 + lane; i < np; i += 32) M = fmaxf(M, __ldcg(a.pm + partial_at(a, b, g, hl, pf, i)));
#pragma unroll
  for (int u = 0; u < R; ++u) M = fmaxf(M, mv[u]);
  M = warp_max(M);
  float L = 0.f;
#pragma unroll
  for (int u = 0; u < R; ++u) L = fmaf(exp_shift(mv[u], M), lv[u], L);
  for (int i = R * 32 + lane; i < np; i += 32) {
    const int64_t pi = partial_at(a, b, g, hl, pf, i);
    L = fmaf(exp_shift(__ldcg(a.pm + pi), M), __ldcg(a.pl + pi), L);
  }
  *Mo = M;
  *Lo = warp_sum(L);
}

template <typename OT>
__global__ void __launch_bounds__(kFinThreads) k_finalize_scores(const __grid_constant__ DecodeArgs a, OT* O,
                                                                 const float* ml_in, float* scores,
                                                                 int64_t stride) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ __align__(128) float fring[];
  __shared__ __align__(8) uint64_t full_bar[kFinStages], empty_bar[kFinStages];
  __shared__ __align__(16) float4 osh[kFinWarps][32];
  __shared__ float red[kFinWarps], redm[kFinWarps];
  __shared__ float cm[16], cl[16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x, g = blockIdx.y;
  const int G = a.G, Gp = a.Gp;
  const float* lg = a.logits + (int64_t)g * a.total_kv * Gp;
  const int stage_floats = kFinChunk * Gp;
  constexpr int NC = 32 * kFinWarps;  // consumer threads
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFinStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kFinWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  // a piece whose offsets disagree with the score stride or the cache is skipped
  // by both roles alike
  auto piece_ok = [&](int b) {
    const int64_t kb = __ldg(a.kvoff + b), N = __ldg(a.kvoff + b + 1) - kb;
    return kb >= 0 && N <= stride && kb + N <= a.total_kv;
  };

  if (warp == kFinWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t dead = policy_evict_first();  // each logit is read once
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    bool ok = true;
    for_each_piece_rev(a, p, [&](int b, int64_t s, int64_t e, int64_t q0) {
      if (!piece_ok(b)) return;
      for (int64_t top = e; top > s && ok; top -= kFinChunk) {
        const int64_t j0 = top - kFinChunk > s ? top - kFinChunk : s;
        if (!mbar_wait(&empty_bar[stage], phase ^ 1)) {
          record_error(a.err, HS2_ERR_TIMEOUT);
          ok = false;
          break;
        }
        const uint32_t bytes = (uint32_t)((top - j0) * Gp * sizeof(float));
        mbar_arrive_expect_tx(&full_bar[stage], bytes);
        bulk_load_hint(fring + stage * stage_floats, lg + j0 * Gp, bytes, &full_bar[stage], dead);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kFinStages) { stage = 0; phase ^= 1; }
      }
    });
    // drain: every copy issued here has landed before the CTA can exit
    for (int s = 0; s < kFinStages; ++s)
      if ((issued >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) record_error(a.err, HS2_ERR_TIMEOUT);
    return;
  }

  // ------------------------------------------------- consumers: 1. O items
  if (!ml_in) {
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x, nct = gridDim.x * gridDim.y;
    if (cta == 0 && threadIdx.x == 0) {
      if (__ldg(a.kvoff + a.B) != a.total_kv || __ldg(a.qoff + a.B) != a.total_q)
        record_error(a.err, HS2_ERR_DEVICE_INPUT);
    }
    for (int64_t it = cta; it < (int64_t)a.B * a.Hq; it += nct) {
      const int b = (int)(it / a.Hq), h = (int)(it % a.Hq);
      const int gi = h / G, hl = h % G;
      const int64_t q0 = __ldg(a.qoff + b), qn = __ldg(a.qoff + b + 1) - q0;
      if (qn < 1) continue;  // a sequence without a query row (uniform over the CTA)
      if (qn > 1 || q0 < 0 || q0 >= a.total_q) {
        if (threadIdx.x == 0 && hl == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
        continue;
      }
      int pf, pn;
      seq_owners(a, b, &pf, &pn);
      const int np = pn * a.nw;
      // warp w merges partials w, w + 8, ... with a running maximum, U of them
      // loaded at once (m, l and its 16 bytes of O per lane), then warp 0
      // merges the eight warps' results
      float M = -INFINITY, L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      constexpr int U = 8;
      for (int i0 = warp; i0 < np; i0 += kFinWarps * U) {
        float mv[U], lv[U];
        float4 ov[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * kFinWarps;
          mv[u] = -INFINITY;
          lv[u] = 0.f;
          ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < np) {
            const int64_t pi = partial_at(a, b, gi, hl, pf, i);
            mv[u] = __ldcg(a.pm + pi);
            lv[u] = __ldcg(a.pl + pi);
            ov[u] = __ldcg(reinterpret_cast<const float4*>(a.po + pi * kD) + lane);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float Mn = fmaxf(M, mv[u]);
          const float so = exp_shift(M, Mn), w = exp_shift(mv[u], Mn);
          L = fmaf(L, so, w * lv[u]);
          acc.x = fmaf(acc.x, so, w * ov[u].x);
          acc.y = fmaf(acc.y, so, w * ov[u].y);
          acc.z = fmaf(acc.z, so, w * ov[u].z);
          acc.w = fmaf(acc.w, so, w * ov[u].w);
          M = Mn;
        }
      }
      osh[warp][lane] = acc;
      if (lane == 0) {
        red[warp] = L;
        redm[warp] = M;
      }
      named_barrier_sync(1, NC);
      if (warp == 0) {
        float Mt = redm[0];
#pragma unroll
        for (int w = 1; w < kFinWarps; ++w) Mt = fmaxf(Mt, redm[w]);
        float Lt = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kFinWarps; ++w) {
          const float f = exp_shift(redm[w], Mt);
          Lt = fmaf(f, red[w], Lt);
          const float4 v = osh[w][lane];
          o.x = fmaf(f, v.x, o.x); o.y = fmaf(f, v.y, o.y); o.z = fmaf(f, v.z, o.z); o.w = fmaf(f, v.w, o.w);
        }
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        OT* dst = O + (q0 * a.Hq + h) * kD + lane * 4;
        dst[0] = from_f<OT>(o.x * inv);
        dst[1] = from_f<OT>(o.y * inv);
        dst[2] = from_f<OT>(o.z * inv);
        dst[3] = from_f<OT>(o.w * inv);
      }
      named_barrier_sync(1, NC);  // osh / red are reused by the next item
    }
  }

  // --------------------------------------- consumers: 2-3. statistics, scores
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  for_each_piece_rev(a, p, [&](int b, int64_t s, int64_t e, int64_t q0) {
    if (!piece_ok(b)) {
      if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
      return;
    }
    const int64_t kb = __ldg(a.kvoff + b);
    if (ml_in) {
      if (threadIdx.x < G) {
        const int64_t row = q0 * a.Hq + (int64_t)g * G + threadIdx.x;
        cm[threadIdx.x] = __ldg(ml_in + row * 2) * kLog2e;
        cl[threadIdx.x] = __ldg(ml_in + row * 2 + 1);
      }
    } else {
      int pf, pn;
      seq_owners(a, b, &pf, &pn);
      for (int hl = warp; hl < G; hl += kFinWarps) {
        float M, L;
        head_stats(a, b, g, hl, pf, pn * a.nw, &M, &L);
        if (lane == 0) {
          cm[hl] = M * kLog2e;
          cl[hl] = L > 0.f ? 1.f / L : 0.f;
        }
      }
    }
    named_barrier_sync(1, NC);
    float mh[16], il[16];  // (m_h log2 e, 1 / l_h) of the group's heads
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      mh[i] = i < G ? cm[i] : 0.f;
      il[i] = i < G ? cl[i] : 0.f;
    }
    named_barrier_sync(1, NC);  // cm / cl are rewritten by the next piece
    float* out = scores + (q0 * a.Hkv + g) * stride - kb;  // indexed by packed key j
    for (int64_t top = e; top > s; top -= kFinChunk) {
      const int64_t j0 = top - kFinChunk > s ? top - kFinChunk : s;
      if (ok && !mbar_wait(&full_bar[stage], phase)) {
        record_error(a.err, HS2_ERR_TIMEOUT);
        ok = false;
      }
      if (ok) {
        const float* x = fring + stage * stage_floats;
        const int n = (int)(top - j0);
#pragma unroll
        for (int u = 0; u < kFinChunk / NC; ++u) {
          const int i = n - 1 - (u * NC + (int)threadIdx.x);
          if (i >= 0) {
            const float* xr = x + i * Gp;
            float sc = 0.f;
            if (Gp == 8) {
              const float4 v0 = reinterpret_cast<const float4*>(xr)[0];
              const float4 v1 = reinterpret_cast<const float4*>(xr)[1];
              const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
              for (int hh = 0; hh < 8; ++hh)
                if (hh < G) sc = fmaf(ex2_approx(fmaf(v[hh], kLog2e, -mh[hh])), il[hh], sc);
            } else {
#pragma unroll
              for (int hh = 0; hh < 16; ++hh)
                if (hh < G) sc = fmaf(ex2_approx(fmaf(xr[hh], kLog2e, -mh[hh])), il[hh], sc);
            }
            out[j0 + i] = sc;
          }
        }
        // The chunk's logits, written by this call's pass, are dead once copied
        // in: drop the L2 lines wholly inside it (no other chunk reads them), so
        // those still held in L2 are never written back to DRAM.  (With ml_in
        // the logits belong to the caller's workspace and are left alone.)
        if (!ml_in) {
          const uintptr_t lo = (reinterpret_cast<uintptr_t>(lg + j0 * Gp) + 127) & ~uintptr_t(127);
          const uintptr_t hi = reinterpret_cast<uintptr_t>(lg + top * Gp) & ~uintptr_t(127);
          for (uintptr_t l = lo + (uintptr_t)threadIdx.x * 128; l < hi; l += (uintptr_t)NC * 128)
            discard_l2(reinterpret_cast<const void*>(l));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[stage]);
      if (++stage == kFinStages) { stage = 0; phase ^= 1; }
    }
  });
}

}  // namespace hs2
