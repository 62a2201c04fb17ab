// chunk_attn.cuh - Full Attention layer of a Hybrid Block for a chunk of new
// query tokens appended to a cached context (agent turns), causal, with the
// per-key selection scores of every query token: shared geometry, and the
// float32 path on the CUDA cores.  The bf16 path runs on the tcgen05 tensor
// cores (chunk_tc.cuh).
//
// Source: "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
// Agents", section "From Hybrid SWA to HySparse2 ..." (one full-attention layer
// per Hybrid Block builds the cache and judges token importance).
//
// Storing per-head logits is out of the question here (Tq x N x Hq floats), so
// the scores take a second pass that recomputes Q K^T with the final softmax
// statistics of the first pass.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

struct ChunkArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hq, Hkv, G, QT;  // QT: query tokens per CTA (128 / G on the tensor cores, 1 for fp32)
  int64_t total_q, total_kv;
  float scale;
  void* O;
  float* ml;              // [total_q, Hq, 2] row max and sum (tcgen05 kernels: max in base 2)
  float* scores;
  int64_t stride;
  int* err;
  // tensor-core kernel, visible keys split over ksplit CTAs per query tile
  // (ksplit = 1: both passes in one CTA, O written directly):
  int ksplit;             // CTAs per query tile; blockIdx.z = sequence * ksplit + split
  int mode;               // 0: both passes; 1: statistics only; 2: scores and O only
  float* part_ml;         // [ksplit][total_q * Hq][2] each split's (max in base 2, sum)
  float* part_o;          // [ksplit][total_q * Hq][D] each split's share of O
};

// Sequence-level geometry of CTA (blockIdx.x = query tile, sequence b).
struct ChTile {
  int64_t q0;       // first query row (packed index) of the tile
  int nq;           // query tokens in the tile
  int64_t kv0;      // first key of the sequence (packed index)
  int64_t N;        // keys of the sequence
  int64_t t0;       // position of the tile's first query
};
__device__ __forceinline__ bool chunk_tile(const ChunkArgs& a, int b, ChTile& c) {
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
// float32 chunk path on the CUDA cores (exact fp32 arithmetic).
// Pass 1: one CTA per (query row, KV group); warp w takes every 4th key.
// ----------------------------------------------------------------------------
template <int GP>
__global__ void __launch_bounds__(128) k_chunk_fwd_f32(const __grid_constant__ ChunkArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
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
  grid_dep_wait();  // the previous kernel on the stream has finished
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
