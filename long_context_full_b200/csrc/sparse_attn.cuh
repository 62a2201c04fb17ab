// sparse_attn.cuh - one Sparse Attention layer of a Hybrid Block: attention of
// the layer's own queries over the rows of the shared KV cache that the
// selection kept (KV Reuse).
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", sections
// "Two-Level KV Sharing" (sparse layers reuse the full-attention layer's cache
// and selection) and "Token-Level Selection and Unified Local Access" (local and
// global tokens come from the one shared cache, in a single sparse computation).
//
// Grid (chunks, rows): the index list of a row (<= k + window entries) is cut
// into chunks of ``chunk`` indices so that every SM has work even at batch 1.
// Each CTA gathers its rows of K and V into shared memory with bulk copies (the
// TMA engine, one 256-byte copy per row and tensor), computes per-warp online
// softmax partials on the tensor cores, and the last CTA of the row (atomic
// ticket, no spinning) merges the partials into O.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

constexpr int kSpWarps = 4;
constexpr int kSpRowBytes = 272;  // 256-byte bf16 row + 16 bytes: conflict-free ldmatrix

struct SparseArgs {
  const void* Q;        // [total_q, Hq, D], this layer's queries
  const void* K;        // [total_kv, Hkv, D]
  const void* V;
  const int32_t* idx;   // [rows, idx_stride]
  const int32_t* count; // [rows]
  int idx_stride;
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hq, Hkv, G;
  int64_t total_q, total_kv;
  float scale;
  int chunk, nchunk;    // indices per CTA, grid.y (grid.x = rows)
  float* pm;            // [rows, nchunk, kSpWarps, G]
  float* pl;
  float* po;            // [rows, nchunk, kSpWarps, G, D]
  uint32_t* ticket;     // [rows], zero on entry
  void* O;              // [total_q, Hq, D]
  int* err;
};

// Last CTA of a row: merge the (nchr x warps) partials into O.  D threads.
template <typename OT>
__device__ void sparse_merge(const SparseArgs& a, int64_t r, int nchr) {
  const int64_t qi = r / a.Hkv;
  const int g = (int)(r % a.Hkv);
  const int d = threadIdx.x;
  if (d >= kD) return;
  OT* O = static_cast<OT*>(a.O);
  for (int hl = 0; hl < a.G; ++hl) {
    float M = -INFINITY;
    for (int c = 0; c < nchr; ++c)
      for (int w = 0; w < kSpWarps; ++w)
        M = fmaxf(M, __ldcg(a.pm + ((r * a.nchunk + c) * kSpWarps + w) * a.G + hl));
    float L = 0.f, acc = 0.f;
    for (int c = 0; c < nchr; ++c)
      for (int w = 0; w < kSpWarps; ++w) {
        const int64_t pi = ((r * a.nchunk + c) * kSpWarps + w) * a.G + hl;
        const float wt = exp_shift(__ldcg(a.pm + pi), M);
        L = fmaf(__ldcg(a.pl + pi), wt, L);
        acc = fmaf(__ldcg(a.po + pi * kD + d), wt, acc);
      }
    O[(qi * a.Hq + (int64_t)g * a.G + hl) * kD + d] = from_f<OT>(L > 0.f ? acc / L : 0.f);
  }
}

// Common prologue: row geometry and this CTA's index range; false = no work.
struct SpRow {
  int64_t r, qi, kv_start, t;
  int g, c, cnt, nchr, j0, n;
};
__device__ __forceinline__ bool sparse_row(const SparseArgs& a, SpRow& s) {
  s.r = blockIdx.x;
  s.c = blockIdx.y;
  s.qi = s.r / a.Hkv;
  s.g = (int)(s.r % a.Hkv);
  const QueryRow q = query_row(a.qoff, a.kvoff, a.B, s.qi);
  s.kv_start = q.kv_start;
  s.t = q.t;
  int cnt = __ldg(a.count + s.r);
  if (cnt < 0 || cnt > a.idx_stride) {
    if (threadIdx.x == 0 && s.c == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    cnt = cnt < 0 ? 0 : a.idx_stride;
  }
  s.cnt = cnt;
  s.nchr = cnt > 0 ? (cnt + a.chunk - 1) / a.chunk : 1;
  if (s.c >= s.nchr) return false;
  s.j0 = s.c * a.chunk;
  const int j1 = s.j0 + a.chunk < cnt ? s.j0 + a.chunk : cnt;
  s.n = j1 > s.j0 ? j1 - s.j0 : 0;
  return true;
}

// Position of index i of the row, or -1 (recorded) if outside 0..t.
__device__ __forceinline__ int64_t sparse_pos(const SparseArgs& a, const SpRow& s, int i) {
  const int64_t pos = __ldg(a.idx + s.r * a.idx_stride + s.j0 + i);
  if (pos < 0 || pos > s.t || s.kv_start + pos >= a.total_kv) {
    record_error(a.err, HS2_ERR_DEVICE_INPUT);
    return -1;
  }
  return pos;
}

template <typename OT>
__device__ __forceinline__ void sparse_finish(const SparseArgs& a, const SpRow& s) {
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket + s.r, 1u) == (uint32_t)(s.nchr - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  sparse_merge<OT>(a, s.r, s.nchr);
  if (threadIdx.x == 0) a.ticket[s.r] = 0u;
}

// ----------------------------------------------------------------------------
// bf16: gathered rows staged by bulk copies, tensor-core S^T = K Q^T and
// O^T += V^T P^T per 16-key slice (same fragment scheme as the decode pass).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * kSpWarps) k_sparse_bf16(const __grid_constant__ SparseArgs a) {
  extern __shared__ __align__(128) uint8_t sp_smem[];
  __shared__ __align__(8) uint64_t bar;
  SpRow s;
  if (!sparse_row(a, s)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* sK = sp_smem;
  uint8_t* sV = sp_smem + (size_t)a.chunk * kSpRowBytes;
  int8_t* valid = reinterpret_cast<int8_t*>(sp_smem + 2 * (size_t)a.chunk * kSpRowBytes);
  const bf16* K = static_cast<const bf16*>(a.K);
  const bf16* V = static_cast<const bf16*>(a.V);

  if (threadIdx.x == 0) {
    mbar_init(&bar, blockDim.x);
    fence_mbar_init();
  }
  __syncthreads();
  // gather: thread i copies rows i, i + 128, ...
  uint32_t bytes = 0;
  for (int i = threadIdx.x; i < s.n; i += blockDim.x) {
    const int64_t pos = sparse_pos(a, s, i);
    valid[i] = pos >= 0;
    if (pos >= 0) bytes += 2 * kD * sizeof(bf16);
  }
  mbar_arrive_expect_tx(&bar, bytes);
  for (int i = threadIdx.x; i < s.n; i += blockDim.x) {
    if (!valid[i]) continue;
    const int64_t pos = __ldg(a.idx + s.r * a.idx_stride + s.j0 + i);
    const int64_t row = (s.kv_start + pos) * a.Hkv + s.g;
    bulk_g2s(sK + (size_t)i * kSpRowBytes, K + row * kD, kD * sizeof(bf16), &bar);
    bulk_g2s(sV + (size_t)i * kSpRowBytes, V + row * kD, kD * sizeof(bf16), &bar);
  }
  // rows past n or invalid must not feed NaNs into the MMAs: zero them
  const int ntile = (s.n + 15) / 16;
  for (int i = threadIdx.x; i < ntile * 16; i += blockDim.x) {
    if (i < s.n && valid[i]) continue;
    uint4* zk = reinterpret_cast<uint4*>(sK + (size_t)i * kSpRowBytes);
    uint4* zv = reinterpret_cast<uint4*>(sV + (size_t)i * kSpRowBytes);
    for (int c = 0; c < 16; ++c) zk[c] = zv[c] = make_uint4(0u, 0u, 0u, 0u);
  }
  const bool landed = mbar_wait(&bar, 0);
  if (!landed) {
    record_error(a.err, HS2_ERR_TIMEOUT);
    mbar_wait(&bar, 0);  // give copies still in flight a second bounded chance to land
  }
  __syncthreads();

  const int r = lane >> 2, qd = lane & 3;
  const int h0 = 2 * qd, h1 = 2 * qd + 1;
  const float NEG = -INFINITY;
  const bf16* Q = static_cast<const bf16*>(a.Q);
  uint32_t qf[8][2];
  const bf16* qrow = Q + ((s.qi * a.Hq) + (int64_t)s.g * a.G + r) * kD;
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
  const uint32_t skb = smem_u32(sK), svb = smem_u32(sV);
  for (int st = warp; landed && st < ntile; st += kSpWarps) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int row = st * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int chunk = kk * 2 + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, skb + row * kSpRowBytes + chunk * 16);
        mma_bf16(c, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      }
    }
    const int ilo = st * 16 + r, ihi = ilo + 8;
    const bool vlo = ilo < s.n && valid[ilo], vhi = ihi < s.n && valid[ihi];
    const float x0 = vlo ? c[0] * a.scale : NEG, x1 = vlo ? c[1] * a.scale : NEG;
    const float x2 = vhi ? c[2] * a.scale : NEG, x3 = vhi ? c[3] * a.scale : NEG;
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
    const int row = st * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int chunk = mt * 2 + ((lane >> 3) & 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(a0, a1, a2, a3, svb + row * kSpRowBytes + chunk * 16);
      mma_bf16(o[mt], a0, a1, a2, a3, b0, b1);
    }
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const int64_t base = ((s.r * a.nchunk + s.c) * kSpWarps + warp) * a.G;
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
  sparse_finish<bf16>(a, s);
}

// ----------------------------------------------------------------------------
// float32 on the CUDA cores: each warp takes every 4th index of the chunk and
// reads its K/V rows directly (lane i holds dims 4i..4i+3).
// ----------------------------------------------------------------------------
template <int GP>
__global__ void __launch_bounds__(32 * kSpWarps) k_sparse_f32(const __grid_constant__ SparseArgs a) {
  SpRow s;
  if (!sparse_row(a, s)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* Q = static_cast<const float*>(a.Q);
  const float* K = static_cast<const float*>(a.K);
  const float* V = static_cast<const float*>(a.V);
  float4 q[GP], o[GP];
  float m[GP], l[GP];
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    q[h] = (h < a.G) ? *reinterpret_cast<const float4*>(Q + ((s.qi * a.Hq) + (int64_t)s.g * a.G + h) * kD + lane * 4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    o[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    m[h] = -INFINITY;
    l[h] = 0.f;
  }
  for (int i = warp; i < s.n; i += kSpWarps) {
    const int64_t pos = sparse_pos(a, s, i);
    if (pos < 0) continue;
    const int64_t row = (s.kv_start + pos) * a.Hkv + s.g;
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
  const int64_t base = ((s.r * a.nchunk + s.c) * kSpWarps + warp) * a.G;
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    if (h >= a.G) break;
    if (lane == 0) { a.pm[base + h] = m[h]; a.pl[base + h] = l[h]; }
    *reinterpret_cast<float4*>(a.po + (base + h) * kD + lane * 4) = o[h];
  }
  sparse_finish<float>(a, s);
}

}  // namespace hs2
