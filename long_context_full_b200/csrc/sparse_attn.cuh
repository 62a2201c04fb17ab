// sparse_attn.cuh - one Sparse Attention layer of a Hybrid Block: attention of
// the layer's own queries over the rows of the shared KV cache that the
// selection kept (KV Reuse).
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", sections
// "Two-Level KV Sharing" (sparse layers reuse the full-attention layer's cache
// and selection) and "Token-Level Selection and Unified Local Access" (local and
// global tokens come from the one shared cache, in a single sparse computation).
//
// Few rows (decode): one thread-block cluster of 8 CTAs (16 when the rows are
// few) per (query, KV group) row.  CTA c takes the c-th share of the row's
// index list and reads those K/V rows - bf16: K by TMA gather4 instructions,
// four rows of a 2-D (position, KV head) x 128 tensor map each, in 64-column
// halves with the 128-byte swizzle, and V at the same time by every thread's
// 16-byte cp.async copies into the same layout; fp32: each warp loads its rows straight into
// registers, 16 bytes per lane - runs an online softmax per warp (tensor cores
// for bf16), folds its warps into one partial,
// and the cluster merges the partials through distributed shared memory, CTA c
// finishing the heads h = c mod kSpCluster after a single cluster barrier.  No
// workspace, no global round trip, no atomics.
// Many rows (a chunk of queries, bf16): one CTA per row, the rows taken KV
// head by KV head (the CTAs resident at once then share one head's part of the
// cache, which mostly stays in L2), each warp streaming its own slices through
// a private ring with 16-byte cp.async copies; there the rows mostly come from
// L2, where per-lane copies keep up better than one TMA request per 256-byte
// row.
//
// The same kernels run the sliding-window layer of the Hybrid SWA baseline
// ("Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for Agents",
// section "From Hybrid SWA to HySparse2, ..."): window mode replaces the index
// list by the contiguous positions max(0, t-window+1) .. t.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "ptx.cuh"

namespace hs2 {

namespace cg = cooperative_groups;

constexpr int kSpWarps = 4;
constexpr int kSpCluster = 8;     // CTAs per row (16 when the rows are few)
constexpr int kSpRowBytes = 272;  // fp32 / row kernels: 256-byte row + 16 bytes, conflict-free ldmatrix
constexpr int kSpPiece = 144;     // gathered rows staged per round (9 slices of 16: a
                                  // 1152-entry list over 8 CTAs in one round, and two
                                  // CTAs fit on an SM)

struct SparseArgs {
  const void* Q;        // [total_q, Hq, D], this layer's queries
  const void* K;        // [total_kv, Hkv, D]
  const void* V;
  const int32_t* idx;   // [rows, idx_stride] (index mode)
  const int32_t* count; // [rows] (index mode)
  int idx_stride;
  int window;           // > 0: window mode, positions max(0, t-window+1) .. t, no index list
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hq, Hkv, G;
  int64_t total_q, total_kv;
  float scale;
  void* O;              // [total_q, Hq, D]
  int* err;
  // context-parallel partials (all zero / null otherwise):
  const int64_t* pos0;  // [B]: the list holds global positions; this rank's local key 0 of
                        // sequence b is global position pos0[b]; entries outside the rank's
                        // rows are skipped without an error
  float* ml_out;        // [total_q, Hq, 2]: (m, 1/l) of each (query, head), 1/l = 0 if no key
  int o_f32;            // 1: O is float32 whatever the input type
};

// This CTA's share of a row: indices [j0, j0 + n) of the row's list.
struct SpRow {
  int64_t r, qi, kv_start, t, pos0;
  int g, cnt, j0, n;
};
// The share of a CTA of a cs-CTA cluster: list entries [rank * per, ...),
// per = ceil(cnt / cs) rounded up to 16.
__device__ __forceinline__ int sparse_share(int cnt, int cs) { return ((cnt + cs - 1) / cs + 15) / 16 * 16; }

// group_major: CTA (cluster) i takes row (query i % total_q, KV head i /
// total_q), so the CTAs that run at the same time gather from one KV head's
// part of the cache (it then mostly stays in L2); otherwise row i.
// block_search: the whole CTA calls it and finds the query's sequence with
// query_row_block.
__device__ __forceinline__ SpRow sparse_row(const SparseArgs& a, int rank, int cs, bool group_major = false,
                                            bool block_search = false) {
  SpRow s;
  const int64_t i = blockIdx.x / cs;
  if (group_major) {
    s.qi = i % a.total_q;
    s.g = (int)(i / a.total_q);
    s.r = s.qi * a.Hkv + s.g;
  } else {
    s.r = i;
    s.qi = s.r / a.Hkv;
    s.g = (int)(s.r % a.Hkv);
  }
  const int cnt_in = a.window > 0 ? 0 : __ldg(a.count + s.r);  // independent of the search
  const QueryRow q = block_search ? query_row_block(a.qoff, a.kvoff, a.B, s.qi)
                                  : query_row(a.qoff, a.kvoff, a.B, s.qi);
  s.kv_start = q.kv_start;
  s.t = q.t;
  s.pos0 = a.pos0 ? __ldg(a.pos0 + q.b) : 0;
  int cnt;
  if (a.window > 0) {  // sliding window: the last min(window, t + 1) positions
    cnt = (int)(s.t + 1 < 0 ? 0 : (s.t + 1 < a.window ? s.t + 1 : a.window));
  } else {
    cnt = cnt_in;
    if (cnt < 0 || cnt > a.idx_stride) {
      if (threadIdx.x == 0 && rank == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
      cnt = cnt < 0 ? 0 : a.idx_stride;
    }
  }
  s.cnt = cnt;
  const int per = sparse_share(cnt, cs);
  s.j0 = rank * per;
  s.n = cnt - s.j0 < 0 ? 0 : (cnt - s.j0 < per ? cnt - s.j0 : per);
  return s;
}

// Cache position of a list entry's value ``pos`` (index mode), or -1
// (recorded) if outside 0..t.
__device__ __forceinline__ int64_t sparse_checked(const SparseArgs& a, const SpRow& s, int64_t pos, bool record) {
  if (a.pos0) {  // a global position: another rank's row is skipped, not an error
    pos -= s.pos0;
    if (pos < 0 || pos > s.t) return -1;
  }
  if (pos < 0 || pos > s.t || s.kv_start + pos < 0 || s.kv_start + pos >= a.total_kv) {
    if (record) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    return -1;
  }
  return pos;
}

// Cache position of list entry i of the CTA's share (window mode: the i-th
// position of the window), or -1 (recorded) if outside 0..t.
__device__ __forceinline__ int64_t sparse_pos(const SparseArgs& a, const SpRow& s, int i,
                                              bool record) {
  const int64_t pos =
      a.window > 0 ? s.t - s.cnt + 1 + s.j0 + i : __ldg(a.idx + s.r * a.idx_stride + s.j0 + i);
  return sparse_checked(a, s, pos, record);
}

// Partials received by the CTA that finishes a head: one slot per source CTA
// and per owned head (heads h with h % cs == rank), slot (c, s) at index
// c * (kSpSlots / cs) + s.  A cluster of cs CTAs (8 or 16) leaves each CTA at
// most kSpSlots / cs heads for G <= 16.
constexpr int kSpSlots = 16;
struct SpRecv {
  float m[kSpSlots];
  float l[kSpSlots];
  float o[kSpSlots][kD];
};

constexpr int kSpHalfBytes = kSpPiece * 128;  // bf16 cluster kernel: 64 columns of the staged rows
constexpr size_t kSpGatherSmem = 4 * (size_t)kSpHalfBytes + (size_t)kSpPiece * 8 + 1024;  // + alignment

// Four rows of a 2-D tensor map (box: 64 columns x 1 row, 128-byte swizzle)
// gathered by one TMA instruction into 4 x 128 bytes at ``dst``, completion
// counted on ``bar``: rows r0..r3, columns c0 .. c0 + 63 (c0 a multiple of 64).
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int r0,
                                            int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

// Cluster merge.  Each CTA folds its warps' partials (wm/wl [kSpWarps][GMAX],
// wo [kSpWarps][GMAX][D]) into one partial per head and pushes it into the
// shared memory of CTA h % cs (distributed shared memory stores); one cluster
// barrier makes them visible, and each CTA finishes its own heads from local
// memory.  Nothing is read remotely after the barrier, so it is the only one.
// The softmax weights exp(m_i - M) are computed once each (thread h for head
// h's warps, thread c for source CTA c) and shared, so every thread then only
// sums its own dimension d.  D threads.
template <typename OT, int GMAX>
__device__ __forceinline__ void sparse_cluster_merge(const SparseArgs& a, int64_t qi, int g,
                                                     cg::cluster_group& cl, int rank, int cs,
                                                     const float* wm, const float* wl,
                                                     const float* wo, SpRecv& recv) {
  __shared__ float wt[kSpWarps * GMAX];        // warp weights per head
  __shared__ float hm[GMAX], hl[GMAX];         // this CTA's (M, L) per head
  __shared__ float ct[kSpSlots];               // source-CTA weights per owned head
  const int d = threadIdx.x;
  if (d < a.G) {
    const int h = d;
    float M = -INFINITY;
    for (int w = 0; w < kSpWarps; ++w) M = fmaxf(M, wm[w * GMAX + h]);
    float L = 0.f;
    for (int w = 0; w < kSpWarps; ++w) {
      const float e = exp_shift(wm[w * GMAX + h], M);
      wt[w * GMAX + h] = e;
      L = fmaf(wl[w * GMAX + h], e, L);
    }
    hm[h] = M;
    hl[h] = L;
  }
  __syncthreads();
  for (int h = 0; h < a.G; ++h) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kSpWarps; ++w) acc = fmaf(wo[(w * GMAX + h) * kD + d], wt[w * GMAX + h], acc);
    SpRecv* dst = cl.map_shared_rank(&recv, h % cs);
    const int at = rank * (kSpSlots / cs) + h / cs;
    dst->o[at][d] = acc;
    if (d == 0) {
      dst->m[at] = hm[h];
      dst->l[at] = hl[h];
    }
  }
  cl.sync();
  // owned heads h = rank, rank + cs, ...: slot (h - rank) / cs
  const int nown = a.G > rank ? (a.G - rank + cs - 1) / cs : 0;
  const int per = kSpSlots / cs;
  if (d < nown * cs) {
    const int slot = d / cs, c = d % cs;
    float M = -INFINITY;
    for (int c2 = 0; c2 < cs; ++c2) M = fmaxf(M, recv.m[c2 * per + slot]);
    ct[d] = exp_shift(recv.m[c * per + slot], M);
  }
  __syncthreads();
  OT* O = static_cast<OT*>(a.O);
  for (int h = rank; h < a.G; h += cs) {
    const int slot = h / cs;
    float L = 0.f, acc = 0.f;
    for (int c = 0; c < cs; ++c) {
      const float e = ct[slot * cs + c];
      L = fmaf(recv.l[c * per + slot], e, L);
      acc = fmaf(recv.o[c * per + slot][d], e, acc);
    }
    const int64_t orow = qi * a.Hq + (int64_t)g * a.G + h;
    O[orow * kD + d] = from_f<OT>(L > 0.f ? acc / L : 0.f);
    if (a.ml_out && d == 0) {
      float M = -INFINITY;
      for (int c = 0; c < cs; ++c) M = fmaxf(M, recv.m[c * per + slot]);
      a.ml_out[orow * 2] = M;
      a.ml_out[orow * 2 + 1] = L > 0.f ? 1.f / L : 0.f;
    }
  }
}

// ----------------------------------------------------------------------------
// bf16: tensor-core S^T = K Q^T and O^T += V^T P^T per 16-key slice, the same
// fragment scheme as the decode pass (P^T by one movmatrix transpose).
// One arrival on ``bar`` once every cp.async this thread has issued so far has
// landed; the barrier's expected count includes it.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * kSpWarps) k_sparse_bf16(const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ SparseArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ uint8_t sp_dyn[];
  __shared__ float wm[kSpWarps * 8], wl[kSpWarps * 8];
  __shared__ float wo[kSpWarps * 8 * kD];
  __shared__ SpRecv recv;
  __shared__ __align__(8) uint64_t gbar[2];  // one per copy group, one phase per piece
  cg::cluster_group cl = cg::this_cluster();
  const int cs = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  if (threadIdx.x == 0) {
    // thread 0 arrives with the bytes of the group's K copies, and every
    // thread once its own V copies of the group have landed
    mbar_init(&gbar[0], 1 + blockDim.x);
    mbar_init(&gbar[1], 1 + blockDim.x);
    fence_mbar_init();
  }
  // the list entries of this CTA's share when the list is full (count ==
  // idx_stride, the usual case), loaded before the count is known
  int64_t spec[2] = {-1, -1};
  const int per_full = sparse_share(a.idx_stride, cs);
  if (a.window == 0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = rank * per_full + (int)threadIdx.x + u * (int)blockDim.x;
      if ((int)threadIdx.x + u * (int)blockDim.x < per_full && e < a.idx_stride)
        spec[u] = __ldg(a.idx + (int64_t)(blockIdx.x / cs) * a.idx_stride + e);
    }
  }
  const SpRow s = sparse_row(a, rank, cs, false, true);
  const bool spec_ok = a.window == 0 && s.j0 == rank * per_full && per_full <= 2 * (int)blockDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // staged rows: K and V, each as two [kSpPiece][128 B] halves (columns 0-63,
  // 64-127) in the 128-byte swizzle of the tensor maps, bases 1024-aligned
  uint8_t* sp_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sp_dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sp_smem;
  uint8_t* sV = sp_smem + 2 * (size_t)kSpHalfBytes;
  int64_t* spos = reinterpret_cast<int64_t*>(sp_smem + 4 * (size_t)kSpHalfBytes);
  const int64_t map_rows = a.total_kv * a.Hkv;  // rows of the 2-D maps: (position, KV head)

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

  for (int p0 = 0, piece = 0; p0 < s.n; p0 += kSpPiece, ++piece) {
    const int pn = s.n - p0 < kSpPiece ? s.n - p0 : kSpPiece;
    const int ntile = (pn + 15) / 16;
    // the piece's cache rows (-1: past the list or invalid), read once
    for (int row = threadIdx.x, u = 0; row < ntile * 16; row += blockDim.x, ++u) {
      int64_t pos = -1;
      if (row < pn)
        pos = (spec_ok && p0 == 0 && u < 2) ? sparse_checked(a, s, u == 0 ? spec[0] : spec[1], true)
                                              : sparse_pos(a, s, p0 + row, true);
      spos[row] = pos;
    }
    __syncthreads();
    // gather: K by TMA, one gather4 per 4 rows and per 64-column half; V by
    // 16-byte cp.async copies of every thread into the same swizzled layout,
    // so the TMA engine and the load/store units fetch at the same time (rows
    // past pn or with an invalid index load a row of the sequence that is then
    // masked out).  Two copy groups on their own barriers: the first half of
    // the slices is scored while the second half is still in flight.  Thread 0
    // arrives on each group with its K byte count before any copy.
    const int nA = (ntile + 1) / 2;
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&gbar[0], (uint32_t)(nA * 16) * 2u * 128u);
      mbar_arrive_expect_tx(&gbar[1], (uint32_t)((ntile - nA) * 16) * 2u * 128u);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < ntile * 4; q += blockDim.x) {
      const int row0 = q * 4;
      uint64_t* bar = &gbar[row0 < nA * 16 ? 0 : 1];
      int rr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t pos = spos[row0 + u];
        int64_t mr = (s.kv_start + (pos >= 0 ? pos : 0)) * a.Hkv + s.g;
        mr = mr < 0 ? 0 : (mr >= map_rows ? map_rows - 1 : mr);
        rr[u] = (int)mr;
      }
      const uint32_t off = (uint32_t)row0 * 128u;
      tma_gather4(sK + off, &tmK, bar, 0, rr[0], rr[1], rr[2], rr[3]);
      tma_gather4(sK + kSpHalfBytes + off, &tmK, bar, 64, rr[0], rr[1], rr[2], rr[3]);
    }
    {
      const bf16* Vg = static_cast<const bf16*>(a.V);
      for (int grp = 0; grp < 2; ++grp) {
        const int c0 = (grp == 0 ? 0 : nA * 16) * 16, c1 = (grp == 0 ? nA * 16 : ntile * 16) * 16;
        for (int j = c0 + (int)threadIdx.x; j < c1; j += blockDim.x) {  // 16 chunks of 16 B a row
          const int row = j >> 4, half = (j >> 3) & 1, chunk = j & 7;
          const int64_t pos = spos[row];
          int64_t mr = (s.kv_start + (pos >= 0 ? pos : 0)) * a.Hkv + s.g;
          mr = mr < 0 ? 0 : (mr >= map_rows ? map_rows - 1 : mr);
          cp_async16(sV + half * kSpHalfBytes + row * 128 + ((chunk ^ (row & 7)) << 4),
                     Vg + mr * kD + half * 64 + chunk * 8, 16);
        }
        cp_async_mbar_arrive_noinc(&gbar[grp]);
      }
    }
    for (int half = 0; half < 2; ++half) {
      if (!mbar_wait(&gbar[half], (uint32_t)(piece & 1))) record_error(a.err, HS2_ERR_TIMEOUT);
      for (int st = (half == 0 ? 0 : nA) + warp; st < (half == 0 ? nA : ntile); st += kSpWarps) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const int row = st * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int chunk = (kk & 3) * 2 + (lane >> 4);
            const uint32_t addr = skb + (kk >> 2) * kSpHalfBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a0, a1, a2, a3, addr);
            mma_bf16(c, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
          }
        }
        const int ilo = st * 16 + r, ihi = ilo + 8;
        const bool vlo = spos[ilo] >= 0, vhi = spos[ihi] >= 0;
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
        const float p0v = exp_shift(x0, mn0), p1v = exp_shift(x1, mn1);
        const float p2v = exp_shift(x2, mn0), p3v = exp_shift(x3, mn1);
        l0 = l0 * al0 + (p0v + p2v);
        l1 = l1 * al1 + (p1v + p3v);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
        }
        const uint32_t b0 = movmatrix_t(pack_bf16(p0v, p1v));
        const uint32_t b1 = movmatrix_t(pack_bf16(p2v, p3v));
        const int row = st * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int chunk = (mt & 3) * 2 + ((lane >> 3) & 1);
          const uint32_t addr = svb + (mt >> 2) * kSpHalfBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(a0, a1, a2, a3, addr);
          mma_bf16(o[mt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    __syncthreads();  // the next piece overwrites the staged rows
    fence_proxy_async_smem();  // ... by TMA copies after these reads
  }
  cp_async_wait_all();  // (after a timed-out wait) no copy lands after the CTA is gone
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (r == 0) {
    wm[warp * 8 + h0] = m0; wl[warp * 8 + h0] = l0;
    wm[warp * 8 + h1] = m1; wl[warp * 8 + h1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d = mt * 16 + r;
    wo[(warp * 8 + h0) * kD + d] = o[mt][0];
    wo[(warp * 8 + h0) * kD + d + 8] = o[mt][2];
    wo[(warp * 8 + h1) * kD + d] = o[mt][1];
    wo[(warp * 8 + h1) * kD + d + 8] = o[mt][3];
  }
  __syncthreads();
  if (a.o_f32) sparse_cluster_merge<float, 8>(a, s.qi, s.g, cl, rank, cs, wm, wl, wo, recv);
  else sparse_cluster_merge<bf16, 8>(a, s.qi, s.g, cl, rank, cs, wm, wl, wo, recv);
}

// ----------------------------------------------------------------------------
// bf16, one CTA per (query, KV group) row, for launches with many rows (a
// chunk of queries): no cluster.  Each of the kSrWarps warps streams its own
// 16-key slices of the row's list (slices w, w + kSrWarps, ...) through a
// private two-deep shared-memory ring with cp.async (the copy of its next
// slice overlaps the tensor-core work on this one), keeps its own online
// softmax, and the warps merge once at the end.  No CTA-wide barrier in the
// main loop.
// ----------------------------------------------------------------------------
constexpr int kSrWarps = 4;
constexpr int kSrSlice = 16 * kSpRowBytes;             // 16 rows of K (or V), padded
constexpr size_t kSrSmem = (size_t)kSrWarps * 2 * 2 * kSrSlice;  // warps x ring x (K, V)

__global__ void __launch_bounds__(32 * kSrWarps) k_sparse_rows_bf16(const __grid_constant__ SparseArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ __align__(128) uint8_t sr_smem[];
  __shared__ float wm[kSrWarps * 8], wl[kSrWarps * 8];
  const SpRow s = sparse_row(a, 0, 1, true);  // the whole row (one CTA), KV head by KV head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16* K = static_cast<const bf16*>(a.K);
  const bf16* V = static_cast<const bf16*>(a.V);
  uint8_t* ring = sr_smem + (size_t)warp * 2 * 2 * kSrSlice;  // [buffer][K, V][16 rows]

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

  const int nslices = (s.n + 15) / 16;
  // issue the gather of slice sl into ring buffer buf: lane l copies 16-byte
  // piece l (K: l < 16, V: l >= 16) of each of the slice's 16 rows; returns the
  // slice's positions (lane i < 16: row i's, -1 when invalid or past the list)
  auto gather = [&](int sl, int buf) -> int64_t {
    const int i = lane & 15;
    const int64_t mypos = (sl * 16 + i < s.n) ? sparse_pos(a, s, sl * 16 + i, lane < 16) : -1;
    uint8_t* dK = ring + (size_t)buf * 2 * kSrSlice;
    uint8_t* dV = dK + kSrSlice;
    const int c16 = lane & 15;
    const bf16* base = lane < 16 ? K : V;
    uint8_t* dst0 = lane < 16 ? dK : dV;
#pragma unroll
    for (int row = 0; row < 16; ++row) {
      const int64_t pos = __shfl_sync(0xffffffffu, mypos, row);
      const bool ok = pos >= 0;
      const bf16* src = ok ? base + ((s.kv_start + pos) * a.Hkv + s.g) * kD + c16 * 8 : base;
      cp_async16(dst0 + (size_t)row * kSpRowBytes + c16 * 16, src, ok ? 16 : 0);
    }
    cp_async_commit();
    return mypos;
  };

  int sl = warp;
  int64_t pos_cur = sl < nslices ? gather(sl, 0) : -1;
  int buf = 0;
  for (; sl < nslices; sl += kSrWarps) {
    const int nxt = sl + kSrWarps;
    int64_t pos_nxt = -1;
    if (nxt < nslices) {
      pos_nxt = gather(nxt, buf ^ 1);
      cp_async_wait_prev();  // this slice's copies have landed (the next may be in flight)
    } else {
      cp_async_wait_all_groups();
    }
    __syncwarp();
    const uint32_t skb = smem_u32(ring + (size_t)buf * 2 * kSrSlice);
    const uint32_t svb = skb + kSrSlice;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int row = ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int chunk = kk * 2 + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a0, a1, a2, a3, skb + row * kSpRowBytes + chunk * 16);
        mma_bf16(c, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      }
    }
    const bool vlo = __shfl_sync(0xffffffffu, pos_cur, r) >= 0;
    const bool vhi = __shfl_sync(0xffffffffu, pos_cur, r + 8) >= 0;
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
    const float p0v = exp_shift(x0, mn0), p1v = exp_shift(x1, mn1);
    const float p2v = exp_shift(x2, mn0), p3v = exp_shift(x3, mn1);
    l0 = l0 * al0 + (p0v + p2v);
    l1 = l1 * al1 + (p1v + p3v);
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
    }
    const uint32_t b0 = movmatrix_t(pack_bf16(p0v, p1v));
    const uint32_t b1 = movmatrix_t(pack_bf16(p2v, p3v));
    {
      const int row = ((lane >> 4) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int chunk = mt * 2 + ((lane >> 3) & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(a0, a1, a2, a3, svb + row * kSpRowBytes + chunk * 16);
        mma_bf16(o[mt], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncwarp();  // the buffer is read before the gather after next overwrites it
    pos_cur = pos_nxt;
    buf ^= 1;
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (r == 0) {
    wm[warp * 8 + h0] = m0; wl[warp * 8 + h0] = l0;
    wm[warp * 8 + h1] = m1; wl[warp * 8 + h1] = l1;
  }
  // the warp's partial O goes into its own ring (its copies have all landed
  // and been read): 8 heads x D floats = 4 KB of the warp's 17 KB
  float* wo_mine = reinterpret_cast<float*>(ring);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d = mt * 16 + r;
    wo_mine[h0 * kD + d] = o[mt][0];
    wo_mine[h0 * kD + d + 8] = o[mt][2];
    wo_mine[h1 * kD + d] = o[mt][1];
    wo_mine[h1 * kD + d + 8] = o[mt][3];
  }
  __syncthreads();
  auto wo = [&](int w, int h, int d) {
    return reinterpret_cast<const float*>(sr_smem + (size_t)w * 2 * 2 * kSrSlice)[h * kD + d];
  };
  // merge the warps: thread (head h, dims) finishes O
  bf16* O = static_cast<bf16*>(a.O);
  for (int e = threadIdx.x; e < a.G * kD; e += blockDim.x) {
    const int h = e / kD, d = e % kD;
    float M = -INFINITY;
    for (int w = 0; w < kSrWarps; ++w) M = fmaxf(M, wm[w * 8 + h]);
    float L = 0.f, acc = 0.f;
    for (int w = 0; w < kSrWarps; ++w) {
      const float wt = exp_shift(wm[w * 8 + h], M);
      L = fmaf(wl[w * 8 + h], wt, L);
      acc = fmaf(wo(w, h, d), wt, acc);
    }
    O[(s.qi * a.Hq + (int64_t)s.g * a.G + h) * kD + d] = from_f<bf16>(L > 0.f ? acc / L : 0.f);
  }
}

// ----------------------------------------------------------------------------
// float32 on the CUDA cores: each warp takes every 4th index of the CTA's share
// and reads its K/V rows directly (lane i holds dims 4i..4i+3).
// ----------------------------------------------------------------------------
template <int GP>
__global__ void __launch_bounds__(32 * kSpWarps) k_sparse_f32(const __grid_constant__ SparseArgs a) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  __shared__ float wm[kSpWarps * GP], wl[kSpWarps * GP];
  __shared__ float wo[kSpWarps * GP * kD];
  __shared__ SpRecv recv;
  cg::cluster_group cl = cg::this_cluster();
  const int cs = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const SpRow s = sparse_row(a, rank, cs);
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
    const int64_t pos = sparse_pos(a, s, i, lane == 0);
    if (pos < 0) continue;  // the CUDA-core path serves float32 checks, not speed
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
#pragma unroll
  for (int h = 0; h < GP; ++h) {
    if (lane == 0) { wm[warp * GP + h] = m[h]; wl[warp * GP + h] = l[h]; }
    *reinterpret_cast<float4*>(wo + (warp * GP + h) * kD + lane * 4) = o[h];
  }
  __syncthreads();
  sparse_cluster_merge<float, GP>(a, s.qi, s.g, cl, rank, cs, wm, wl, wo, recv);
}

}  // namespace hs2
