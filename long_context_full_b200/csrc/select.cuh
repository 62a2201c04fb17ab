// select.cuh - token-level top-k selection with a forced local window, and the
// first-generation block-level selection used as a comparison path.
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
// "Token-Level Selection and Unified Local Access" (1,024 global tokens chosen
// outside the 128 most recent tokens, which are always kept) and "Xiaomi
// discloses MiMo-V3 plans to adopt HySparse2 architecture", section "Article"
// (the previous generation kept whole groups of 64 tokens).
//
// Exact radix select over the order-preserving 32-bit keys of the float
// scores.  One thread-block cluster (8 or 16 CTAs) per row; CTA c of the
// cluster owns the c-th slice of the row's candidates, kept in shared memory
// when it fits.  Three histogram passes fix the key bits [31:21], [20:10] and
// [9:0] of the k-th largest key T: each CTA histograms its slice (among keys
// that match the prefix found so far), the CTAs reduce-scatter the histograms
// through distributed shared memory, every CTA gathers the totals and derives
// the same digit.  Then each CTA counts its keys > T and == T, reads the counts
// of the CTAs before it, and writes its selected positions in ascending order:
// keys > T, and the lowest-position ties until k are taken.  All waits are
// hardware cluster barriers.  The result equals a full stable sort by
// (score desc, position asc), whatever the cluster size.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace hs2 {

namespace cg = cooperative_groups;

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBins = 2048;
constexpr int kSelChunkAlign = 128 * kSelWarps;  // slices are multiples of this

struct SelectArgs {
  const float* data;   // rows of values to select from
  int64_t stride;      // row stride of ``data`` (floats)
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hkv;
  int64_t rows;        // total_q * Hkv
  int k, window;
  int block;           // 0: token rows; > 0: rows of block maxima (block size)
  int64_t slice;       // keys per CTA of a row's cluster (multiple of kSelChunkAlign)
  int smem_keys;       // 1: slices staged in shared memory; 0: re-read from global
  int32_t* out;        // compacted selection, [rows, out_stride]
  int64_t out_stride;
  int* err;
};

// Number of candidates of a row: positions [0, t-window] (token rows) or the
// blocks holding at least one of them (block rows).  Sets *t.
__device__ __forceinline__ int64_t sel_row_candidates(const SelectArgs& a, int64_t r, int64_t* t) {
  const QueryRow q = query_row(a.qoff, a.kvoff, a.B, r / a.Hkv);
  *t = q.t;
  int64_t nc = q.t - a.window + 1;
  if (nc < 0) nc = 0;
  if (a.block > 0) nc = (nc + a.block - 1) / a.block;
  if (nc > a.stride) {  // offsets disagree with the stride the host was given
    record_error(a.err, HS2_ERR_DEVICE_INPUT);
    nc = 0;
  }
  return nc;
}

// The digit of the need-th largest key, from the per-CTA bin totals of a
// histogram of nb bins reduce-scattered over the cluster (CTA c owns bins
// [c*own, (c+1)*own) and their sum ``ctot``).  Warp 0 finds the owning CTA from
// the CS sums, then the bin inside it; the result goes to *digit / *krem.
template <int CS>
__device__ __forceinline__ void sel_find_digit(cg::cluster_group& cl, const uint32_t* tot,
                                               const uint32_t* ctot, int own, int need,
                                               uint32_t* digit, int* krem) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // chunk totals, highest chunk first: lane i holds chunk CS-1-i
    const int ci = CS - 1 - lane;
    const int v = lane < CS ? (int)*cl.map_shared_rank(ctot, ci) : 0;
    int incl = v;  // keys in chunks >= ci
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, lane < CS && incl >= need && incl - v < need);
    const int hl = __ffs(hit) - 1;
    const int cstar = CS - 1 - hl;
    const int above = __shfl_sync(0xffffffffu, incl - v, hl);
    const int need2 = need - above;
    // bins of chunk cstar: lane i holds bins, highest first, ``per`` each
    const int per = own / 32;
    const uint32_t* rt = cl.map_shared_rank(tot, cstar);
    int mine = 0;
    uint32_t vals[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      vals[j] = j < per ? rt[own - 1 - (lane * per + j)] : 0u;
      mine += (int)vals[j];
    }
    int inc2 = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc2, o);
      if (lane >= o) inc2 += y;
    }
    const int ab2 = inc2 - mine;
    if (ab2 < need2 && inc2 >= need2) {
      int acc = ab2;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < per && acc < need2 && acc + (int)vals[j] >= need2) {
          *digit = (uint32_t)(cstar * own + own - 1 - (lane * per + j));
          *krem = need2 - acc;
        }
        acc += (int)vals[j];
      }
    }
  }
  __syncthreads();
}

template <int CS>
__global__ void __launch_bounds__(kSelThreads) k_select_cluster(const __grid_constant__ SelectArgs a,
                                                                int32_t* count) {
  extern __shared__ uint4 skeys4[];
  uint32_t* skeys = reinterpret_cast<uint32_t*>(skeys4);
  __shared__ uint32_t h[kSelBins];          // this CTA's histogram
  __shared__ uint32_t tot[kSelBins / CS];   // cluster totals of the bins this CTA owns
  __shared__ uint32_t ctot;                 // their sum
  __shared__ int wgt[kSelWarps], weq[kSelWarps];
  __shared__ int ccnt[2];                   // this CTA's keys > T and == T
  __shared__ uint32_t s_digit;
  __shared__ int s_krem;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int64_t r = blockIdx.x / CS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's slice: [j0, j0 + S) of the row (S fixed by the host)
  const int64_t S = a.slice;
  const int64_t j0 = (int64_t)rank * S;
  const float* row = a.data + r * a.stride + j0;
  const bool use_smem = a.smem_keys != 0;
  const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
  if (use_smem) {
    // stage the slice (up to the row's capacity) before the row geometry is
    // known; keys past the row's candidates are ignored below
    int64_t cap = a.stride - j0 < S ? a.stride - j0 : S;
    if (cap < 0) cap = 0;  // a slice past the row's capacity stages nothing
    constexpr int kBatch = 8;
    if (vec) {
      const int64_t cap4 = cap & ~int64_t(3);
      for (int64_t base = threadIdx.x * 4; base < cap4; base += (int64_t)kSelThreads * 4 * kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int64_t i = base + (int64_t)u * kSelThreads * 4;
          v[u] = i < cap4 ? __ldg(reinterpret_cast<const float4*>(row + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int64_t i = base + (int64_t)u * kSelThreads * 4;
          if (i < cap4)
            skeys4[i >> 2] = make_uint4(score_key(v[u].x), score_key(v[u].y), score_key(v[u].z),
                                        score_key(v[u].w));
        }
      }
      for (int64_t i = cap4 + threadIdx.x; i < cap; i += kSelThreads) skeys[i] = score_key(__ldg(row + i));
    } else {
      for (int64_t base = threadIdx.x; base < cap; base += (int64_t)kSelThreads * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int64_t i = base + (int64_t)u * kSelThreads;
          v[u] = i < cap ? __ldg(row + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int64_t i = base + (int64_t)u * kSelThreads;
          if (i < cap) skeys[i] = score_key(v[u]);
        }
      }
    }
  }
  int64_t t;
  int64_t nc = sel_row_candidates(a, r, &t);
  if (nc > (int64_t)CS * S) {  // longer than the host's maximum
    if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    nc = 0;
  }
  int32_t* out = a.out + r * a.out_stride;
  const int64_t nsel_total = nc < a.k ? nc : a.k;
  if (rank == 0 && count) {
    // window [max(0, t-window+1), t] after the global part, then -1 padding
    const int64_t wlen = t + 1 < a.window ? (t + 1 > 0 ? t + 1 : 0) : a.window;
    const int64_t w0 = t - wlen + 1;
    for (int64_t i = threadIdx.x; i < a.out_stride - nsel_total; i += kSelThreads)
      out[nsel_total + i] = i < wlen ? (int32_t)(w0 + i) : -1;
    if (threadIdx.x == 0) count[r] = (int32_t)(nsel_total + wlen);
  }
  const int64_t len = nc - j0 < 0 ? 0 : (nc - j0 < S ? nc - j0 : S);
  if (nc <= a.k) {  // every candidate is kept (uniform over the cluster: no barrier)
    for (int64_t i = threadIdx.x; i < len; i += kSelThreads) out[j0 + i] = (int32_t)(j0 + i);
    return;
  }
  __syncthreads();  // staged keys visible to every warp
  const int64_t C = S / kSelWarps;  // keys per warp chunk, a multiple of 128
  const int64_t wbeg = warp * C;
  // four consecutive keys at slice offset o (o % 4 == 0); invalid past len
  auto keys4 = [&](int64_t o, uint32_t (&u)[4]) {
    if (use_smem) {
      const uint4 v = skeys4[o >> 2];
      u[0] = v.x; u[1] = v.y; u[2] = v.z; u[3] = v.w;
    } else if (vec && o + 3 < len) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + o));
      u[0] = score_key(v.x); u[1] = score_key(v.y); u[2] = score_key(v.z); u[3] = score_key(v.w);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) u[j] = o + j < len ? score_key(__ldg(row + o + j)) : 0u;
    }
  };
  const int64_t len4 = (len + 3) & ~int64_t(3);

  uint32_t pre = 0;
  int need = a.k;
  for (int pass = 0; pass < 3; ++pass) {
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) h[i] = 0u;
    __syncthreads();
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t mask = pass == 2 ? 0x3FFu : 0x7FFu;
    const int pshift = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
    for (int64_t o = (int64_t)threadIdx.x * 4; o < len4; o += (int64_t)kSelThreads * 4) {
      uint32_t u[4];
      keys4(o, u);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (o + j < len && (pass == 0 || (u[j] >> pshift) == pre)) atomicAdd(&h[(u[j] >> shift) & mask], 1u);
    }
    cl.sync();
    // reduce-scatter: this CTA sums its share of the bins over the cluster
    const int nb = pass == 2 ? 1024 : kSelBins;
    const int own = nb / CS;
    // (ctot and tot of the previous pass were last read before this pass's
    // first cluster barrier, so they may be rewritten now)
    if (threadIdx.x < own) {
      const int bin = rank * own + threadIdx.x;
      uint32_t v[CS];
#pragma unroll
      for (int c = 0; c < CS; ++c) v[c] = *cl.map_shared_rank(&h[bin], c);
      uint32_t sum = 0;
#pragma unroll
      for (int c = 0; c < CS; ++c) sum += v[c];
      tot[threadIdx.x] = sum;
      const uint32_t ws = __reduce_add_sync(0xffffffffu, sum);  // own is a multiple of 32
      if (lane == 0) wgt[warp] = (int)ws;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t c = 0;
      for (int w = 0; w < own / 32; ++w) c += (uint32_t)wgt[w];
      ctot = c;
    }
    cl.sync();
    sel_find_digit<CS>(cl, tot, &ctot, own, need, &s_digit, &s_krem);
    pre = pass == 0 ? s_digit : ((pre << (pass == 1 ? 11 : 10)) | s_digit);
    need = s_krem;
  }
  const uint32_t T = pre;
  const int kr = need;
  // keys > T and == T of each warp's chunk (the compaction walks the chunks in
  // order), then of the CTA
  const int64_t wend = wbeg + C < len ? wbeg + C : len;
  int cgt = 0, ceq = 0;
  for (int64_t o = wbeg + lane * 4; o < wend; o += 128) {
    uint32_t u[4];
    keys4(o, u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool v = o + j < wend;
      cgt += v && u[j] > T;
      ceq += v && u[j] == T;
    }
  }
  cgt = __reduce_add_sync(0xffffffffu, cgt);
  ceq = __reduce_add_sync(0xffffffffu, ceq);
  if (lane == 0) { wgt[warp] = cgt; weq[warp] = ceq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int tg = 0, te = 0;
    for (int w = 0; w < kSelWarps; ++w) { tg += wgt[w]; te += weq[w]; }
    ccnt[0] = tg;
    ccnt[1] = te;
  }
  cl.sync();
  // counts of the CTAs before this one, then of the warps before this one
  int gt_before = 0, eq_before = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    if (c < rank) {
      gt_before += *cl.map_shared_rank(&ccnt[0], c);
      eq_before += *cl.map_shared_rank(&ccnt[1], c);
    }
  }
  int gt_w = 0, eq_w = 0;
  for (int w = 0; w < warp; ++w) { gt_w += wgt[w]; eq_w += weq[w]; }
  // selected before this warp: every key > T, and the ties of rank < kr
  int tie_rank = eq_before + eq_w;
  int pos = gt_before + gt_w + (tie_rank < kr ? tie_rank : kr);
  // ordered compaction, 128 keys per step: lane l holds keys 4l..4l+3 of the step
  for (int64_t o = wbeg + lane * 4; o - lane * 4 < wend; o += 128) {
    uint32_t u[4];
    keys4(o < len4 ? o : 0, u);
    bool g4[4], e4[4];
    int ec = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool v = o + j < wend;
      g4[j] = v && u[j] > T;
      e4[j] = v && u[j] == T;
      ec += e4[j];
    }
    if (!__any_sync(0xffffffffu, g4[0] | g4[1] | g4[2] | g4[3] | (ec > 0))) continue;
    int ex = ec;  // inclusive scan of the lanes' ties
#pragma unroll
    for (int s2 = 1; s2 < 32; s2 <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ex, s2);
      if (lane >= s2) ex += y;
    }
    const int eq_step = __shfl_sync(0xffffffffu, ex, 31);
    int er = tie_rank + ex - ec;
    bool sel[4];
    int sc = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sel[j] = g4[j] || (e4[j] && er < kr);
      er += e4[j];
      sc += sel[j];
    }
    int sx = sc;
#pragma unroll
    for (int s2 = 1; s2 < 32; s2 <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sx, s2);
      if (lane >= s2) sx += y;
    }
    const int sel_step = __shfl_sync(0xffffffffu, sx, 31);
    int w = pos + sx - sc;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (sel[j]) out[w++] = (int32_t)(j0 + o + j);
    pos += sel_step;
    tie_rank += eq_step;
  }
  cl.sync();  // other CTAs may still read this CTA's shared memory until here
}

// Block maxima over candidate positions: bmax[r][b] = max score in block b.
// One warp per block.
__global__ void __launch_bounds__(256) k_block_max(const float* scores, int64_t stride,
                                                   const int64_t* qoff, const int64_t* kvoff, int B,
                                                   int Hkv, int block, int window, float* bmax,
                                                   int64_t bstride, int* err) {
  const int64_t r = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int64_t bi = (int64_t)blockIdx.y * 8 + (threadIdx.x >> 5);
  const QueryRow q = query_row(qoff, kvoff, B, r / Hkv);
  int64_t nc = q.t - window + 1;
  if (nc < 0) nc = 0;
  if (nc > stride) { if (lane == 0) record_error(err, HS2_ERR_DEVICE_INPUT); return; }
  const int64_t nb = (nc + block - 1) / block;
  if (nb > bstride) { if (lane == 0 && bi == 0) record_error(err, HS2_ERR_DEVICE_INPUT); return; }
  if (bi >= nb) return;
  const int64_t a0 = bi * block;
  const int64_t a1 = a0 + block < nc ? a0 + block : nc;
  float m = -INFINITY;
  for (int64_t j = a0 + lane; j < a1; j += 32) m = fmaxf(m, __ldg(scores + r * stride + j));
  m = warp_max(m);
  if (lane == 0) bmax[r * bstride + bi] = m;
}

// Expands the selected blocks (ascending block ids) into their candidate
// positions, then the window, the -1 padding and the count.
__global__ void __launch_bounds__(256) k_block_expand(const int32_t* bsel, int nbsel_max,
                                                      const int64_t* qoff, const int64_t* kvoff, int B,
                                                      int Hkv, int block, int window, int32_t* idx,
                                                      int64_t idx_stride, int32_t* count) {
  const int64_t r = blockIdx.x;
  const QueryRow q = query_row(qoff, kvoff, B, r / Hkv);
  int64_t nc = q.t - window + 1;
  if (nc < 0) nc = 0;
  const int64_t nb = (nc + block - 1) / block;
  const int64_t nsel = nb < nbsel_max ? nb : nbsel_max;
  int32_t* out = idx + r * idx_stride;
  const int32_t* bs = bsel + r * nbsel_max;
  int64_t ntok = 0;
  if (nsel > 0) {
    // every selected block but possibly the last (the highest id) is full
    const int64_t last = bs[nsel - 1];
    const int64_t last_len = (last * block + block < nc ? block : nc - last * block);
    ntok = (nsel - 1) * block + last_len;
    for (int64_t i = threadIdx.x; i < ntok; i += blockDim.x) {
      const int64_t bi = i / block, o = i % block;
      out[i] = (int32_t)((int64_t)bs[bi] * block + o);
    }
  }
  const int64_t wlen = q.t + 1 < window ? (q.t + 1 > 0 ? q.t + 1 : 0) : window;
  const int64_t w0 = q.t - wlen + 1;
  for (int64_t i = threadIdx.x; i < idx_stride - ntok; i += blockDim.x)
    out[ntok + i] = i < wlen ? (int32_t)(w0 + i) : -1;
  if (threadIdx.x == 0) count[r] = (int32_t)(ntok + wlen);
}

}  // namespace hs2
