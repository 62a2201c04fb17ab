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
#include "ptx.cuh"

namespace hs2 {

namespace cg = cooperative_groups;

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBins = 2048;
constexpr int kSelChunkAlign = 128 * kSelWarps;  // slices are multiples of this
constexpr int kSsCap = 8192;       // sampled kernel: candidates (or samples) one CTA holds
constexpr int kSsSortMax = 2048;   // sampled kernel: largest k
constexpr int kSsMinRho = 16;      // sampled kernel: at most one key in 16 is sampled
constexpr int kSsBcast = 256;      // sampled kernel: keys of the threshold's 22-bit prefix sent to every CTA

// Adds v to the 32-bit word at ``p`` (this CTA's shared memory) in CTA
// ``cta`` of the cluster, without waiting for a result; the next cluster
// barrier makes it visible there.
__device__ __forceinline__ void cluster_red_add(const uint32_t* p, int cta, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(cta));
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}

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

// Shared state of one CTA of a selection cluster of CS CTAs.
template <int CS>
struct SelState {
  uint32_t h[kSelBins];          // this CTA's histogram
  uint32_t tot[kSelBins / CS];   // cluster totals of the bins this CTA owns
  uint32_t ctot;                 // their sum
  int wgt[kSelWarps], weq[kSelWarps];
  int ccnt[2];                   // this CTA's keys > T and == T
  uint32_t digit;
  int krem;
  int ns, n, ngt, neq, nsel;     // sampled kernel: samples, collected, > T, == T, selected
};

// Number of candidates of a row: positions [0, t-window] (token rows) or the
// blocks holding at least one of them (block rows).  Sets *t.
// block_search: the whole CTA calls it (query_row_block).
__device__ __forceinline__ int64_t sel_row_candidates(const SelectArgs& a, int64_t r, int64_t* t,
                                                      bool block_search = false) {
  const QueryRow q = block_search ? query_row_block(a.qoff, a.kvoff, a.B, r / a.Hkv)
                                  : query_row(a.qoff, a.kvoff, a.B, r / a.Hkv);
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

// Window [max(0, t-window+1), t] after the nsel global picks, then -1 padding
// and the row's count.  Run by one CTA of the row.
__device__ __forceinline__ void sel_write_window(const SelectArgs& a, int64_t r, int64_t t,
                                                 int64_t nsel, int32_t* out, int32_t* count) {
  const int64_t wlen = t + 1 < a.window ? (t + 1 > 0 ? t + 1 : 0) : a.window;
  const int64_t w0 = t - wlen + 1;
  for (int64_t i = threadIdx.x; i < a.out_stride - nsel; i += blockDim.x)
    out[nsel + i] = i < wlen ? (int32_t)(w0 + i) : -1;
  if (threadIdx.x == 0) count[r] = (int32_t)(nsel + wlen);
}

// After the histograms of a pass (and a cluster barrier): this CTA sums its
// share ``own`` = nb/CS of the nb bins over the cluster into ``tot`` and their
// total into ``ctot``; ends with a cluster barrier.  Returns own.
template <int CS>
__device__ __forceinline__ int sel_reduce_bins(cg::cluster_group& cl, SelState<CS>& st, int nb) {
  const int own = nb / CS;
  const int rank = (int)cl.block_rank();
  uint32_t part = 0;
  for (int i = threadIdx.x; i < own; i += kSelThreads) {
    const int bin = rank * own + i;
    uint32_t v[CS];
#pragma unroll
    for (int c = 0; c < CS; ++c) v[c] = *cl.map_shared_rank(&st.h[bin], c);
    uint32_t sum = 0;
#pragma unroll
    for (int c = 0; c < CS; ++c) sum += v[c];
    st.tot[i] = sum;
    part += sum;
  }
  const uint32_t ws = __reduce_add_sync(0xffffffffu, part);
  if ((threadIdx.x & 31) == 0) st.wgt[threadIdx.x >> 5] = (int)ws;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t c = 0;
    for (int w = 0; w < kSelWarps; ++w) c += (uint32_t)st.wgt[w];
    st.ctot = c;
  }
  cl.sync();
  return own;
}

// The digit of the need-th largest key, from the bin totals reduce-scattered
// over the cluster (CTA c owns bins [c*own, (c+1)*own) and their sum ctot).
// Warp 0 finds the owning CTA from the CS sums, then the bin inside it; the
// result goes to st.digit / st.krem (the rank left inside that bin).
template <int CS>
__device__ __forceinline__ void sel_find_digit(cg::cluster_group& cl, SelState<CS>& st, int own,
                                               int need) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // chunk totals, highest chunk first: lane i holds chunk CS-1-i
    const int ci = CS - 1 - lane;
    const int v = lane < CS ? (int)*cl.map_shared_rank(&st.ctot, ci) : 0;
    int incl = v;  // keys in chunks >= ci
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, lane < CS && incl >= need && incl - v < need);
    if (hit == 0) {  // fewer keys than asked for: cannot happen for consistent counts
      if (lane == 0) {
        st.digit = 0u;
        st.krem = 1;
      }
    } else {
      const int hl = __ffs(hit) - 1;
      const int cstar = CS - 1 - hl;
      const int above = __shfl_sync(0xffffffffu, incl - v, hl);
      const int need2 = need - above;
      // bins of chunk cstar: lane i holds ``per`` bins, highest first
      const int per = own / 32;
      const uint32_t* rt = cl.map_shared_rank(st.tot, cstar);
      int mine = 0;
      for (int j = 0; j < per; ++j) mine += (int)rt[own - 1 - (lane * per + j)];
      int inc2 = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc2, o);
        if (lane >= o) inc2 += y;
      }
      const int ab2 = inc2 - mine;
      if (ab2 < need2 && inc2 >= need2) {
        int acc = ab2;
        for (int j = 0; j < per; ++j) {
          const int vj = (int)rt[own - 1 - (lane * per + j)];
          if (acc < need2 && acc + vj >= need2) {
            st.digit = (uint32_t)(cstar * own + own - 1 - (lane * per + j));
            st.krem = need2 - acc;
          }
          acc += vj;
        }
      }
    }
  }
  __syncthreads();
}

// Exact selection of the row's k largest keys from its slices (staged in
// shared memory, or re-read from global memory), written in ascending
// position order.  Every CTA of the cluster calls it; ends with a cluster
// barrier.
template <int CS>
__device__ void sel_exact(cg::cluster_group& cl, SelState<CS>& st, const SelectArgs& a,
                          const float* row, int64_t j0, int64_t S, int64_t len, bool use_smem,
                          bool vec, const uint4* skeys4, int32_t* out) {
  const int rank = (int)cl.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
    __syncthreads();
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t mask = pass == 2 ? 0x3FFu : 0x7FFu;
    const int pshift = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
    for (int64_t o = (int64_t)threadIdx.x * 4; o < len4; o += (int64_t)kSelThreads * 4) {
      uint32_t u[4];
      keys4(o, u);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (o + j < len && (pass == 0 || (u[j] >> pshift) == pre)) atomicAdd(&st.h[(u[j] >> shift) & mask], 1u);
    }
    cl.sync();
    const int own = sel_reduce_bins<CS>(cl, st, pass == 2 ? 1024 : kSelBins);
    sel_find_digit<CS>(cl, st, own, need);
    pre = pass == 0 ? st.digit : ((pre << (pass == 1 ? 11 : 10)) | st.digit);
    need = st.krem;
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
  if (lane == 0) { st.wgt[warp] = cgt; st.weq[warp] = ceq; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int tg = 0, te = 0;
    for (int w = 0; w < kSelWarps; ++w) { tg += st.wgt[w]; te += st.weq[w]; }
    st.ccnt[0] = tg;
    st.ccnt[1] = te;
  }
  cl.sync();
  // counts of the CTAs before this one, then of the warps before this one
  int gt_before = 0, eq_before = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    if (c < rank) {
      gt_before += *cl.map_shared_rank(&st.ccnt[0], c);
      eq_before += *cl.map_shared_rank(&st.ccnt[1], c);
    }
  }
  int gt_w = 0, eq_w = 0;
  for (int w = 0; w < warp; ++w) { gt_w += st.wgt[w]; eq_w += st.weq[w]; }
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

// Exact radix select, one cluster of CS CTAs per row; CTA c owns the c-th
// slice of the row's candidates, staged in shared memory when it fits.
template <int CS>
__global__ void __launch_bounds__(kSelThreads) k_select_cluster(const __grid_constant__ SelectArgs a,
                                                                int32_t* count) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ uint4 skeys4[];
  uint32_t* skeys = reinterpret_cast<uint32_t*>(skeys4);
  __shared__ SelState<CS> st;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int64_t r = blockIdx.x / CS;
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
  if (rank == 0 && count) sel_write_window(a, r, t, nsel_total, out, count);
  const int64_t len = nc - j0 < 0 ? 0 : (nc - j0 < S ? nc - j0 : S);
  if (nc <= a.k) {  // every candidate is kept (uniform over the cluster: no barrier)
    for (int64_t i = threadIdx.x; i < len; i += kSelThreads) out[j0 + i] = (int32_t)(j0 + i);
    return;
  }
  __syncthreads();  // staged keys visible to every warp
  sel_exact<CS>(cl, st, a, row, j0, S, len, use_smem, vec, skeys4, out);
}

// Ascending in-place sort of v[0, n) (n <= P, P a power of two, v holding P
// entries): bitonic network over the whole CTA, padding with the largest value.
template <typename T>
__device__ __forceinline__ void sel_sort_asc(T* v, int n, int P, T pad) {
  for (int i = n + threadIdx.x; i < P; i += blockDim.x) v[i] = pad;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const T x = v[i], y = v[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            v[i] = y;
            v[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int sel_pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Adds one to h[bin] for every lane with ``valid``: lanes with the same bin
// are merged first (one atomic per distinct bin of the warp), which keeps
// concentrated keys from serialising on one address.  All 32 lanes call it.
__device__ __forceinline__ void sel_hist_add(uint32_t* h, uint32_t bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!valid) return;
  const unsigned peers = __match_any_sync(act, bin);
  if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], (uint32_t)__popc(peers));
}

// Block-local: the bin of the need-th largest key from a histogram ``hist``
// of nb bins (1024 or 2048), counted from the highest bin; *digit gets the
// bin and *rem the rank left inside it.  All threads of the CTA call it; it
// ends with a CTA barrier.
__device__ __forceinline__ void sel_block_find(const uint32_t* hist, int nb, int need, int* scan_sh,
                                               uint32_t* digit, int* rem) {
  const int E = nb / kSelThreads;  // 2 or 4 bins per thread, the highest bins to thread 0
  const int top = nb - 1 - (int)threadIdx.x * E;
  int v[4] = {0, 0, 0, 0};
  int mine = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < E) {
      v[e] = (int)hist[top - e];
      mine += v[e];
    }
  int total;
  const int above = block_exclusive_scan(mine, scan_sh, &total);
  if (above < need && above + mine >= need) {
    int acc = above;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < E) {
        if (acc < need && acc + v[e] >= need) {
          *digit = (uint32_t)(top - e);
          *rem = need - acc;
        }
        acc += v[e];
      }
  }
  __syncthreads();
}

// Writes the nsel distinct positions sel[0, nsel), all in [lo, lo + span), to
// out[0, nsel) in ascending order: a counting sort over kSelBins position
// bins, then an insertion sort of the (few) positions of each bin.  tmp holds
// nsel ints of scratch.  All threads of the CTA call it.
template <int CS>
__device__ void sel_write_ordered(SelState<CS>& st, const int32_t* sel, int nsel, int64_t lo,
                                  int64_t span, int32_t* tmp, int32_t* out) {
  int sh = 0;
  while (((span - 1) >> sh) >= kSelBins) ++sh;
  auto bin_of = [&](int32_t v) { return (int)(((int64_t)v - lo) >> sh); };
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
  __syncthreads();
  for (int e = threadIdx.x; e < nsel; e += kSelThreads) atomicAdd(&st.h[bin_of(sel[e])], 1u);
  __syncthreads();
  {
    constexpr int E = kSelBins / kSelThreads;  // bins per thread, in order
    uint32_t c[E];
    int mine = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      c[e] = st.h[threadIdx.x * E + e];
      mine += (int)c[e];
    }
    int tot;
    int run = block_exclusive_scan(mine, st.wgt, &tot);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      st.h[threadIdx.x * E + e] = (uint32_t)run;  // start of the bin
      run += (int)c[e];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < nsel; e += kSelThreads) {
    const int32_t v = sel[e];
    tmp[atomicAdd(&st.h[bin_of(v)], 1u)] = v;  // afterwards st.h[b] = end of bin b
  }
  __syncthreads();
  {
    constexpr int E = kSelBins / kSelThreads;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int bin = threadIdx.x * E + e;
      const int b0 = bin ? (int)st.h[bin - 1] : 0, b1 = (int)st.h[bin];
      for (int i = b0 + 1; i < b1; ++i) {
        const int32_t v = tmp[i];
        int j = i - 1;
        while (j >= b0 && tmp[j] > v) {
          tmp[j + 1] = tmp[j];
          --j;
        }
        tmp[j + 1] = v;
      }
      for (int i = b0; i < b1; ++i) out[i] = tmp[i];
    }
  }
}

// Cluster-wide state of the gather-free finish of a sampled row (CS > 1).
template <int CS>
struct SelFinish {
  uint32_t hs[kSelBins];  // the cluster's histogram of the sampled keys' top 11 bits
  uint32_t h1[kSelBins];  // the cluster's histogram of the kept keys' top 11 bits
  uint32_t h2[kSelBins];  // the cluster's histogram of bits 10-20 of the kept keys of bin d1
  uint64_t bc[kSsBcast];  // the cluster's kept keys of the 22-bit prefix (d1, d2), with positions
  int nbc;                // entries in bc
  int base[CS];           // where this CTA's prefix keys go in CTA c's bc
  int cgt[CS];            // per CTA: its kept keys above bin d1
  int cgt2[CS];           // per CTA: its kept keys of bin d1 above sub-bin d2
  int csel[CS];           // per CTA: its keys of (d1, d2) taken
};

// The end of a sampled row on a cluster without gathering the kept keys on
// one CTA.  On entry every CTA holds its kept keys (all >= tau) in cand[0, n)
// and fin.h1 the cluster's histogram of their top 11 bits (each CTA added its
// own to every CTA's copy before the last cluster barrier).
//  a. d1 = the bin of the k-th largest kept key, r1 its rank inside the bin;
//  b. each CTA adds the histogram of bits 10-20 of its keys of bin d1 to every
//     CTA's h2 and sends its count of keys above bin d1; a cluster barrier;
//     d2 = the sub-bin of the r1-th largest key of bin d1, r2 its rank there;
//  c. each CTA sends its keys of the prefix (d1, d2) -- the threshold key, its
//     ties and near-ties: few -- with their positions to every CTA, and its
//     count of keys above the prefix; a cluster barrier;
//  d. every CTA ranks the prefix's keys by (key desc, position asc) and takes
//     the r2 first; each CTA writes its selected positions (every key above
//     the prefix and the taken ones of its slice) in ascending order after
//     those of the CTAs before it, whose slices hold the lower positions.
// The selection is the same as the gathering path's.  Returns false, with
// every CTA alike and the kept keys untouched, when more than kSsBcast keys
// share the prefix; the caller then takes the gathering path.
template <int CS>
__device__ bool sel_cluster_finish(cg::cluster_group& cl, SelState<CS>& st, SelFinish<CS>& fin,
                                   const SelectArgs& a, uint64_t* cand, int n, int32_t* sel,
                                   int rank, int64_t S, int32_t* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < CS) fin.csel[threadIdx.x] = 0;
  if (threadIdx.x == 0) st.nsel = 0;
  // a.
  sel_block_find(fin.h1, kSelBins, a.k, st.wgt, &st.digit, &st.krem);
  const uint32_t d1 = st.digit;
  const int r1 = st.krem;
  // b.
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
  __syncthreads();
  int gt = 0;
  for (int base = warp * 32; base < n; base += kSelThreads) {
    const int i = base + lane;
    const uint32_t u = i < n ? (uint32_t)cand[i] : 0u;
    gt += (i < n && (u >> 21) > d1) ? 1 : 0;
    sel_hist_add(st.h, (u >> 10) & 0x7FFu, i < n && (u >> 21) == d1);
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  if (lane == 0) st.wgt[warp] = gt;
  __syncthreads();
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) {
    const uint32_t v = st.h[i];
    if (v)
      for (int c = 0; c < CS; ++c) cluster_red_add(&fin.h2[i], c, v);
  }
  if (threadIdx.x < CS) {  // thread c sends this CTA's count to CTA c
    int sum = 0;
    for (int w = 0; w < kSelWarps; ++w) sum += st.wgt[w];
    *cl.map_shared_rank(&fin.cgt[rank], (int)threadIdx.x) = sum;
  }
  cl.sync();
  sel_block_find(fin.h2, kSelBins, r1, st.wgt, &st.digit, &st.krem);
  const uint32_t d2 = st.digit;
  const int r2 = st.krem;
  const uint32_t pre = (d1 << 11) | d2;  // the threshold's top 22 bits
  if ((int)fin.h2[d2] > kSsBcast) return false;  // the same on every CTA
  // c. (the prefix keys first to a local list: one slot reservation per CTA
  // of the cluster instead of one per key)
  uint64_t* lst = reinterpret_cast<uint64_t*>(sel);  // sel is written only after the barrier
  if (threadIdx.x == 0) st.neq = 0;
  __syncthreads();
  int gt2 = 0;
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint64_t cv = cand[i];
    const uint32_t u22 = (uint32_t)cv >> 10;
    if (u22 > pre && (u22 >> 11) == d1) ++gt2;
    if (u22 == pre) {
      const int slot = atomicAdd(&st.neq, 1);
      if (slot < kSsBcast) lst[slot] = cv;
    }
  }
  gt2 = __reduce_add_sync(0xffffffffu, gt2);
  if (lane == 0) st.weq[warp] = gt2;
  __syncthreads();
  const int m = st.neq < kSsBcast ? st.neq : kSsBcast;
  if (threadIdx.x < CS) {
    int sum = 0;
    for (int w = 0; w < kSelWarps; ++w) sum += st.weq[w];
    *cl.map_shared_rank(&fin.cgt2[rank], (int)threadIdx.x) = sum;
    fin.base[threadIdx.x] = m ? atomicAdd(cl.map_shared_rank(&fin.nbc, (int)threadIdx.x), m) : 0;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < m * CS; j += kSelThreads) {
    const int c = j / m, i = j - c * m;
    const int slot = fin.base[c] + i;
    if (slot < kSsBcast) *cl.map_shared_rank(&fin.bc[slot], c) = lst[i];
  }
  cl.sync();  // no CTA reads another's shared memory after this
  // d.
  const int nb = fin.nbc < kSsBcast ? fin.nbc : kSsBcast;
  for (int t = threadIdx.x; t < nb; t += kSelThreads) {
    const uint64_t me = fin.bc[t];
    const uint32_t u = (uint32_t)me, p = (uint32_t)(me >> 32);
    int rk = 0;
    for (int j = 0; j < nb; ++j) {
      const uint64_t o = fin.bc[j];
      const uint32_t uo = (uint32_t)o, po = (uint32_t)(o >> 32);
      rk += (uo > u || (uo == u && po < p)) ? 1 : 0;
    }
    if (rk < r2) {
      const int c = (int)(p / (uint32_t)S);
      atomicAdd(&fin.csel[c], 1);
      if (c == rank) sel[atomicAdd(&st.nsel, 1)] = (int32_t)p;
    }
  }
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint64_t cv = cand[i];
    if (((uint32_t)cv >> 10) > pre) sel[atomicAdd(&st.nsel, 1)] = (int32_t)(cv >> 32);
  }
  __syncthreads();
  int before = 0;
  for (int c = 0; c < rank; ++c) before += fin.cgt[c] + fin.cgt2[c] + fin.csel[c];
  const int nown = st.nsel;
  if (nown <= 160) {  // few (a decode row's share): each one's rank among them by counting
    for (int t = threadIdx.x; t < nown; t += kSelThreads) {
      const int32_t p = sel[t];
      int rk = 0;
      for (int j = 0; j < nown; ++j) rk += sel[j] < p ? 1 : 0;
      out[before + rk] = p;
    }
  } else {  // the kept keys are no longer read: their buffer is the scratch
    sel_write_ordered(st, sel, nown, (int64_t)rank * S, S, reinterpret_cast<int32_t*>(cand), out + before);
  }
  return true;
}

// Sample-guided exact selection (k <= kSsSortMax), one cluster of CS CTAs
// (CS may be 1) per row; CTA c owns the c-th slice of the row's candidates.
//  1. Sample: one group of four consecutive keys from every 4*rho keys (rho >=
//     16, at a hashed offset inside the group).  Every CTA adds its histogram
//     of the sampled keys' top 11 bits to every CTA's copy of the cluster's
//     histogram and takes tau = the smallest key of the bin holding the rs-th
//     largest sample, rs = k/rho plus a margin of four standard deviations.
//  2. Collect: one pass over the slice keeps every key >= tau with its
//     position.  When the cluster holds at least k such keys, the row's k
//     largest keys are all among them.
//  3. Clusters over rows that reach the last CTA's slice: every CTA finds the
//     threshold from the cluster's histograms of the kept keys and writes its
//     own share of the result (sel_cluster_finish).  Otherwise, or when too
//     many keys share the threshold's 22-bit prefix, CTA
//     0 gathers the kept keys of the cluster, finds the k-th largest key T and
//     the number kr of keys == T to take by a radix select, keeps every key > T
//     and the kr lowest-position keys == T, and writes the kept positions in
//     ascending order.
// Otherwise (fewer than k kept, or more than one CTA holds) the cluster runs
// the exact selection over the slices in global memory.  Either way the result
// equals a full stable sort by (score desc, position asc).
template <int CS>
__global__ void __launch_bounds__(kSelThreads, 2) k_select_sampled(const __grid_constant__ SelectArgs a,
                                                                int32_t* count) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ uint4 ss_dyn[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(ss_dyn);            // kept: (position << 32 | key)
  int32_t* sel = reinterpret_cast<int32_t*>(cand + kSsCap);       // selected positions
  __shared__ SelState<CS> st;
  __shared__ int offs[CS + 1];
  __shared__ SelFinish<CS> fin;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = CS == 1 ? 0 : (int)cl.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto csync = [&]() {
    if (CS == 1) __syncthreads();
    else cl.sync();
  };
  const int64_t r = blockIdx.x / CS;
  const int64_t S = a.slice;
  const int64_t j0 = (int64_t)rank * S;
  const float* row = a.data + r * a.stride + j0;
  const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
  int64_t t;
  int64_t nc = sel_row_candidates(a, r, &t, true);
  if (nc > (int64_t)CS * S) {  // longer than the host's maximum
    if (threadIdx.x == 0) record_error(a.err, HS2_ERR_DEVICE_INPUT);
    nc = 0;
  }
  int32_t* out = a.out + r * a.out_stride;
  const int64_t nsel_total = nc < a.k ? nc : a.k;
  if (rank == 0 && count) sel_write_window(a, r, t, nsel_total, out, count);
  const int64_t len = nc - j0 < 0 ? 0 : (nc - j0 < S ? nc - j0 : S);
  if (nc <= a.k) {  // every candidate is kept (uniform over the cluster: no barrier)
    for (int64_t i = threadIdx.x; i < len; i += kSelThreads) out[j0 + i] = (int32_t)(j0 + i);
    return;
  }
  auto key_at = [&](int64_t o) { return score_key(__ldg(row + o)); };

  // ---- 1. sample (rho depends on the slice size only: the same on every CTA)
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
  if constexpr (CS > 1) {  // the finish's cluster histograms, filled by every CTA later
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) fin.hs[i] = fin.h1[i] = fin.h2[i] = 0u;
    if (threadIdx.x == 0) fin.nbc = 0;
  }
  if (threadIdx.x == 0) {
    st.n = 0;
    st.ns = 0;
  }
  const int64_t rho = max((int64_t)kSsMinRho, (S + kSsCap - 1) / kSsCap);
  const int64_t gsz = 4 * rho;
  const int ngroups = (int)(len / gsz);  // whole groups only: at most kSsCap / 4
  __syncthreads();  // histogram cleared
  {
    constexpr int kSB = 4;
    for (int g00 = 0; g00 < ngroups; g00 += kSelThreads * kSB) {
      uint32_t u[kSB][4];
#pragma unroll
      for (int b = 0; b < kSB; ++b) {
        const int gi = g00 + b * kSelThreads + (int)threadIdx.x;
        if (gi < ngroups) {
          const uint32_t hsh = (uint32_t)(j0 / gsz + gi) * 0x9E3779B1u;
          const int64_t o = gi * gsz + 4 * (int64_t)((hsh >> 8) % (uint32_t)rho);
          if (vec) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(row + o));
            u[b][0] = score_key(v.x); u[b][1] = score_key(v.y);
            u[b][2] = score_key(v.z); u[b][3] = score_key(v.w);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) u[b][j] = key_at(o + j);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kSB; ++b) {
        const bool ok = g00 + b * kSelThreads + (int)threadIdx.x < ngroups;
#pragma unroll
        for (int j = 0; j < 4; ++j) sel_hist_add(st.h, ok ? u[b][j] >> 21 : 0u, ok);
      }
    }
  }
  if (threadIdx.x == 0) st.ns = 4 * ngroups;
  if constexpr (CS > 1) {
    // this CTA's sample histogram added to every CTA's fin.hs
    __syncthreads();
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) {
      const uint32_t v = st.h[i];
      if (v)
        for (int c = 0; c < CS; ++c) cluster_red_add(&fin.hs[i], c, v);
    }
  }
  csync();
  // tau = the lower edge of the bin holding the rs-th largest sample of the
  // row (every CTA finds the same bin in its copy of the cluster's sample
  // histogram); a row with fewer than rs samples keeps tau = 0.
  const float kr_f = (float)a.k / (float)rho;
  const int rs = (int)ceilf(kr_f + 4.f * sqrtf(kr_f)) + 8;
  uint32_t tau = 0u;
  if constexpr (CS > 1) {
    if (threadIdx.x == 0) st.digit = 0u;  // kept when the samples are fewer than rs
    sel_block_find(fin.hs, kSelBins, rs, st.wgt, &st.digit, &st.krem);
    tau = st.digit << 21;
  } else if (st.ns >= rs) {
    sel_block_find(st.h, kSelBins, rs, st.wgt, &st.digit, &st.krem);
    tau = st.digit << 21;
  }

  // ---- 2. collect every key >= tau of the slice (unordered)
  {
    constexpr int kBatch = 8;
    const int64_t len4 = vec ? (len & ~int64_t(3)) : 0;
    auto keep = [&](uint32_t u, int64_t o) {
      if (u >= tau) {
        const int at = atomicAdd(&st.n, 1);
        if (at < kSsCap) cand[at] = ((uint64_t)(uint32_t)(j0 + o) << 32) | u;
      }
    };
    for (int64_t base = threadIdx.x * 4; base < len4; base += (int64_t)kSelThreads * 4 * kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t i = base + (int64_t)u * kSelThreads * 4;
        v[u] = i < len4 ? __ldg(reinterpret_cast<const float4*>(row + i)) : make_float4(-1.f, -1.f, -1.f, -1.f);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t i = base + (int64_t)u * kSelThreads * 4;
        if (i < len4) {
          keep(score_key(v[u].x), i);
          keep(score_key(v[u].y), i + 1);
          keep(score_key(v[u].z), i + 2);
          keep(score_key(v[u].w), i + 3);
        }
      }
    }
    for (int64_t i = len4 + threadIdx.x; i < len; i += kSelThreads) keep(key_at(i), i);
  }
  // the gather-free finish when every CTA of the cluster holds part of the
  // row (a shorter row leaves CTAs idle there: the gathering path lets them
  // go early)
  const bool spread = CS > 1 && nc > (int64_t)(CS - 1) * S;
  if (spread) {
    // this CTA's histogram of its kept keys' top 11 bits, added to every CTA's
    // fin.h1
    __syncthreads();  // st.n is final
    const int nloc = st.n < kSsCap ? st.n : kSsCap;
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
    __syncthreads();
    for (int base = warp * 32; base < nloc; base += kSelThreads) {
      const int i = base + lane;
      sel_hist_add(st.h, i < nloc ? (uint32_t)cand[i] >> 21 : 0u, i < nloc);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) {
      const uint32_t v = st.h[i];
      if (v)
        for (int c = 0; c < CS; ++c) cluster_red_add(&fin.h1[i], c, v);
    }
  }
  csync();
  int collected = 0, most = 0;
  if (threadIdx.x == 0) offs[0] = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    const int nci = CS == 1 ? st.n : *cl.map_shared_rank(&st.n, c);
    collected += nci;
    most = max(most, nci);
    if (threadIdx.x == 0) offs[c + 1] = collected;
  }
  if (most > kSsCap || collected > kSsCap || collected < a.k) {
    // the sample misled: exact selection over the slices in global memory
    sel_exact<CS>(cl, st, a, row, j0, S, len, false, vec, nullptr, out);
    return;
  }
  if (spread) {
    if (sel_cluster_finish<CS>(cl, st, fin, a, cand, st.n, sel, rank, S, out)) return;
  }

  // ---- 3. CTA 0 gathers the cluster's kept keys and finishes the row
  if (CS > 1) {
    __syncthreads();  // offs
    if (rank == 0) {
      const int n0 = offs[1];
      for (int j00 = n0; j00 < collected; j00 += kSelThreads * 4) {
        uint64_t v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j00 + e * kSelThreads + (int)threadIdx.x;
          if (j < collected) {
            int c = 1;
            while (c < CS && offs[c + 1] <= j) ++c;
            v[e] = *cl.map_shared_rank(&cand[j - offs[c]], c);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j00 + e * kSelThreads + (int)threadIdx.x;
          if (j < collected) cand[j] = v[e];
        }
      }
    }
    cl.sync();  // the other CTAs' shared memory is not read after this
    if (rank != 0) return;
  }
  const int n = collected;
  // radix select of the k-th largest key among cand[0, n) (three local passes)
  uint32_t pre = 0;
  int need = a.k;
  for (int pass = 0; pass < 3; ++pass) {
    for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) st.h[i] = 0u;
    __syncthreads();
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t mask = pass == 2 ? 0x3FFu : 0x7FFu;
    const int pshift = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
    for (int base = warp * 32; base < n; base += kSelThreads) {
      const int i = base + lane;
      const uint32_t u = i < n ? (uint32_t)cand[i] : 0u;
      const bool ok = i < n && (pass == 0 || (u >> pshift) == pre);
      sel_hist_add(st.h, (u >> shift) & mask, ok);
    }
    __syncthreads();
    sel_block_find(st.h, pass == 2 ? 1024 : kSelBins, need, st.wgt, &st.digit, &st.krem);
    pre = pass == 0 ? st.digit : ((pre << (pass == 1 ? 11 : 10)) | st.digit);
    need = st.krem;
  }
  const uint32_t T = pre;
  const int kr = need;
  // keys > T go to sel[] unordered; keys == T are counted
  if (threadIdx.x == 0) {
    st.ngt = 0;
    st.neq = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t u = (uint32_t)cand[i];
    if (u > T) sel[atomicAdd(&st.ngt, 1)] = (int32_t)(cand[i] >> 32);
    else if (u == T) atomicAdd(&st.neq, 1);
  }
  __syncthreads();
  const int ngt = st.ngt, neq = st.neq;
  // the kr lowest-position keys == T follow at sel[ngt ..)
  if (kr == neq) {  // every tie is taken (the usual case: T is unique)
    if (threadIdx.x == 0) st.nsel = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kSelThreads)
      if ((uint32_t)cand[i] == T) sel[ngt + atomicAdd(&st.nsel, 1)] = (int32_t)(cand[i] >> 32);
  } else {
    // more ties than places: order the kept keys by position, take ties in order
    sel_sort_asc(cand, n, sel_pow2_at_least(n), ~uint64_t(0));
    const int E = (n + kSelThreads - 1) / kSelThreads;
    const int lo = min(n, (int)threadIdx.x * E), hi = min(n, lo + E);
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += (uint32_t)cand[i] == T;
    int tot;
    int tb = block_exclusive_scan(mine, st.wgt, &tot);
    for (int i = lo; i < hi; ++i)
      if ((uint32_t)cand[i] == T) {
        if (tb < kr) sel[ngt + tb] = (int32_t)(cand[i] >> 32);
        ++tb;
      }
  }
  __syncthreads();
  // ascending order by a counting sort over position bins (positions < nc)
  sel_write_ordered(st, sel, ngt + kr, 0, nc, reinterpret_cast<int32_t*>(cand), out);
}

// Block maxima over candidate positions: bmax[r][b] = max score in block b.
// One warp per block.
__global__ void __launch_bounds__(256) k_block_max(const float* scores, int64_t stride,
                                                   const int64_t* qoff, const int64_t* kvoff, int B,
                                                   int Hkv, int block, int window, float* bmax,
                                                   int64_t bstride, int* err) {
  grid_dep_wait();  // the previous kernel on the stream has finished
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
// positions, then the window, the -1 padding and the count.  A row whose
// geometry the block-max kernel rejected (more candidates than the score
// stride, or more blocks than the block-max stride; already reported) gets
// count 0 and all -1, so its output never depends on earlier scratch.
__global__ void __launch_bounds__(256) k_block_expand(const int32_t* bsel, int nbsel_max,
                                                      const int64_t* qoff, const int64_t* kvoff, int B,
                                                      int Hkv, int block, int window, int64_t stride,
                                                      int64_t bstride, int32_t* idx, int64_t idx_stride,
                                                      int32_t* count, int* err) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int64_t r = blockIdx.x;
  const QueryRow q = query_row(qoff, kvoff, B, r / Hkv);
  int64_t nc = q.t - window + 1;
  if (nc < 0) nc = 0;
  const int64_t nb = (nc + block - 1) / block;
  const bool bad = nc > stride || nb > bstride;
  int64_t nsel = bad ? 0 : (nb < nbsel_max ? nb : nbsel_max);
  int32_t* out = idx + r * idx_stride;
  const int32_t* bs = bsel + r * nbsel_max;
  int64_t ntok = 0;
  if (nsel > 0) {
    // every selected block but possibly the last (the highest id) is full
    const int64_t last = bs[nsel - 1];
    if (last < 0 || last >= nb) {  // not a block of this row: the selection did not run on it
      if (threadIdx.x == 0) record_error(err, HS2_ERR_DEVICE_INPUT);
      nsel = 0;
    } else {
      const int64_t last_len = (last * block + block < nc ? block : nc - last * block);
      ntok = (nsel - 1) * block + last_len;
      for (int64_t i = threadIdx.x; i < ntok; i += blockDim.x) {
        const int64_t bi = i / block, o = i % block;
        out[i] = (int32_t)((int64_t)bs[bi] * block + o);
      }
    }
  }
  const int64_t wlen = bad ? 0 : (q.t + 1 < window ? (q.t + 1 > 0 ? q.t + 1 : 0) : window);
  const int64_t w0 = q.t - wlen + 1;
  for (int64_t i = threadIdx.x; i < idx_stride - ntok; i += blockDim.x)
    out[ntok + i] = i < wlen ? (int32_t)(w0 + i) : -1;
  if (threadIdx.x == 0) count[r] = (int32_t)(ntok + wlen);
}

}  // namespace hs2
