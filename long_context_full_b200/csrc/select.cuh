// select.cuh - token-level top-k selection with a forced local window, and the
// first-generation block-level selection used as a comparison path.
//
// Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
// "Token-Level Selection and Unified Local Access" (1,024 global tokens chosen
// outside the 128 most recent tokens, which are always kept) and "Xiaomi
// discloses MiMo-V3 plans to adopt HySparse2 architecture", section "Article"
// (the previous generation kept whole groups of 64 tokens).
//
// Exact radix select over the order-preserving 32-bit keys of the float scores,
// spread over many CTAs per row (a row is 128K-1M candidates at batch 1-8):
//   pass 0..2  histogram of key bits [31:21], [20:10], [9:0] among the keys that
//              match the prefix fixed so far; the last CTA of a row to finish
//              (atomic ticket, no spinning) scans the histogram and fixes the
//              next prefix digit and the rank still needed inside it.  After
//              pass 2 the prefix is the k-th largest key T and ``krem`` is the
//              number of keys equal to T that belong to the result.
//   count      per-slice counts of keys > T and == T.
//   compact    ordered compaction: slice s knows, from the counts of slices
//              before it, how many keys precede it and how many T-ties were
//              already taken, so keys > T plus the lowest-position krem ties are
//              written in ascending position order - independent of the grid.
// The result therefore equals a full stable sort by (score desc, position asc).
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int kSelThreads = 256;
constexpr int kSelItems = 16;                     // keys per thread per slice
constexpr int kSelSlice = kSelThreads * kSelItems;  // 4096 keys per CTA
constexpr int kSelBins = 2048;

struct SelectArgs {
  const float* data;   // rows of values to select from
  int64_t stride;      // row stride of ``data``
  const int64_t* qoff;
  const int64_t* kvoff;
  int B, Hkv;
  int64_t rows;        // total_q * Hkv
  int k, window;
  int block;           // 0: token rows; > 0: rows of block maxima (block size)
  int nslices;         // grid.y: slices per row (max over rows); grid.x = rows
  uint32_t* hist;      // [rows, kSelBins]
  uint32_t* ticket;    // [rows]
  uint32_t* prefix;    // [rows]
  int32_t* krem;       // [rows]
  int32_t* cnt;        // [rows, nslices, 2]
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
  return nc;
}

__device__ __forceinline__ int64_t sel_row_checked(const SelectArgs& a, int64_t r, int64_t* t) {
  int64_t nc = sel_row_candidates(a, r, t);
  if (nc > a.stride || nc > (int64_t)a.nslices * kSelSlice) {  // offsets disagree with the sizes
    record_error(a.err, HS2_ERR_DEVICE_INPUT);
    nc = 0;
  }
  return nc;
}

// One histogram pass.  pass 0: bits [31:21]; 1: [20:10] under the 11-bit
// prefix; 2: [9:0] under the 22-bit prefix.
__global__ void __launch_bounds__(kSelThreads) k_select_hist(const __grid_constant__ SelectArgs a,
                                                             int pass) {
  const int64_t r = blockIdx.x;
  const int s = blockIdx.y;
  int64_t t;
  const int64_t nc = sel_row_checked(a, r, &t);
  if (nc <= a.k) return;
  const int nsl = (int)((nc + kSelSlice - 1) / kSelSlice);
  if (s >= nsl) return;

  __shared__ uint32_t h[kSelBins];
  __shared__ int sh[kSelThreads / 32 + 1];
  __shared__ int is_last;
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) h[i] = 0;
  __syncthreads();

  const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
  const uint32_t mask = pass == 2 ? 0x3FFu : 0x7FFu;
  const int pshift = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
  const uint32_t pre = pass == 0 ? 0u : a.prefix[r];
  const float* row = a.data + r * a.stride;
  const int64_t j0 = (int64_t)s * kSelSlice;
  for (int i = 0; i < kSelItems; ++i) {
    const int64_t j = j0 + (int64_t)i * kSelThreads + threadIdx.x;
    if (j < nc) {
      const uint32_t u = score_key(__ldg(row + j));
      if (pass == 0 || (u >> pshift) == pre) atomicAdd(&h[(u >> shift) & mask], 1u);
    }
  }
  __syncthreads();
  uint32_t* gh = a.hist + r * kSelBins;
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.ticket + r, 1u) == (uint32_t)(nsl - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // Last CTA of the row: find the digit holding the krem-th largest key.
  const int nb = pass == 2 ? 1024 : kSelBins;
  const int per = nb / kSelThreads;  // 8 or 4 bins per thread, ascending
  uint32_t mine[8];
  int tsum = 0;
  for (int i = 0; i < per; ++i) {
    mine[i] = __ldcg(gh + threadIdx.x * per + i);
    tsum += (int)mine[i];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kSelBins; i += kSelThreads) gh[i] = 0u;  // clean for reuse
  // keys in the bins above this thread's range: thread i's sum is stored at
  // position 255-i, so an exclusive scan over positions sums the higher threads
  __shared__ int rv[kSelThreads];
  const int rev = kSelThreads - 1 - threadIdx.x;
  rv[rev] = tsum;
  __syncthreads();
  int total;
  const int ex = block_exclusive_scan(rv[threadIdx.x], sh, &total);
  rv[threadIdx.x] = ex;
  __syncthreads();
  const int above = rv[rev];
  const int need = pass == 0 ? a.k : a.krem[r];
  if (above < need && above + tsum >= need) {
    int acc = above;
    for (int i = per - 1; i >= 0; --i) {
      if (acc + (int)mine[i] >= need) {
        const uint32_t digit = (uint32_t)(threadIdx.x * per + i);
        a.prefix[r] = pass == 0 ? digit : ((pre << (pass == 1 ? 11 : 10)) | digit);
        a.krem[r] = need - acc;
        break;
      }
      acc += (int)mine[i];
    }
  }
  if (threadIdx.x == 0) a.ticket[r] = 0u;
}

// Per-slice counts of keys > T and == T.
__global__ void __launch_bounds__(kSelThreads) k_select_count(const __grid_constant__ SelectArgs a) {
  const int64_t r = blockIdx.x;
  const int s = blockIdx.y;
  int64_t t;
  const int64_t nc = sel_row_checked(a, r, &t);
  if (nc <= a.k) return;
  const int nsl = (int)((nc + kSelSlice - 1) / kSelSlice);
  if (s >= nsl) return;
  __shared__ int sh[kSelThreads / 32 + 1];
  const uint32_t T = a.prefix[r];
  const float* row = a.data + r * a.stride;
  const int64_t j0 = (int64_t)s * kSelSlice;
  int gt = 0, eq = 0;
  for (int i = 0; i < kSelItems; ++i) {
    const int64_t j = j0 + (int64_t)i * kSelThreads + threadIdx.x;
    if (j < nc) {
      const uint32_t u = score_key(__ldg(row + j));
      gt += u > T;
      eq += u == T;
    }
  }
  int tot_gt, tot_eq;
  block_exclusive_scan(gt, sh, &tot_gt);
  block_exclusive_scan(eq, sh, &tot_eq);
  if (threadIdx.x == 0) {
    a.cnt[(r * a.nslices + s) * 2] = tot_gt;
    a.cnt[(r * a.nslices + s) * 2 + 1] = tot_eq;
  }
}

// Ordered compaction of the selected positions of each slice; rows with at
// most k candidates take all of them.  Slice 0 of token rows also writes the
// window, the -1 padding and the count (``count`` non-null).
__global__ void __launch_bounds__(kSelThreads) k_select_compact(const __grid_constant__ SelectArgs a,
                                                                int32_t* count) {
  const int64_t r = blockIdx.x;
  const int s = blockIdx.y;
  int64_t t;
  const int64_t nc = sel_row_checked(a, r, &t);
  int32_t* out = a.out + r * a.out_stride;
  const int64_t nsel_total = nc < a.k ? nc : a.k;
  if (s == 0 && count) {
    // window [max(0, t-window+1), t] after the global part, then padding
    const int64_t wlen = t + 1 < a.window ? (t + 1 > 0 ? t + 1 : 0) : a.window;
    const int64_t w0 = t - wlen + 1;
    for (int64_t i = threadIdx.x; i < a.out_stride - nsel_total; i += kSelThreads)
      out[nsel_total + i] = i < wlen ? (int32_t)(w0 + i) : -1;
    if (threadIdx.x == 0) count[r] = (int32_t)(nsel_total + wlen);
  }
  const int nsl = (int)((nc + kSelSlice - 1) / kSelSlice);
  if (s >= nsl) return;
  const int64_t j0 = (int64_t)s * kSelSlice;
  // thread-contiguous items so that positions come out in ascending order
  const int64_t jt = j0 + (int64_t)threadIdx.x * kSelItems;
  if (nc <= a.k) {
    for (int i = 0; i < kSelItems; ++i)
      if (jt + i < nc) out[jt + i] = (int32_t)(jt + i);
    return;
  }
  __shared__ int sh[kSelThreads / 32 + 1];
  __shared__ int before[2];
  const uint32_t T = a.prefix[r];
  const int kr = a.krem[r];
  // counts of the slices before this one
  int bg = 0, be = 0;
  for (int q = threadIdx.x; q < s; q += kSelThreads) {
    bg += a.cnt[(r * a.nslices + q) * 2];
    be += a.cnt[(r * a.nslices + q) * 2 + 1];
  }
  int tg, te;
  block_exclusive_scan(bg, sh, &tg);
  block_exclusive_scan(be, sh, &te);
  if (threadIdx.x == 0) { before[0] = tg; before[1] = te; }
  __syncthreads();
  const int before_gt = before[0], before_eq = before[1];

  const float* row = a.data + r * a.stride;
  uint32_t u[kSelItems];
  int neq = 0;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i) {
    u[i] = (jt + i < nc) ? score_key(__ldg(row + jt + i)) : 0u;
    neq += (jt + i < nc) && u[i] == T;
  }
  int tot;
  const int eq_base = block_exclusive_scan(neq, sh, &tot);
  int nsel = 0, er = before_eq + eq_base;
  uint32_t selmask = 0;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i) {
    if (jt + i >= nc) continue;
    bool sel = u[i] > T;
    if (u[i] == T) { sel = er < kr; ++er; }
    if (sel) { selmask |= 1u << i; ++nsel; }
  }
  const int sel_base = block_exclusive_scan(nsel, sh, &tot);
  const int tie_taken = before_eq < kr ? before_eq : kr;
  int o = before_gt + tie_taken + sel_base;
#pragma unroll
  for (int i = 0; i < kSelItems; ++i)
    if ((selmask >> i) & 1u) out[o++] = (int32_t)(jt + i);
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
