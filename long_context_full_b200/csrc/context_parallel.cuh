// context_parallel.cuh - the merge steps of a decode Hybrid Block whose KV
// cache is split by position across ranks (context parallelism): rank r holds
// positions [pos0_b, pos0_b + n_b) of every sequence b, runs the full-attention
// pass, the local top-k and the sparse layers on its own rows, and the ranks
// exchange only small partials.
//
// Sources: the Full Attention layer and the selection it drives ("Xiaomi
// Releases HySparse2, Targeting Long-Horizon Reasoning for Agents", section
// "From Hybrid SWA to HySparse2, ..."), the shared cache and index set of the
// sparse layers ("Xiaomi Unveils HySparse2 for Faster Long-Context AI",
// sections "Two-Level KV Sharing" and "Token-Level Selection and Unified Local
// Access").  The pages describe one device; the split is this library's.
//
// Each merge reproduces the unsplit definition exactly up to rounding order:
//   * softmax partials (m_r, l_r, O_r normalised) of one (query, head):
//     M = max_r m_r, w_r = l_r exp(m_r - M), O = sum_r w_r O_r / sum_r w_r,
//     L = sum_r w_r - the same O, max and sum as one pass over all keys;
//   * top-k: every key of the global top-k (by score desc, position asc) is in
//     the local top-(k + window) of the rank that holds it, because at most
//     `window` of a rank's keys are window positions; the merge drops window
//     positions and keeps the k best of the union under the same order.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace hs2 {

// Softmax partials of R ranks -> merged output.  O_parts [R][rows][D] fp32
// (each normalised by its own sum), ml_parts [R][rows][2] = (m, 1/l) with
// 1/l = 0 for a rank that saw no key; O [rows][D] of type OT, ml [rows][2] =
// (M, 1/L) or null.  Grid: rows; D threads.
template <typename OT>
__global__ void __launch_bounds__(kD) k_cp_merge(const float* O_parts, const float* ml_parts, int R,
                                                 int64_t rows, OT* O, float* ml) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int64_t row = blockIdx.x;
  const int d = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) {
    const float il = __ldg(ml_parts + ((int64_t)r * rows + row) * 2 + 1);
    if (il > 0.f) M = fmaxf(M, __ldg(ml_parts + ((int64_t)r * rows + row) * 2));
  }
  float L = 0.f, acc = 0.f;
  for (int r = 0; r < R; ++r) {
    const float m = __ldg(ml_parts + ((int64_t)r * rows + row) * 2);
    const float il = __ldg(ml_parts + ((int64_t)r * rows + row) * 2 + 1);
    const float w = il > 0.f ? exp_shift(m, M) / il : 0.f;
    L += w;
    acc = fmaf(__ldg(O_parts + ((int64_t)r * rows + row) * kD + d), w, acc);
  }
  O[row * kD + d] = from_f<OT>(L > 0.f ? acc / L : 0.f);
  if (d == 0 && ml) {
    ml[row * 2] = M;
    ml[row * 2 + 1] = L > 0.f ? 1.f / L : 0.f;
  }
}

// A rank's local picks -> (score, global position) pairs.  idx/count: the local
// selection (window 0, so every entry below count is a pick); pos0 [B]: global
// position of the rank's local key 0 of each sequence.  Pairs [rows][kk], past
// count padded with position -1.  Grid: rows; 128 threads.
__global__ void __launch_bounds__(128) k_cp_pack(const float* scores, int64_t stride, const int32_t* idx,
                                                 const int32_t* count, int kk, const int64_t* qoff,
                                                 const int64_t* kvoff, int B, int Hkv,
                                                 const int64_t* pos0, float* pair_score,
                                                 int32_t* pair_pos, int* err) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  const int64_t row = blockIdx.x;
  const QueryRow q = query_row(qoff, kvoff, B, row / Hkv);
  int n = __ldg(count + row);
  if (n < 0 || n > kk) {
    if (threadIdx.x == 0) record_error(err, HS2_ERR_DEVICE_INPUT);
    n = 0;
  }
  const int64_t p0 = __ldg(pos0 + q.b);
  for (int i = threadIdx.x; i < kk; i += blockDim.x) {
    float sc = 0.f;
    int64_t gp = -1;
    if (i < n) {
      const int32_t j = __ldg(idx + row * kk + i);
      if (j >= 0 && j < stride && j <= q.t && p0 >= 0 && p0 + j <= INT32_MAX) {
        sc = __ldg(scores + row * stride + j);
        gp = p0 + j;
      } else if (j >= 0) {
        record_error(err, HS2_ERR_DEVICE_INPUT);
      }
    }
    pair_score[row * kk + i] = sc;
    pair_pos[row * kk + i] = (int32_t)gp;
  }
}

// Global top-k from the ranks' pairs (R x kk per row, kk = k + window): keys
// at positions <= t - window are candidates; the k best by (score desc,
// position asc) are written ascending, then the window max(0, t-window+1)..t,
// then -1 padding; count = picks + window length (as hs2_topk_select).  t from
// the global offsets.  The candidates are compacted into shared memory as
// (position << 32 | score key); a three-pass radix select (11/11/10 bits)
// finds the k-th largest score key T and how many keys equal to T to take
// (kr); every key > T is taken, and the kr lowest positions among the keys ==
// T (all of them in the usual case of no ties at T; else after ordering the
// candidates by position); the picks are then sorted by position.  Grid:
// rows; kSelThreads threads (the block-level digit search assumes it);
// dynamic shared memory kCpMergeCap x 8 bytes of keys + kCpPickCap x 4 bytes.
constexpr int kCpMergeThreads = kSelThreads;
constexpr int kCpMergeCap = 16384;  // R x kk at most (a power of two)
constexpr int kCpPickCap = 2048;    // k at most

__global__ void __launch_bounds__(kSelThreads) k_cp_topk_merge(
    const float* pair_score, const int32_t* pair_pos, int R, int kk, int k, int window,
    const int64_t* qoff, const int64_t* kvoff, int B, int Hkv, int64_t rows, int32_t* idx,
    int out_stride, int32_t* count) {
  grid_dep_wait();  // the previous kernel on the stream has finished
  extern __shared__ __align__(16) uint64_t cpm_keys[];
  int32_t* picks = reinterpret_cast<int32_t*>(cpm_keys + kCpMergeCap);
  __shared__ uint32_t hist[kSelBins];
  __shared__ int scan_sh[kSelThreads / 32 + 1];
  __shared__ int nvalid, ngt, neq, ntie;
  __shared__ uint32_t s_digit;
  __shared__ int s_rem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = blockIdx.x;
  const QueryRow q = query_row(qoff, kvoff, B, row / Hkv);
  const int64_t cut = q.t - window;  // candidates: positions 0..cut
  if (threadIdx.x == 0) {
    nvalid = 0;
    ngt = 0;
    neq = 0;
    ntie = 0;
  }
  __syncthreads();
  const int n = R * kk;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int r = i / kk, j = i % kk;
    const int64_t at = ((int64_t)r * rows + row) * kk + j;
    const int32_t pos = __ldg(pair_pos + at);
    if (pos >= 0 && pos <= cut)
      cpm_keys[atomicAdd(&nvalid, 1)] = ((uint64_t)(uint32_t)pos << 32) | score_key(__ldg(pair_score + at));
  }
  __syncthreads();
  const int nv = nvalid;
  const int npick = nv < k ? nv : k;
  if (nv <= k) {
    for (int i = threadIdx.x; i < nv; i += blockDim.x) picks[i] = (int32_t)(cpm_keys[i] >> 32);
  } else {
    uint32_t pre = 0;
    int need = k;
    for (int pass = 0; pass < 3; ++pass) {
      for (int i = threadIdx.x; i < kSelBins; i += blockDim.x) hist[i] = 0u;
      __syncthreads();
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t mask = pass == 2 ? 0x3FFu : 0x7FFu;
      const int pshift = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
      for (int base = warp * 32; base < nv; base += blockDim.x) {
        const int i = base + lane;
        const uint32_t u = i < nv ? (uint32_t)cpm_keys[i] : 0u;
        const bool ok = i < nv && (pass == 0 || (u >> pshift) == pre);
        sel_hist_add(hist, (u >> shift) & mask, ok);
      }
      __syncthreads();
      sel_block_find(hist, pass == 2 ? 1024 : kSelBins, need, scan_sh, &s_digit, &s_rem);
      pre = pass == 0 ? s_digit : ((pre << (pass == 1 ? 11 : 10)) | s_digit);
      need = s_rem;
    }
    const uint32_t T = pre;
    const int kr = need;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const uint32_t u = (uint32_t)cpm_keys[i];
      if (u > T) picks[atomicAdd(&ngt, 1)] = (int32_t)(cpm_keys[i] >> 32);
      else if (u == T) atomicAdd(&neq, 1);
    }
    __syncthreads();
    const int g = ngt;
    if (kr == neq) {  // every key equal to T is taken
      for (int i = threadIdx.x; i < nv; i += blockDim.x)
        if ((uint32_t)cpm_keys[i] == T) picks[g + atomicAdd(&ntie, 1)] = (int32_t)(cpm_keys[i] >> 32);
    } else {  // more ties than places: take the lowest positions among them
      sel_sort_asc(cpm_keys, nv, sel_pow2_at_least(nv), ~uint64_t(0));
      const int E = (nv + blockDim.x - 1) / blockDim.x;
      const int lo = min(nv, (int)threadIdx.x * E), hi = min(nv, lo + E);
      int mine = 0;
      for (int i = lo; i < hi; ++i) mine += (uint32_t)cpm_keys[i] == T;
      int tot;
      int tb = block_exclusive_scan(mine, scan_sh, &tot);
      for (int i = lo; i < hi; ++i)
        if ((uint32_t)cpm_keys[i] == T) {
          if (tb < kr) picks[g + tb] = (int32_t)(cpm_keys[i] >> 32);
          ++tb;
        }
    }
  }
  __syncthreads();
  sel_sort_asc(picks, npick, sel_pow2_at_least(npick), INT32_MAX);
  int32_t* out = idx + row * out_stride;
  const int64_t wlen = q.t + 1 < window ? (q.t + 1 > 0 ? q.t + 1 : 0) : window;
  const int64_t w0 = q.t - wlen + 1;
  for (int i = threadIdx.x; i < out_stride; i += blockDim.x) {
    int32_t v = -1;
    if (i < npick) v = picks[i];
    else if (i < npick + wlen) v = (int32_t)(w0 + (i - npick));
    out[i] = v;
  }
  if (threadIdx.x == 0) count[row] = (int32_t)(npick + wlen);
}

}  // namespace hs2
