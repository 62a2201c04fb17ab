// hs2.cu - the C ABI (include/hs2.h): argument checks, workspace planning and
// kernel launches of the HySparse2 hybrid-block attention path on sm_100a.
// One translation unit, so the device error word is a single object.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "hs2.h"
#include "decode_attn.cuh"
#include "select.cuh"
#include "sparse_attn.cuh"
#include "chunk_attn.cuh"

namespace hs2 {

__device__ int g_device_error;  // first error recorded by a kernel, 0 if none

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDecStages = 3;     // bf16 decode ring depth (2 CTAs per SM)
constexpr size_t kAlign = 256;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

hs2_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HS2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error) != cudaSuccess)
      return HS2_ERR_CUDA;
    const int dec_smem = kDecStages * kDecStageBytes + 1024;
    if (cudaFuncSetAttribute(k_decode_bf16<kDecStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dec_smem) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaFuncSetAttribute(k_sparse_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * 256 * kSpRowBytes + 256) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaFuncSetAttribute(k_chunk_bf16<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kChStages * 2 * kChKBytes + 1024) != cudaSuccess ||
        cudaFuncSetAttribute(k_chunk_bf16<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kChStages * kChKBytes + 1024) != cudaSuccess)
      return HS2_ERR_CUDA;
    d.ready = true;
  }
  *out = &d;
  return HS2_OK;
}

// Bump allocator over the caller's workspace (sizes rounded to 256 bytes).
struct Carve {
  char* base;
  size_t used = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t n) {
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += (n * sizeof(T) + kAlign - 1) / kAlign * kAlign;
    return p;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hs2_status check_problem(const hs2_problem* p) {
  if (!p) return HS2_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv != 0) return HS2_ERR_INVALID_ARG;
  if (p->reserved != 0) return HS2_ERR_INVALID_ARG;
  if (p->dtype != HS2_F32 && p->dtype != HS2_BF16) return HS2_ERR_INVALID_ARG;
  if (!p->q_offsets || !p->kv_offsets) return HS2_ERR_INVALID_ARG;
  if (p->total_q < 0 || p->total_kv < 0 || p->max_q_len < 0 || p->max_kv_len < 0)
    return HS2_ERR_INVALID_ARG;
  if (p->max_q_len > p->max_kv_len || p->total_q > (int64_t)p->B * p->max_q_len ||
      p->total_kv > (int64_t)p->B * p->max_kv_len)
    return HS2_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return HS2_ERR_INVALID_ARG;
  if (p->D != kD) return HS2_ERR_UNSUPPORTED;
  if (p->total_kv >= (int64_t(1) << 31) || p->max_kv_len >= (int64_t(1) << 31) ||
      p->total_q * p->Hkv >= (int64_t(1) << 31))
    return HS2_ERR_UNSUPPORTED;
  const int G = p->Hq / p->Hkv;
  if (p->dtype == HS2_BF16 && G > 8) return HS2_ERR_UNSUPPORTED;
  if (p->dtype == HS2_F32 && G > 16) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

hs2_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

// --------------------------------------------------------------------------
// full attention: decode plan
// --------------------------------------------------------------------------
struct DecodePlan {
  int P;
  float *logits, *pm, *pl, *po, *ml;
  size_t bytes;
};

DecodePlan plan_decode(const hs2_problem* p, const DeviceInfo& dev, void* ws) {
  DecodePlan pl{};
  const int G = p->Hq / p->Hkv;
  const int per_sm = p->dtype == HS2_BF16 ? 2 : 4;
  const int64_t target = std::max<int64_t>(1, (int64_t)dev.sms * per_sm / p->Hkv);
  const int64_t by_size = std::max<int64_t>(1, (p->total_kv + kDecTile - 1) / kDecTile);
  pl.P = (int)std::min(target, by_size);
  Carve c(ws);
  const size_t slots = (size_t)(pl.P + p->B) * p->Hkv * kDecWarps * G;
  pl.logits = c.take<float>((size_t)p->total_kv * p->Hq);
  pl.pm = c.take<float>(slots);
  pl.pl = c.take<float>(slots);
  pl.po = c.take<float>(slots * kD);
  pl.ml = c.take<float>((size_t)p->total_q * p->Hq * 2);
  pl.bytes = c.used;
  return pl;
}

hs2_status encode_kv_map(CUtensorMap* map, const void* base, const hs2_problem* p) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return HS2_ERR_CUDA;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)p->Hkv,
                              (cuuint64_t)std::max<int64_t>(p->total_kv, 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)p->Hkv * kD * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kDecTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HS2_OK : HS2_ERR_CUDA;
}

template <int GP>
void launch_decode_f32(dim3 grid, cudaStream_t st, const DecodeArgs& a) {
  k_decode_f32<GP><<<grid, 32 * kDecWarps, 0, st>>>(a);
}

hs2_status run_decode(const hs2_problem* p, const DeviceInfo& dev, const void* Q, const void* K,
                      const void* V, void* O, float* scores, int64_t stride, void* ws,
                      cudaStream_t st) {
  const DecodePlan pl = plan_decode(p, dev, ws);
  DecodeArgs a{};
  a.Q = Q; a.K = K; a.V = V;
  a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv; a.P = pl.P;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.logits = pl.logits; a.pm = pl.pm; a.pl = pl.pl; a.po = pl.po; a.err = dev.err;
  const dim3 grid(pl.P, p->Hkv);
  if (p->dtype == HS2_BF16) {
    CUtensorMap mk, mv;
    if (encode_kv_map(&mk, K, p) != HS2_OK || encode_kv_map(&mv, V, p) != HS2_OK) return HS2_ERR_CUDA;
    k_decode_bf16<kDecStages><<<grid, 32 * (kDecWarps + 1), kDecStages * kDecStageBytes + 1024, st>>>(mk, mv, a);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    k_decode_combine<bf16><<<dim3(p->B, p->Hkv), kD, 0, st>>>(a, static_cast<bf16*>(O), pl.ml);
  } else {
    const int G = a.G;
    if (G <= 1) launch_decode_f32<1>(grid, st, a);
    else if (G <= 2) launch_decode_f32<2>(grid, st, a);
    else if (G <= 4) launch_decode_f32<4>(grid, st, a);
    else if (G <= 8) launch_decode_f32<8>(grid, st, a);
    else launch_decode_f32<16>(grid, st, a);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    k_decode_combine<float><<<dim3(p->B, p->Hkv), kD, 0, st>>>(a, static_cast<float*>(O), pl.ml);
  }
  if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  if (p->total_kv > 0) {
    k_finalize_scores<<<(unsigned)((p->total_kv + 63) / 64), 256, 0, st>>>(a, pl.ml, scores, stride);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  }
  return HS2_OK;
}


// --------------------------------------------------------------------------
// full attention: chunk plan (more than one query token per sequence)
// --------------------------------------------------------------------------
struct ChunkPlan {
  float* ml;
  size_t bytes;
};

ChunkPlan plan_chunk(const hs2_problem* p, const DeviceInfo&, void* ws) {
  ChunkPlan c{};
  Carve w(ws);
  c.ml = w.take<float>((size_t)p->total_q * p->Hq * 2);
  c.bytes = w.used;
  return c;
}

hs2_status check_chunk(const hs2_problem* p) {
  const int G = p->Hq / p->Hkv;
  if (p->dtype == HS2_BF16 && (G & (G - 1)) != 0) return HS2_ERR_UNSUPPORTED;
  if (p->dtype == HS2_F32 && p->total_q > 65535) return HS2_ERR_UNSUPPORTED;
  if (p->B > 65535) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

template <int GP>
void launch_chunk_f32(const hs2_problem* p, cudaStream_t st, const ChunkArgs& a) {
  k_chunk_fwd_f32<GP><<<dim3((unsigned)p->total_q, p->Hkv), 128, 0, st>>>(a);
  k_chunk_scores_f32<GP><<<dim3((unsigned)((p->max_kv_len + 31) / 32), p->Hkv, (unsigned)p->total_q), 128, 0, st>>>(a);
}

hs2_status run_chunk(const hs2_problem* p, const DeviceInfo& dev, const void* Q, const void* K,
                     const void* V, void* O, float* scores, int64_t stride, void* ws,
                     cudaStream_t st) {
  hs2_status s = check_chunk(p);
  if (s != HS2_OK) return s;
  const ChunkPlan pl = plan_chunk(p, dev, ws);
  ChunkArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.O = O; a.ml = pl.ml; a.scores = scores; a.stride = stride; a.err = dev.err;
  if (p->dtype == HS2_BF16) {
    a.QT = kChRows / a.G;
    CUtensorMap mk, mv;
    if (encode_kv_map(&mk, K, p) != HS2_OK || encode_kv_map(&mv, V, p) != HS2_OK) return HS2_ERR_CUDA;
    const dim3 grid((unsigned)((p->max_q_len + a.QT - 1) / a.QT), p->Hkv, p->B);
    k_chunk_bf16<false><<<grid, 32 * (kChWarps + 1), kChStages * 2 * kChKBytes + 1024, st>>>(mk, mv, a);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    k_chunk_bf16<true><<<grid, 32 * (kChWarps + 1), kChStages * kChKBytes + 1024, st>>>(mk, mv, a);
    return launch_status();
  }
  a.QT = 1;
  const int G = a.G;
  if (G <= 1) launch_chunk_f32<1>(p, st, a);
  else if (G <= 2) launch_chunk_f32<2>(p, st, a);
  else if (G <= 4) launch_chunk_f32<4>(p, st, a);
  else if (G <= 8) launch_chunk_f32<8>(p, st, a);
  else launch_chunk_f32<16>(p, st, a);
  return launch_status();
}

// --------------------------------------------------------------------------
// selection
// --------------------------------------------------------------------------
struct SelectPlan {
  int nslices;
  uint32_t *hist, *ticket, *prefix;
  int32_t *krem, *cnt;
  size_t bytes;
};

SelectPlan plan_select(int64_t rows, int64_t max_len, Carve& c) {
  SelectPlan s{};
  s.nslices = (int)std::max<int64_t>(1, (max_len + kSelSlice - 1) / kSelSlice);
  const size_t before = c.used;
  s.hist = c.take<uint32_t>((size_t)rows * kSelBins);
  s.ticket = c.take<uint32_t>((size_t)rows);
  s.prefix = c.take<uint32_t>((size_t)rows);
  s.krem = c.take<int32_t>((size_t)rows);
  s.cnt = c.take<int32_t>((size_t)rows * s.nslices * 2);
  s.bytes = c.used - before;
  return s;
}

// Runs the radix select over ``data`` rows and writes the ascending selection
// to ``out``; ``count`` non-null for token rows (window, padding and count).
hs2_status run_select(const hs2_problem* p, const DeviceInfo& dev, const SelectPlan& sp,
                      const float* data, int64_t stride, int k, int window, int block,
                      int32_t* out, int64_t out_stride, int32_t* count, cudaStream_t st) {
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  // histogram and tickets start at zero; the last CTA of each pass cleans up after itself
  if (cudaMemsetAsync(sp.hist, 0, (size_t)rows * kSelBins * 4, st) != cudaSuccess) return HS2_ERR_CUDA;
  if (cudaMemsetAsync(sp.ticket, 0, (size_t)rows * 4, st) != cudaSuccess) return HS2_ERR_CUDA;
  SelectArgs a{};
  a.data = data; a.stride = stride; a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hkv = p->Hkv; a.rows = rows; a.k = k; a.window = window; a.block = block;
  a.nslices = sp.nslices; a.hist = sp.hist; a.ticket = sp.ticket; a.prefix = sp.prefix;
  a.krem = sp.krem; a.cnt = sp.cnt; a.out = out; a.out_stride = out_stride; a.err = dev.err;
  const dim3 grid((unsigned)rows, sp.nslices);
  for (int pass = 0; pass < 3; ++pass) {
    k_select_hist<<<grid, kSelThreads, 0, st>>>(a, pass);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  }
  k_select_count<<<grid, kSelThreads, 0, st>>>(a);
  if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  k_select_compact<<<grid, kSelThreads, 0, st>>>(a, count);
  return launch_status();
}

// --------------------------------------------------------------------------
// sparse attention plan
// --------------------------------------------------------------------------
struct SparsePlan {
  int chunk, nchunk;
  float *pm, *pl, *po;
  uint32_t* ticket;
  size_t bytes;
};

SparsePlan plan_sparse(const hs2_problem* p, const DeviceInfo& dev, int idx_stride, void* ws) {
  SparsePlan s{};
  const int64_t rows = std::max<int64_t>(1, p->total_q * p->Hkv);
  const int64_t target = (int64_t)dev.sms * 2;
  int64_t ch = (rows * idx_stride + target - 1) / target;
  ch = (ch + 15) / 16 * 16;
  s.chunk = (int)std::min<int64_t>(256, std::max<int64_t>(16, ch));
  s.nchunk = (int)std::max<int64_t>(1, (idx_stride + s.chunk - 1) / s.chunk);
  const int G = p->Hq / p->Hkv;
  Carve c(ws);
  const size_t slots = (size_t)rows * s.nchunk * kSpWarps * G;
  s.pm = c.take<float>(slots);
  s.pl = c.take<float>(slots);
  s.po = c.take<float>(slots * kD);
  s.ticket = c.take<uint32_t>((size_t)rows);
  s.bytes = c.used;
  return s;
}

template <int GP>
void launch_sparse_f32(dim3 grid, cudaStream_t st, const SparseArgs& a) {
  k_sparse_f32<GP><<<grid, 32 * kSpWarps, 0, st>>>(a);
}

hs2_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return HS2_OK;
  if (!ws || have < need || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return HS2_ERR_WORKSPACE;
  return HS2_OK;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

hs2_status hs2_full_attn_workspace_size(const hs2_problem* p, size_t* bytes) {
  if (!bytes) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  if (p->max_q_len <= 1) *bytes = plan_decode(p, *dev, nullptr).bytes;
  else *bytes = plan_chunk(p, *dev, nullptr).bytes;
  return HS2_OK;
}

hs2_status hs2_full_attn_scores(const hs2_problem* p, const void* Q, const void* K, const void* V,
                                void* O, float* scores, int64_t score_stride, void* workspace,
                                size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (!Q || !K || !V || !O || !scores) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(scores))
    return HS2_ERR_INVALID_ARG;
  if (score_stride < p->max_kv_len || score_stride < 1) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->total_q == 0) return HS2_OK;
  if (p->max_q_len <= 1) {
    if ((s = check_ws(workspace, workspace_bytes, plan_decode(p, *dev, nullptr).bytes)) != HS2_OK) return s;
    return run_decode(p, *dev, Q, K, V, O, scores, score_stride, workspace, st);
  }
  if ((s = check_ws(workspace, workspace_bytes, plan_chunk(p, *dev, nullptr).bytes)) != HS2_OK) return s;
  return run_chunk(p, *dev, Q, K, V, O, scores, score_stride, workspace, st);
}

hs2_status hs2_topk_workspace_size(const hs2_problem* p, int32_t k, int32_t window, size_t* bytes) {
  if (!bytes || k < 1 || window < 1) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  Carve c(nullptr);
  plan_select(p->total_q * p->Hkv, p->max_kv_len, c);
  *bytes = c.used;
  return HS2_OK;
}

hs2_status hs2_topk_select(const hs2_problem* p, const float* scores, int64_t score_stride, int32_t k,
                           int32_t window, int32_t* idx, int32_t* count, void* workspace,
                           size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (!scores || !idx || !count || k < 1 || window < 1) return HS2_ERR_INVALID_ARG;
  if ((int64_t)k + window >= (int64_t(1) << 30)) return HS2_ERR_INVALID_ARG;
  if (!aligned16(scores) || score_stride < std::max<int64_t>(1, p->max_kv_len)) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  Carve c(nullptr);
  plan_select(p->total_q * p->Hkv, p->max_kv_len, c);
  if ((s = check_ws(workspace, workspace_bytes, c.used)) != HS2_OK) return s;
  Carve w(workspace);
  const SelectPlan sp = plan_select(p->total_q * p->Hkv, p->max_kv_len, w);
  return run_select(p, *dev, sp, scores, score_stride, k, window, 0, idx, (int64_t)k + window, count,
                    static_cast<cudaStream_t>(stream));
}

hs2_status hs2_block_select_workspace_size(const hs2_problem* p, int32_t n_blocks, int32_t block,
                                           int32_t window, size_t* bytes) {
  if (!bytes || n_blocks < 1 || block < 1 || window < 1) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  const int64_t rows = p->total_q * p->Hkv;
  const int64_t nb = std::max<int64_t>(1, (p->max_kv_len + block - 1) / block);
  Carve c(nullptr);
  c.take<float>((size_t)rows * nb);
  c.take<int32_t>((size_t)rows * n_blocks);
  plan_select(rows, nb, c);
  *bytes = c.used;
  return HS2_OK;
}

hs2_status hs2_block_select(const hs2_problem* p, const float* scores, int64_t score_stride,
                            int32_t n_blocks, int32_t block, int32_t window, int32_t* idx,
                            int32_t* count, void* workspace, size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (!scores || !idx || !count || n_blocks < 1 || block < 1 || window < 1) return HS2_ERR_INVALID_ARG;
  if ((int64_t)n_blocks * block + window >= (int64_t(1) << 30)) return HS2_ERR_INVALID_ARG;
  if (!aligned16(scores) || score_stride < std::max<int64_t>(1, p->max_kv_len)) return HS2_ERR_INVALID_ARG;
  size_t need;
  if ((s = hs2_block_select_workspace_size(p, n_blocks, block, window, &need)) != HS2_OK) return s;
  if ((s = check_ws(workspace, workspace_bytes, need)) != HS2_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  const int64_t nb = std::max<int64_t>(1, (p->max_kv_len + block - 1) / block);
  Carve w(workspace);
  float* bmax = w.take<float>((size_t)rows * nb);
  int32_t* bsel = w.take<int32_t>((size_t)rows * n_blocks);
  const SelectPlan sp = plan_select(rows, nb, w);
  k_block_max<<<dim3((unsigned)rows, (unsigned)((nb + 7) / 8)), 256, 0, st>>>(
      scores, score_stride, p->q_offsets, p->kv_offsets, p->B, p->Hkv, block, window, bmax, nb, dev->err);
  if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  if ((s = run_select(p, *dev, sp, bmax, nb, n_blocks, window, block, bsel, n_blocks, nullptr, st)) != HS2_OK)
    return s;
  k_block_expand<<<(unsigned)rows, 256, 0, st>>>(bsel, n_blocks, p->q_offsets, p->kv_offsets, p->B,
                                                 p->Hkv, block, window, idx,
                                                 (int64_t)n_blocks * block + window, count);
  return launch_status();
}

hs2_status hs2_sparse_attn_workspace_size(const hs2_problem* p, int32_t idx_stride, size_t* bytes) {
  if (!bytes || idx_stride < 1) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  *bytes = plan_sparse(p, *dev, idx_stride, nullptr).bytes;
  return HS2_OK;
}

hs2_status hs2_sparse_attn(const hs2_problem* p, const void* Q_l, const void* K, const void* V,
                           const int32_t* idx, const int32_t* count, int32_t idx_stride, void* O_l,
                           void* workspace, size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (!Q_l || !K || !V || !idx || !count || !O_l || idx_stride < 1) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q_l) || !aligned16(K) || !aligned16(V) || !aligned16(O_l)) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const SparsePlan sp0 = plan_sparse(p, *dev, idx_stride, nullptr);
  if ((s = check_ws(workspace, workspace_bytes, sp0.bytes)) != HS2_OK) return s;
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SparsePlan sp = plan_sparse(p, *dev, idx_stride, workspace);
  if (cudaMemsetAsync(sp.ticket, 0, (size_t)rows * 4, st) != cudaSuccess) return HS2_ERR_CUDA;
  SparseArgs a{};
  a.Q = Q_l; a.K = K; a.V = V; a.idx = idx; a.count = count; a.idx_stride = idx_stride;
  a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.chunk = sp.chunk; a.nchunk = sp.nchunk; a.pm = sp.pm; a.pl = sp.pl; a.po = sp.po;
  a.ticket = sp.ticket; a.O = O_l; a.err = dev->err;
  const dim3 grid((unsigned)rows, sp.nchunk);
  if (p->dtype == HS2_BF16) {
    const size_t smem = 2 * (size_t)sp.chunk * kSpRowBytes + sp.chunk;
    k_sparse_bf16<<<grid, 32 * kSpWarps, smem, st>>>(a);
  } else {
    const int G = a.G;
    if (G <= 1) launch_sparse_f32<1>(grid, st, a);
    else if (G <= 2) launch_sparse_f32<2>(grid, st, a);
    else if (G <= 4) launch_sparse_f32<4>(grid, st, a);
    else if (G <= 8) launch_sparse_f32<8>(grid, st, a);
    else launch_sparse_f32<16>(grid, st, a);
  }
  return launch_status();
}

hs2_status hs2_get_last_device_error(void* stream) {
  DeviceInfo* dev;
  hs2_status s = device_info(&dev);
  if (s != HS2_OK) return s;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HS2_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, dev->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HS2_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(dev->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return HS2_ERR_CUDA;
  return static_cast<hs2_status>(v);
}

const char* hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARG: return "invalid argument";
    case HS2_ERR_UNSUPPORTED: return "unsupported shape or type";
    case HS2_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case HS2_ERR_CUDA: return "CUDA runtime error";
    case HS2_ERR_TIMEOUT: return "a bounded device wait ran out";
    case HS2_ERR_DEVICE_INPUT: return "device found inputs that break the contract";
  }
  return "unknown status";
}

int32_t hs2_version(void) { return (0 << 16) | 1; }

}  // extern "C"
