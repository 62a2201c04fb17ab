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
#include "kv_append.cuh"
#include "bridge.cuh"
#include "sparse_attn.cuh"
#include "chunk_attn.cuh"
#include "chunk_tc.cuh"
#include "wait_selftest.cuh"
#include "context_parallel.cuh"

namespace hs2 {

__device__ int g_device_error;  // first error recorded by a kernel, 0 if none

namespace {

// Launches ``kern`` on ``st`` with programmatic dependent launch allowed (each
// kernel starts with griddepcontrol.wait, so nothing is read or written before
// the previous kernel on the stream has finished) and, if cluster > 0, in
// thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = (unsigned)n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int kMaxDevices = 64;
constexpr int kDecStages = 3;     // bf16 decode ring depth (2 CTAs per SM)
constexpr int kMaxHq = 192;      // query heads the score finalize can stage
constexpr int kSelSmemKeys = 16384;  // select: per-CTA slice kept in shared memory (64 KB)
constexpr size_t kAlign = 256;

struct DeviceInfo {
  bool ready = false;
  bool cluster16 = false;  // non-portable 16-CTA clusters allowed for the select kernel
  bool sparse16 = false;   // ... and for the bf16 sparse kernel
  int sms = 0;
  int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];

constexpr size_t kCpMergeSmem = (size_t)kCpMergeCap * 8 + (size_t)kCpPickCap * 4;
std::mutex g_dev_mu;

template <int G>
cudaError_t set_chunk_tc_smem() {
  return cudaFuncSetAttribute(k_chunk_tc<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chunk_tc_smem());
}

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
                             (int)kSpGatherSmem) != cudaSuccess ||
        cudaFuncSetAttribute(k_sparse_rows_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSrSmem) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (set_chunk_tc_smem<1>() != cudaSuccess || set_chunk_tc_smem<2>() != cudaSuccess ||
        set_chunk_tc_smem<4>() != cudaSuccess || set_chunk_tc_smem<8>() != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaFuncSetAttribute(k_select_cluster<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelSmemKeys * 4) != cudaSuccess ||
        cudaFuncSetAttribute(k_select_cluster<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelSmemKeys * 4) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaFuncSetAttribute(k_kv_bridge<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bridge_smem<256>()) != cudaSuccess ||
        cudaFuncSetAttribute(k_kv_bridge<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bridge_smem<128>()) != cudaSuccess)
      return HS2_ERR_CUDA;
    constexpr int ss_smem = kSsCap * 8 + kSsSortMax * 4;
    if (cudaFuncSetAttribute(k_select_sampled<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ss_smem) != cudaSuccess ||
        cudaFuncSetAttribute(k_select_sampled<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ss_smem) != cudaSuccess ||
        cudaFuncSetAttribute(k_select_sampled<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ss_smem) != cudaSuccess)
      return HS2_ERR_CUDA;
    d.cluster16 = cudaFuncSetAttribute(k_select_cluster<16>,
                                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
                  cudaFuncSetAttribute(k_select_sampled<16>,
                                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    d.sparse16 = cudaFuncSetAttribute(k_sparse_bf16, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                 cudaSuccess;
    cudaGetLastError();  // a refused non-portable size is not an error
    if (cudaFuncSetAttribute(k_finalize_scores<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)finalize_smem(16)) != cudaSuccess ||
        cudaFuncSetAttribute(k_finalize_scores<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)finalize_smem(16)) != cudaSuccess)
      return HS2_ERR_CUDA;
    if (cudaFuncSetAttribute(k_cp_topk_merge, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kCpMergeSmem) != cudaSuccess)
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
  if (p->B > 65535 || p->Hkv > 65535 || p->Hq > kMaxHq) return HS2_ERR_UNSUPPORTED;
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
  pl.logits = c.take<float>((size_t)p->Hkv * p->total_kv * logit_pitch(G));
  pl.pm = c.take<float>(slots);
  pl.pl = c.take<float>(slots);
  pl.po = c.take<float>(slots * kD);
  pl.ml = c.take<float>((size_t)p->total_q * p->Hq * 2);
  pl.bytes = c.used;
  return pl;
}

// 3-D bf16 tensor map over a [rows, heads, 128] token-major array, boxes of
// 64 dims x box_heads x box_rows, 128-byte swizzle.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return encode;
}

hs2_status encode_map3(CUtensorMap* map, const void* base, int64_t rows, int heads, int box_heads,
                       int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return HS2_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)std::max<int64_t>(rows, 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)heads * kD * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HS2_OK : HS2_ERR_CUDA;
}

// 2-D bf16 tensor map over a row-major [rows, cols] array, boxes of 64 columns
// x box_rows rows, 128-byte swizzle.
hs2_status encode_map2(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return HS2_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)std::max<int64_t>(rows, 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HS2_OK : HS2_ERR_CUDA;
}

hs2_status encode_kv_map(CUtensorMap* map, const void* base, const hs2_problem* p) {
  return encode_map3(map, base, p->total_kv, p->Hkv, 1, kDecTile);
}

template <int GP>
void launch_decode_f32(dim3 grid, cudaStream_t st, const DecodeArgs& a) {
  launch(k_decode_f32<GP>, dim3(grid), dim3(32 * kDecWarps), 0, st, 0, a);
}

// Decode scores from the logits the split-context pass kept and the final
// (m, 1/l) of every (query, head).
// The finish of a decode call: O (when ``O`` is given: merged from the
// partials, as are the statistics) and the scores (statistics from ``ml_in``
// when it is given).
template <typename OT>
hs2_status launch_finalize(const hs2_problem* p, const DecodeArgs& a, OT* O, const float* ml_in, float* scores,
                           int64_t stride, cudaStream_t st) {
  if (p->max_kv_len <= 0 || p->total_kv <= 0) return HS2_OK;
  launch(k_finalize_scores<OT>, dim3((unsigned)a.P, (unsigned)p->Hkv), dim3(kFinThreads), finalize_smem(a.G), st,
         0, a, O, ml_in, scores, stride);
  return launch_status();
}

// Decode: split-context pass, combine, score finalize.  partial_ml != null:
// context-parallel partial - O is float32, the combine writes (m, 1/l) to
// partial_ml, and no scores are made (hs2_cp_scores makes them later from the
// logits kept in the workspace).
hs2_status run_decode(const hs2_problem* p, const DeviceInfo& dev, const void* Q, const void* K,
                      const void* V, void* O, float* scores, int64_t stride, void* ws,
                      cudaStream_t st, float* partial_ml = nullptr) {
  const DecodePlan pl = plan_decode(p, dev, ws);
  DecodeArgs a{};
  a.Q = Q; a.K = K; a.V = V;
  a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv; a.P = pl.P;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.logits = pl.logits; a.pm = pl.pm; a.pl = pl.pl; a.po = pl.po; a.err = dev.err;
  a.Gp = logit_pitch(a.G);
  a.nw = p->dtype == HS2_BF16 ? 1 : kDecWarps;  // the bf16 pass folds its warps' partials
  const dim3 grid(pl.P, p->Hkv);
  const dim3 cgrid((unsigned)((int64_t)p->B * p->Hq));
  if (p->dtype == HS2_BF16) {
    CUtensorMap mk, mv;
    if (encode_kv_map(&mk, K, p) != HS2_OK || encode_kv_map(&mv, V, p) != HS2_OK) return HS2_ERR_CUDA;
    launch(k_decode_bf16<kDecStages>, dim3(grid), dim3(32 * (kDecWarps + 1)), kDecStages * kDecStageBytes + 1024, st, 0, mk, mv, a);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    if (!partial_ml) return launch_finalize(p, a, static_cast<bf16*>(O), nullptr, scores, stride, st);
    launch(k_decode_combine<float>, cgrid, dim3(kCombThreads), 0, st, 0, a, static_cast<float*>(O), partial_ml);
  } else {
    const int G = a.G;
    if (G <= 1) launch_decode_f32<1>(grid, st, a);
    else if (G <= 2) launch_decode_f32<2>(grid, st, a);
    else if (G <= 4) launch_decode_f32<4>(grid, st, a);
    else if (G <= 8) launch_decode_f32<8>(grid, st, a);
    else launch_decode_f32<16>(grid, st, a);
    if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
    if (!partial_ml) return launch_finalize(p, a, static_cast<float*>(O), nullptr, scores, stride, st);
    launch(k_decode_combine<float>, cgrid, dim3(kCombThreads), 0, st, 0, a, static_cast<float*>(O), partial_ml);
  }
  return launch_status();
}


// --------------------------------------------------------------------------
// full attention: chunk plan (more than one query token per sequence)
// --------------------------------------------------------------------------
struct ChunkPlan {
  float* ml;
  int ks;          // key ranges per query tile of the tensor-core kernel
  float* part_ml;  // ks > 1: each range's row statistics
  float* part_o;   // ks > 1: each range's share of O (float32)
  size_t bytes;
};

// Key ranges per query tile of the tensor-core chunk kernel (one CTA per SM):
// the count in 1 .. 8 that runs the CTAs in the fewest waves per unit of work
// (the smallest on a tie), each range keeping at least 64 key tiles (8192 keys)
// of the longest sequence: with 36 tiles a range (a 16K-key context) the two
// launches and the O shares cost more than the fuller waves win.
int chunk_ksplit(const hs2_problem* p, const DeviceInfo& dev) {
  if (p->dtype != HS2_BF16 || dev.sms <= 0) return 1;
  const int64_t G = p->Hq / p->Hkv;
  const int64_t QT = kTcQTiles * kTcRows / G;
  const int64_t units = (p->max_q_len + QT - 1) / QT * p->Hkv * p->B;
  const int64_t tiles = (p->max_kv_len + kTcKeys - 1) / kTcKeys;
  int best = 1;
  int64_t best_waves = (units + dev.sms - 1) / dev.sms;  // for ks = 1
  for (int k = 2; k <= 8; ++k) {
    if (tiles < 64 * (int64_t)k || (int64_t)p->B * k > 65535) break;
    const int64_t waves = (units * k + dev.sms - 1) / dev.sms;
    if (waves * best < best_waves * k) {  // waves / k < best_waves / best
      best = k;
      best_waves = waves;
    }
  }
  return best;
}

ChunkPlan plan_chunk(const hs2_problem* p, const DeviceInfo& dev, void* ws) {
  ChunkPlan c{};
  Carve w(ws);
  c.ml = w.take<float>((size_t)p->total_q * p->Hq * 2);
  c.ks = chunk_ksplit(p, dev);
  if (c.ks > 1) {
    c.part_ml = w.take<float>((size_t)c.ks * p->total_q * p->Hq * 2);
    c.part_o = w.take<float>((size_t)c.ks * p->total_q * p->Hq * kD);
  }
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

template <int G>
void launch_chunk_tc(dim3 grid, cudaStream_t st, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const ChunkArgs& a) {
  launch(k_chunk_tc<G>, grid, dim3(kTcThreads), chunk_tc_smem(), st, 0, mq, mk, mv, a);
}

template <int GP>
void launch_chunk_f32(const hs2_problem* p, cudaStream_t st, const ChunkArgs& a) {
  launch(k_chunk_fwd_f32<GP>, dim3(dim3((unsigned)p->total_q, p->Hkv)), dim3(128), 0, st, 0, a);
  launch(k_chunk_scores_f32<GP>, dim3(dim3((unsigned)((p->max_kv_len + 31) / 32), p->Hkv, (unsigned)p->total_q)), dim3(128), 0, st, 0, a);
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
    a.QT = kTcQTiles * kTcRows / a.G;  // queries per CTA (two Q tiles)
    CUtensorMap mq, mk, mv;
    if (encode_map3(&mq, Q, p->total_q, p->Hq, a.G, kTcRows / a.G) != HS2_OK ||
        encode_map3(&mk, K, p->total_kv, p->Hkv, 1, kTcKeys) != HS2_OK ||
        encode_map3(&mv, V, p->total_kv, p->Hkv, 1, kTcKeys) != HS2_OK)
      return HS2_ERR_CUDA;
    a.ksplit = pl.ks;
    a.part_ml = pl.part_ml;
    a.part_o = pl.part_o;
    const dim3 grid((unsigned)((p->max_q_len + a.QT - 1) / a.QT), p->Hkv, (unsigned)(p->B * pl.ks));
    auto run = [&](int mode) {
      a.mode = mode;
      switch (a.G) {
        case 1: launch_chunk_tc<1>(grid, st, mq, mk, mv, a); break;
        case 2: launch_chunk_tc<2>(grid, st, mq, mk, mv, a); break;
        case 4: launch_chunk_tc<4>(grid, st, mq, mk, mv, a); break;
        default: launch_chunk_tc<8>(grid, st, mq, mk, mv, a); break;
      }
    };
    if (pl.ks == 1) {
      run(0);
    } else {  // statistics per key range, then scores and O shares, then O
      run(1);
      run(2);
      const int64_t nrows = p->total_q * p->Hq;
      const int64_t n4 = nrows * (kD / 4);
      launch(k_chunk_o_sum, dim3((unsigned)((n4 + 255) / 256)), dim3(256), 0, st, 0,
             (const float*)pl.part_o, pl.ks, nrows, static_cast<bf16*>(O));
    }
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
// Runs the radix select over ``data`` rows and writes the ascending selection
// to ``out``; ``count`` non-null for token rows (window, padding and count).
// One cluster of CTAs per row: 16 when the rows are long and that size is
// allowed, else 8.
hs2_status run_select(const hs2_problem* p, const DeviceInfo& dev, const float* data,
                      int64_t stride, int64_t max_len, int k, int window, int block, int32_t* out,
                      int64_t out_stride, int32_t* count, cudaStream_t st) {
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  SelectArgs a{};
  a.data = data; a.stride = stride; a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hkv = p->Hkv; a.rows = rows; a.k = k; a.window = window; a.block = block;
  a.out = out; a.out_stride = out_stride; a.err = dev.err;
  const int64_t len = std::max<int64_t>(1, max_len);
  // k <= kSsSortMax: the sample-guided kernel, one CTA per row when the rows
  // alone fill the GPU, else a cluster per row; larger k: the exact kernel
  const bool sampled = k <= kSsSortMax;
  int cs = (dev.cluster16 && len > 8 * (int64_t)kSelSmemKeys) ? 16 : 8;
  if (sampled && rows >= 2 * (int64_t)dev.sms) cs = 1;
  int64_t S = (len + cs - 1) / cs;
  S = (S + kSelChunkAlign - 1) / kSelChunkAlign * kSelChunkAlign;
  a.slice = S;
  a.smem_keys = (!sampled && S <= kSelSmemKeys) ? 1 : 0;
  if (rows * cs >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)(rows * cs)), threads(kSelThreads);
  const size_t smem = sampled ? (size_t)kSsCap * 8 + kSsSortMax * 4 : (a.smem_keys ? (size_t)S * 4 : 0);
  cudaError_t e;
  if (sampled)
    e = cs == 16 ? launch(k_select_sampled<16>, grid, threads, smem, st, cs, a, count)
                 : (cs == 8 ? launch(k_select_sampled<8>, grid, threads, smem, st, cs, a, count)
                            : launch(k_select_sampled<1>, grid, threads, smem, st, cs, a, count));
  else
    e = cs == 16 ? launch(k_select_cluster<16>, grid, threads, smem, st, cs, a, count)
                 : launch(k_select_cluster<8>, grid, threads, smem, st, cs, a, count);
  return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

// --------------------------------------------------------------------------
// sparse attention: one cluster of kSpCluster CTAs per (query, KV group) row
// --------------------------------------------------------------------------
template <typename Kern>
cudaError_t launch_cluster(Kern kern, unsigned ctas, unsigned threads, size_t smem, int cs,
                           cudaStream_t st, const SparseArgs& a) {
  return launch(kern, dim3(ctas), dim3(threads), smem, st, cs, a);
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

hs2_status hs2_full_attn_launches(const hs2_problem* p, int32_t* n) {
  if (!n) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  if (p->total_q == 0) *n = 0;
  else if (p->max_q_len <= 1) *n = 2;
  else if (p->dtype == HS2_BF16) *n = chunk_ksplit(p, *dev) > 1 ? 3 : 1;
  else *n = 2;
  return HS2_OK;
}

hs2_status hs2_full_attn_scores(const hs2_problem* p, const void* Q, const void* K, const void* V,
                                void* O, float* scores, int64_t score_stride, void* workspace,
                                size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->total_q == 0) return HS2_OK;  // no query rows: nothing to read or write
  if (!Q || !K || !V || !O || !scores) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(scores))
    return HS2_ERR_INVALID_ARG;
  if (score_stride < p->max_kv_len || score_stride < 1) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
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
  *bytes = 0;  // the selection keeps all of its state on chip
  return HS2_OK;
}

hs2_status hs2_topk_select(const hs2_problem* p, const float* scores, int64_t score_stride, int32_t k,
                           int32_t window, int32_t* idx, int32_t* count, void* workspace,
                           size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (k < 1 || window < 1 || (int64_t)k + window >= (int64_t(1) << 30)) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no rows
  if (!scores || !idx || !count) return HS2_ERR_INVALID_ARG;
  if (!aligned16(scores) || score_stride < std::max<int64_t>(1, p->max_kv_len)) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  return run_select(p, *dev, scores, score_stride, p->max_kv_len, k, window, 0, idx,
                    (int64_t)k + window, count, static_cast<cudaStream_t>(stream));
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
  *bytes = c.used;
  return HS2_OK;
}

hs2_status hs2_block_select(const hs2_problem* p, const float* scores, int64_t score_stride,
                            int32_t n_blocks, int32_t block, int32_t window, int32_t* idx,
                            int32_t* count, void* workspace, size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (n_blocks < 1 || block < 1 || window < 1) return HS2_ERR_INVALID_ARG;
  if ((int64_t)n_blocks * block + window >= (int64_t(1) << 30)) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no rows: the workspace is not needed either
  if (!scores || !idx || !count) return HS2_ERR_INVALID_ARG;
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
  launch(k_block_max, dim3(dim3((unsigned)rows, (unsigned)((nb + 7) / 8))), dim3(256), 0, st, 0, 
      scores, score_stride, p->q_offsets, p->kv_offsets, p->B, p->Hkv, block, window, bmax, nb, dev->err);
  if (launch_status() != HS2_OK) return HS2_ERR_CUDA;
  if ((s = run_select(p, *dev, bmax, nb, nb, n_blocks, window, block, bsel, n_blocks, nullptr, st)) != HS2_OK)
    return s;
  launch(k_block_expand, dim3((unsigned)rows), dim3(256), 0, st, 0, bsel, n_blocks, p->q_offsets, p->kv_offsets,
         p->B, p->Hkv, block, window, score_stride, nb, idx, (int64_t)n_blocks * block + window, count,
         dev->err);
  return launch_status();
}

hs2_status hs2_sparse_attn_workspace_size(const hs2_problem* p, int32_t idx_stride, size_t* bytes) {
  if (!bytes || idx_stride < 1) return HS2_ERR_INVALID_ARG;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  *bytes = 0;  // the partials of a row are merged on chip, inside its cluster
  return HS2_OK;
}

namespace {
// One sparse-attention launch: index mode (idx/count) or window mode (window > 0).
// Context-parallel options of a sparse launch (see SparseArgs).
struct SparseShard {
  const int64_t* pos0;
  float* ml_out;
};

hs2_status run_sparse(const hs2_problem* p, const void* Q_l, const void* K, const void* V,
                      const int32_t* idx, const int32_t* count, int32_t idx_stride, int32_t window,
                      void* O_l, void* stream, const SparseShard* shard = nullptr) {
  hs2_status s;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  if (rows * kSpCluster >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  SparseArgs a{};
  a.Q = Q_l; a.K = K; a.V = V; a.idx = idx; a.count = count; a.idx_stride = idx_stride;
  a.window = window;
  a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.O = O_l; a.err = dev->err;
  if (shard) {
    a.pos0 = shard->pos0; a.ml_out = shard->ml_out; a.o_f32 = 1;
  }
  const unsigned ctas = (unsigned)(rows * kSpCluster);
  // the cluster kernel gathers rows through a 2-D tensor map of (position, KV head) rows
  const bool map_fits = p->total_kv * p->Hkv < (int64_t(1) << 31);
  cudaError_t e;
  if (p->dtype == HS2_BF16 && ((rows >= 4 * (int64_t)dev->sms && !shard) || !map_fits)) {
    // many rows (a chunk of queries): one CTA per row, no cluster
    e = launch(k_sparse_rows_bf16, dim3((unsigned)rows), dim3(32 * kSrWarps), kSrSmem, st, 0, a);
  } else if (p->dtype == HS2_BF16) {
    CUtensorMap mk;  // K rows by TMA; V rows by cp.async
    const int64_t map_rows = p->total_kv * p->Hkv;
    if (encode_map2(&mk, K, map_rows, kD, 1) != HS2_OK) return HS2_ERR_CUDA;
    // few rows (a small decode batch): 16 CTAs per row, half the gathers each
    const int cs = (dev->sparse16 && rows * 16 <= (int64_t)dev->sms) ? 16 : kSpCluster;
    e = launch(k_sparse_bf16, dim3((unsigned)(rows * cs)), dim3(32 * kSpWarps), kSpGatherSmem, st, cs, mk, a);
  } else {
    const int G = a.G;
    if (G <= 1) e = launch_cluster(k_sparse_f32<1>, ctas, 32 * kSpWarps, 0, kSpCluster, st, a);
    else if (G <= 2) e = launch_cluster(k_sparse_f32<2>, ctas, 32 * kSpWarps, 0, kSpCluster, st, a);
    else if (G <= 4) e = launch_cluster(k_sparse_f32<4>, ctas, 32 * kSpWarps, 0, kSpCluster, st, a);
    else if (G <= 8) e = launch_cluster(k_sparse_f32<8>, ctas, 32 * kSpWarps, 0, kSpCluster, st, a);
    else e = launch_cluster(k_sparse_f32<16>, ctas, 32 * kSpWarps, 0, kSpCluster, st, a);
  }
  return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}
}  // namespace

hs2_status hs2_sparse_attn(const hs2_problem* p, const void* Q_l, const void* K, const void* V,
                           const int32_t* idx, const int32_t* count, int32_t idx_stride, void* O_l,
                           void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (idx_stride < 1) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no query rows
  if (!Q_l || !K || !V || !idx || !count || !O_l) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q_l) || !aligned16(K) || !aligned16(V) || !aligned16(O_l)) return HS2_ERR_INVALID_ARG;
  return run_sparse(p, Q_l, K, V, idx, count, idx_stride, 0, O_l, stream);
}

hs2_status hs2_swa_attn(const hs2_problem* p, const void* Q, const void* K, const void* V,
                        int32_t window, void* O, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (window < 1) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no query rows
  if (!Q || !K || !V || !O) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return HS2_ERR_INVALID_ARG;
  return run_sparse(p, Q, K, V, nullptr, nullptr, 0, window, O, stream);
}

// ---------------------------------------------------------------------------
// Block selection without a caller workspace.  Some callers cannot hand the
// library device memory: a host engine or plugin interface that owns every
// allocation and offers no workspace pointer, or code that must not call
// cudaMalloc because it can synchronise the device and fragment a memory pool
// that the engine manages.  For them the scratch of block selection (block
// maxima and chosen block ids) lives in this fixed array instead.  Every GPU
// that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace hs2 {
namespace {
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device.  Host code only
// sees a stand-in for the array's name, so the address is looked up once per
// device, with that device current.
hs2_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HS2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HS2_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HS2_OK;
}
}  // namespace
}  // namespace hs2

hs2_status hs2_block_select_noalloc(const hs2_problem* p, const float* scores, int64_t score_stride,
                                    int32_t n_blocks, int32_t block, int32_t window, int32_t* idx,
                                    int32_t* count, void* stream) {
  size_t need = 0;
  hs2_status s = hs2_block_select_workspace_size(p, n_blocks, block, window, &need);
  if (s != HS2_OK) return s;
  if (need > kNoAllocScratchBytes) return HS2_ERR_WORKSPACE;  // larger than the fixed scratch
  if (p->total_q == 0) return HS2_OK;  // no rows: nothing to look up or launch
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != HS2_OK) return s;
  return hs2_block_select(p, scores, score_stride, n_blocks, block, window, idx, count, scratch,
                          kNoAllocScratchBytes, stream);
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

// ---------------------------------------------------------------------------
// Context parallelism (decode): each rank holds a position range of every
// sequence; these calls make its partials and merge the ranks' partials.
hs2_status hs2_cp_attn_partial(const hs2_problem* p, const void* Q, const void* K, const void* V,
                               float* O_part, float* ml_part, void* workspace, size_t workspace_bytes,
                               void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->max_q_len > 1) return HS2_ERR_UNSUPPORTED;
  if (p->total_q == 0) return HS2_OK;  // no query rows
  if (!Q || !K || !V || !O_part || !ml_part) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O_part)) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  if ((s = check_ws(workspace, workspace_bytes, plan_decode(p, *dev, nullptr).bytes)) != HS2_OK) return s;
  return run_decode(p, *dev, Q, K, V, O_part, nullptr, 0, workspace, static_cast<cudaStream_t>(stream),
                    ml_part);
}

hs2_status hs2_cp_scores(const hs2_problem* p, const float* ml, float* scores, int64_t score_stride,
                         void* workspace, size_t workspace_bytes, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->max_q_len > 1) return HS2_ERR_UNSUPPORTED;
  if (p->total_q == 0) return HS2_OK;  // no query rows
  if (!ml || !scores || !aligned16(scores) || score_stride < std::max<int64_t>(1, p->max_kv_len))
    return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const DecodePlan pl = plan_decode(p, *dev, workspace);
  if ((s = check_ws(workspace, workspace_bytes, pl.bytes)) != HS2_OK) return s;
  DecodeArgs a{};
  a.qoff = p->q_offsets; a.kvoff = p->kv_offsets;
  a.B = p->B; a.Hq = p->Hq; a.Hkv = p->Hkv; a.G = p->Hq / p->Hkv; a.P = pl.P;
  a.total_q = p->total_q; a.total_kv = p->total_kv; a.scale = p->scale;
  a.logits = pl.logits; a.err = dev->err;
  a.Gp = logit_pitch(a.G);
  a.nw = p->dtype == HS2_BF16 ? 1 : kDecWarps;
  return launch_finalize(p, a, static_cast<float*>(nullptr), ml, scores, score_stride,
                         static_cast<cudaStream_t>(stream));
}

hs2_status hs2_cp_merge(int64_t rows, int32_t R, const float* O_parts, const float* ml_parts, int32_t dtype,
                        void* O, float* ml, void* stream) {
  if (rows < 0 || rows >= (int64_t(1) << 31) || R < 1 || !O_parts || !ml_parts || !O)
    return HS2_ERR_INVALID_ARG;
  if (dtype != HS2_BF16 && dtype != HS2_F32) return HS2_ERR_INVALID_ARG;
  if (rows == 0) return HS2_OK;
  DeviceInfo* dev;
  hs2_status s = device_info(&dev);
  if (s != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == HS2_BF16)
    launch(k_cp_merge<bf16>, dim3((unsigned)rows), dim3(kD), 0, st, 0, O_parts, ml_parts, (int)R, rows,
           static_cast<bf16*>(O), ml);
  else
    launch(k_cp_merge<float>, dim3((unsigned)rows), dim3(kD), 0, st, 0, O_parts, ml_parts, (int)R, rows,
           static_cast<float*>(O), ml);
  return launch_status();
}

hs2_status hs2_cp_topk_local(const hs2_problem* p, const float* scores, int64_t score_stride, int32_t k,
                             int32_t window, const int64_t* pos0, int32_t* idx_tmp, int32_t* count_tmp,
                             float* pair_score, int32_t* pair_pos, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->max_q_len > 1) return HS2_ERR_UNSUPPORTED;
  if (k < 1 || window < 0 || (int64_t)k + window >= (int64_t(1) << 30)) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no rows
  if (!scores || !pos0 || !idx_tmp || !count_tmp || !pair_score || !pair_pos) return HS2_ERR_INVALID_ARG;
  if (!aligned16(scores) || score_stride < std::max<int64_t>(1, p->max_kv_len)) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const int kk = k + window;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the local top-(k + window) over all of the rank's positions (no window of its own)
  if ((s = run_select(p, *dev, scores, score_stride, p->max_kv_len, kk, 0, 0, idx_tmp, kk, count_tmp, st)) !=
      HS2_OK)
    return s;
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;
  launch(k_cp_pack, dim3((unsigned)rows), dim3(128), 0, st, 0, scores, score_stride, idx_tmp, count_tmp, kk,
         p->q_offsets, p->kv_offsets, p->B, p->Hkv, pos0, pair_score, pair_pos, dev->err);
  return launch_status();
}

hs2_status hs2_cp_topk_merge(const hs2_problem* p, int32_t R, int32_t k, int32_t window, const float* pair_score,
                             const int32_t* pair_pos, int32_t* idx, int32_t* count, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->max_q_len > 1) return HS2_ERR_UNSUPPORTED;
  if (R < 1 || k < 1 || window < 0) return HS2_ERR_INVALID_ARG;
  if (k > kCpPickCap || (int64_t)R * (k + window) > kCpMergeCap) return HS2_ERR_UNSUPPORTED;
  const int64_t rows = p->total_q * p->Hkv;
  if (rows == 0) return HS2_OK;  // no rows
  if (!pair_score || !pair_pos || !idx || !count) return HS2_ERR_INVALID_ARG;
  if (rows >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  launch(k_cp_topk_merge, dim3((unsigned)rows), dim3(kCpMergeThreads), kCpMergeSmem,
         static_cast<cudaStream_t>(stream), 0, pair_score, pair_pos, (int)R, (int)(k + window), (int)k,
         (int)window, p->q_offsets, p->kv_offsets, p->B, p->Hkv, rows, idx, (int)(k + window), count);
  return launch_status();
}

hs2_status hs2_cp_sparse_partial(const hs2_problem* p, const void* Q_l, const void* K, const void* V,
                                 const int32_t* idx, const int32_t* count, int32_t idx_stride,
                                 const int64_t* pos0, float* O_part, float* ml_part, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->max_q_len > 1) return HS2_ERR_UNSUPPORTED;
  if (idx_stride < 1) return HS2_ERR_INVALID_ARG;
  if (p->total_q == 0) return HS2_OK;  // no query rows
  if (!Q_l || !K || !V || !idx || !count || !pos0 || !O_part || !ml_part) return HS2_ERR_INVALID_ARG;
  if (!aligned16(Q_l) || !aligned16(K) || !aligned16(V) || !aligned16(O_part)) return HS2_ERR_INVALID_ARG;
  const SparseShard sh{pos0, ml_part};
  return run_sparse(p, Q_l, K, V, idx, count, idx_stride, 0, O_part, stream, &sh);
}

hs2_status hs2_wait_selftest(int32_t mode, int64_t limit_cycles, void* stream) {
  if (mode != 0 && mode != 1) return HS2_ERR_INVALID_ARG;
  if (limit_cycles < 0) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  hs2_status s = device_info(&dev);
  if (s != HS2_OK) return s;
  const long long limit = limit_cycles < kWaitLimitCycles ? (long long)limit_cycles : kWaitLimitCycles;
  launch(k_wait_selftest, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), 0, (int)mode, limit,
         dev->err);
  return launch_status();
}

hs2_status hs2_kv_append(const hs2_problem* p, const void* K_new, const void* V_new, void* K,
                         void* V, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->total_q == 0) return HS2_OK;
  if (!K_new || !V_new || !K || !V) return HS2_ERR_INVALID_ARG;
  if (!aligned16(K_new) || !aligned16(V_new) || !aligned16(K) || !aligned16(V)) return HS2_ERR_INVALID_ARG;
  if (p->total_q > p->total_kv) return HS2_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const int64_t warps = p->total_q * p->Hkv;
  const unsigned grid = (unsigned)((warps * 32 + kAppendThreads - 1) / kAppendThreads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* kn = static_cast<const uint8_t*>(K_new);
  const uint8_t* vn = static_cast<const uint8_t*>(V_new);
  uint8_t* k = static_cast<uint8_t*>(K);
  uint8_t* v = static_cast<uint8_t*>(V);
  if (p->dtype == HS2_BF16)
    launch(k_kv_append<kD * 2>, dim3(grid), dim3(kAppendThreads), 0, st, 0, kn, vn, k, v, p->q_offsets,
           p->kv_offsets, p->B, p->Hkv, p->total_q, p->total_kv, dev->err);
  else
    launch(k_kv_append<kD * 4>, dim3(grid), dim3(kAppendThreads), 0, st, 0, kn, vn, k, v, p->q_offsets,
           p->kv_offsets, p->B, p->Hkv, p->total_q, p->total_kv, dev->err);
  return launch_status();
}

hs2_status hs2_kv_bridge(const hs2_problem* p, const void* H, int32_t hidden, const void* Wk_t,
                         const void* Wv_t, void* K, void* V, void* stream) {
  hs2_status s = check_problem(p);
  if (s != HS2_OK) return s;
  if (p->dtype != HS2_BF16) return HS2_ERR_UNSUPPORTED;
  if (!H || !Wk_t || !Wv_t || !K || !V || hidden < kBrKC || hidden % kBrKC != 0) return HS2_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(Wk_t) || !aligned16(Wv_t) || !aligned16(K) || !aligned16(V))
    return HS2_ERR_INVALID_ARG;
  if (p->total_kv == 0) return HS2_OK;
  const int64_t mtiles = (p->total_kv + kBrRows - 1) / kBrRows;
  if (mtiles > 65535) return HS2_ERR_UNSUPPORTED;
  DeviceInfo* dev;
  if ((s = device_info(&dev)) != HS2_OK) return s;
  const int ncols = p->Hkv * kD;
  const int NT = ncols % 256 == 0 ? 256 : 128;
  CUtensorMap mh, mk, mv;
  if (encode_map2(&mh, H, p->total_kv, hidden, kBrRows) != HS2_OK ||
      encode_map2(&mk, Wk_t, ncols, hidden, NT) != HS2_OK ||
      encode_map2(&mv, Wv_t, ncols, hidden, NT) != HS2_OK)
    return HS2_ERR_CUDA;
  BridgeArgs a{};
  a.rows = p->total_kv; a.hidden = hidden; a.ncols = ncols;
  a.K = static_cast<bf16*>(K); a.V = static_cast<bf16*>(V); a.err = dev->err;
  const dim3 grid((unsigned)(2 * ncols / NT), (unsigned)mtiles);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (NT == 256)
    launch(k_kv_bridge<256>, grid, dim3(kBrThreads), bridge_smem<256>(), st, 0, mh, mk, mv, a);
  else
    launch(k_kv_bridge<128>, grid, dim3(kBrThreads), bridge_smem<128>(), st, 0, mh, mk, mv, a);
  return launch_status();
}

int32_t hs2_version(void) { return (0 << 16) | 1; }

}  // extern "C"
