// C ABI of the approximate-attention prefill layer (declared in include/spava.h).
// One translation unit: it owns the device error word and every kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <memory>
#include <mutex>
#include <vector>

#include "../../include/spava.h"
#include "attention.cuh"
#include "compress.cuh"
#include "compress_fused.cuh"
#include "merge.cuh"
#include "plan.hpp"
#include "ptx.cuh"

using namespace spava;

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// Tensor map over a [rows, heads, d] bf16 tensor; box = 128 rows x 1 head x
// 64 elements (one 128-byte swizzled slab).  Rows past the end read as zero.
bool make_tmap(CUtensorMap* m, const void* base, int d, int heads, int64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows < 1) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(heads) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kBM)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

spava_status_t last_launch() {
  return cudaGetLastError() == cudaSuccess ? SPAVA_OK : SPAVA_ERR_CUDA;
}

// ----------------------------------------------------------------- stages
spava_status_t run_score(const Plan& P, const void* Q, const void* K, float* qsum, float* scores,
                         cudaStream_t st) {
  if (!Q || !K || !qsum || !scores || !aligned16(Q) || !aligned16(K)) return SPAVA_ERR_INVALID_ARG;
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  dim3 qgrid(kQsumSplit, P.Hkv);
  if (P.d == 128)
    qsum_kernel<128><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  else
    qsum_kernel<64><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  if (last_launch() != SPAVA_OK) return SPAVA_ERR_CUDA;
  const size_t smem = sizeof(float) * P.Hkv * P.d;
  const int64_t chunks = P.score_cols * P.Hkv * (P.d / 8);
  int64_t blocks = (chunks + kScoreThreads * kScoreUnroll - 1) / (kScoreThreads * kScoreUnroll);
  blocks = std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(sm_count()) * 8));
  if (P.d == 128) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    score_kernel<128><<<static_cast<unsigned>(blocks), kScoreThreads, smem, st>>>(k, qsum, scores, P.la,
                                                                                  P.score_cols, P.Hkv);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    score_kernel<64><<<static_cast<unsigned>(blocks), kScoreThreads, smem, st>>>(k, qsum, scores, P.la,
                                                                                 P.score_cols, P.Hkv);
  }
  return last_launch();
}

spava_status_t run_topk(const Plan& P, const float* scores, int32_t* idx, cudaStream_t st) {
  if (P.lp == 0) return SPAVA_OK;
  if (!scores || !idx) return SPAVA_ERR_INVALID_ARG;
  TopkParams tp;
  std::memset(&tp, 0, sizeof(tp));
  for (int h = 0; h < P.V - 1; ++h) {
    tp.start[h] = P.start[h] - P.la;
    tp.L[h] = P.L[h];
    tp.k[h] = P.lpe[h];
  }
  tp.Hkv = P.Hkv;
  tp.lp = P.lp;
  tp.score_cols = P.score_cols;
  topk_kernel<<<(P.V - 1) * P.Hkv, kTopkThreads, 0, st>>>(scores, idx, tp);
  return last_launch();
}

spava_status_t run_gather(const Plan& P, const void* K, const void* V, const int32_t* idx, void* Kp,
                          void* Vp, cudaStream_t st) {
  if (P.passing_rows == 0) return SPAVA_OK;
  if (!K || !V || !idx || !Kp || !Vp) return SPAVA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Kp) || !aligned16(Vp)) return SPAVA_ERR_INVALID_ARG;
  GatherParams gp;
  std::memset(&gp, 0, sizeof(gp));
  for (int h = 0; h < P.V; ++h) {
    gp.start[h] = P.start[h];
    gp.L[h] = P.L[h];
  }
  for (int h = 0; h <= P.V; ++h) gp.poff[h] = P.poff[h];
  gp.nblocks = P.V - 1;
  gp.Hkv = P.Hkv;
  gp.lp = P.lp;
  gp.rows = P.passing_rows;
  const int64_t chunks = 2 * P.passing_rows * P.Hkv * (P.d / 8);
  int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((chunks + 255) / 256, static_cast<int64_t>(sm_count()) * 16));
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  const auto* v = static_cast<const __nv_bfloat16*>(V);
  auto* kp = static_cast<__nv_bfloat16*>(Kp);
  auto* vp = static_cast<__nv_bfloat16*>(Vp);
  if (P.d == 128)
    gather_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(k, v, idx, kp, vp, gp);
  else
    gather_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(k, v, idx, kp, vp, gp);
  return last_launch();
}

bool compress_fits(const Plan& P) {
  for (int h = 0; h < P.V - 1; ++h)
    if ((P.L[h] + kCompressCtas - 1) / kCompressCtas > kCompressMaxSlice) return false;
  return true;
}

// Steps 1-3 in one launch: one cluster of kCompressCtas CTAs per (block, KV head).
spava_status_t run_compress(const Plan& P, const void* Q, const void* K, const void* V, float* qsum,
                            float* scores, int32_t* idx, void* Kp, void* Vp, cudaStream_t st) {
  if (P.lp == 0) return SPAVA_OK;
  if (!Q || !K || !V || !qsum || !scores || !idx || !Kp || !Vp) return SPAVA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Kp) || !aligned16(Vp))
    return SPAVA_ERR_INVALID_ARG;
  if (!compress_fits(P)) return SPAVA_ERR_UNSUPPORTED;
  CompressParams cp;
  std::memset(&cp, 0, sizeof(cp));
  for (int h = 0; h < P.V; ++h) {
    cp.start[h] = P.start[h];
    cp.L[h] = P.L[h];
    cp.k[h] = P.lpe[h];
  }
  for (int h = 0; h <= P.V; ++h) cp.poff[h] = P.poff[h];
  cp.Hq = P.Hq;
  cp.Hkv = P.Hkv;
  cp.G = P.G;
  cp.lq = P.lq;
  cp.lp = P.lp;
  cp.qs = P.qs;
  cp.la = P.la;
  cp.score_cols = P.score_cols;
  cp.scale = P.scale;
  const dim3 grid(kCompressCtas, P.V - 1, P.Hkv);
  const int smem = 12 * kCompressMaxSlice;
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  const auto* v = static_cast<const __nv_bfloat16*>(V);
  auto* kp = static_cast<__nv_bfloat16*>(Kp);
  auto* vp = static_cast<__nv_bfloat16*>(Vp);
  if (P.d == 128) {
    if (cudaFuncSetAttribute(compress_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return SPAVA_ERR_CUDA;
    compress_kernel<128><<<grid, kCompressThreads, smem, st>>>(q, k, v, qsum, scores, idx, kp, vp, cp);
  } else {
    if (cudaFuncSetAttribute(compress_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return SPAVA_ERR_CUDA;
    compress_kernel<64><<<grid, kCompressThreads, smem, st>>>(q, k, v, qsum, scores, idx, kp, vp, cp);
  }
  return last_launch();
}

template <int D>
spava_status_t launch_attn(const AttnParams& prm, int grid, cudaStream_t st) {
  using C = AttnCfg<D>;
  if (cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return SPAVA_ERR_CUDA;
  // The kernel moves registers from warpgroup 0 to the softmax warpgroups
  // (setmaxnreg); refuse to launch unless the launch allocation covers that
  // split, since an uncovered increase would never be granted.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, attn_kernel<D>) != cudaSuccess) return SPAVA_ERR_CUDA;
  if (static_cast<long>(fa.numRegs) * C::kThreads < 128L * C::kRegsLow + 256L * C::kRegsHigh)
    return SPAVA_ERR_UNSUPPORTED;
  attn_kernel<D><<<grid, C::kThreads, C::kSmemBytes, st>>>(prm);
  return last_launch();
}

spava_status_t run_attn(const Plan& P, const void* Q, const void* K, const void* V, const void* Kp,
                        const void* Vp, void* O, float* lse, float* O_part, float* lse_part,
                        cudaStream_t st) {
  if (!Q || !K || !V || !O || !lse || !O_part || !lse_part) return SPAVA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(O_part))
    return SPAVA_ERR_INVALID_ARG;
  if (P.passing_rows > 0 && (!Kp || !Vp || !aligned16(Kp) || !aligned16(Vp))) return SPAVA_ERR_INVALID_ARG;
  std::vector<uint32_t> items;
  spava_status_t s = make_items(P, &items);
  if (s != SPAVA_OK) return s;
  auto prm = std::make_unique<AttnParams>();
  std::memset(prm.get(), 0, sizeof(AttnParams));
  if (!make_tmap(&prm->tm_q, Q, P.d, P.Hq, P.n) || !make_tmap(&prm->tm_k, K, P.d, P.Hkv, P.n) ||
      !make_tmap(&prm->tm_v, V, P.d, P.Hkv, P.n))
    return SPAVA_ERR_CUDA;
  if (P.passing_rows > 0) {
    if (!make_tmap(&prm->tm_kp, Kp, P.d, P.Hkv, P.passing_rows) ||
        !make_tmap(&prm->tm_vp, Vp, P.d, P.Hkv, P.passing_rows))
      return SPAVA_ERR_CUDA;
  } else {   // never read: no segment refers to the passing buffer
    prm->tm_kp = prm->tm_k;
    prm->tm_vp = prm->tm_v;
  }
  prm->O = static_cast<__nv_bfloat16*>(O);
  prm->lse = lse;
  prm->O_part = O_part;
  prm->lse_part = lse_part;
  prm->n = static_cast<int32_t>(P.n);
  prm->Hq = P.Hq;
  prm->G = P.G;
  prm->lq = P.lq;
  prm->qs = static_cast<int32_t>(P.qs);
  prm->scale_log2 = P.scale * 1.44269504088896340736f;
  prm->nregions = P.nregions;
  prm->nitems = static_cast<int32_t>(items.size());
  for (int r = 0; r < P.nregions; ++r) prm->regions[r] = P.regions[r];
  std::memcpy(prm->items, items.data(), items.size() * sizeof(uint32_t));
  const int64_t grid = static_cast<int64_t>(items.size()) * P.Hq;
  if (grid > 0x7FFFFFFF) return SPAVA_ERR_UNSUPPORTED;
  return P.d == 128 ? launch_attn<128>(*prm, static_cast<int>(grid), st)
                    : launch_attn<64>(*prm, static_cast<int>(grid), st);
}

spava_status_t run_merge(const Plan& P, const float* O_part, const float* lse_part, void* O, float* lse,
                         cudaStream_t st) {
  if (!O_part || !lse_part || !O || !lse || !aligned16(O_part) || !aligned16(O)) return SPAVA_ERR_INVALID_ARG;
  const int64_t total = static_cast<int64_t>(P.lq) * P.Hq * (P.d / 4);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, sm_count() * 8));
  auto* o = static_cast<__nv_bfloat16*>(O);
  if (P.d == 128)
    merge_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(O_part, lse_part, o, lse, P.V, P.lq, P.Hq,
                                                                    P.qs, P.n);
  else
    merge_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(O_part, lse_part, o, lse, P.V, P.lq, P.Hq,
                                                                   P.qs, P.n);
  return last_launch();
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

spava_status_t spava_problem_sizes(const spava_problem_t* prob, spava_sizes_t* out) {
  if (!out) return SPAVA_ERR_INVALID_ARG;
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  out->seq_len = P.n;
  out->query_start = P.qs;
  out->score_cols = P.score_cols;
  out->passing_rows = P.passing_rows;
  out->attn_pairs = P.pairs;
  out->attn_flops = 4.0 * P.d * P.Hq * static_cast<double>(P.pairs);
  out->attn_tiles = P.tiles;
  out->workspace_bytes = P.ws_total;
  return SPAVA_OK;
}

spava_status_t spava_workspace_size(const spava_problem_t* prob, size_t* bytes) {
  if (!bytes) return SPAVA_ERR_INVALID_ARG;
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  *bytes = P.ws_total;
  return SPAVA_OK;
}

spava_status_t spava_score(const spava_problem_t* prob, const void* Q, const void* K, float* qsum,
                           float* scores, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_score(P, Q, K, qsum, scores, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_select_topk(const spava_problem_t* prob, const float* scores, int32_t* idx,
                                 spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_topk(P, scores, idx, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_gather_passing(const spava_problem_t* prob, const void* K, const void* V,
                                    const int32_t* idx, void* Kp, void* Vp, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_gather(P, K, V, idx, Kp, Vp, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_compress(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                              float* qsum, float* scores, int32_t* idx, void* Kp, void* Vp,
                              spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_compress(P, Q, K, V, qsum, scores, idx, Kp, Vp, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_attn_fwd(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                              const void* Kp, const void* Vp, void* O, float* lse, float* O_part,
                              float* lse_part, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_lse_merge(const spava_problem_t* prob, const float* O_part, const float* lse_part,
                               void* O, float* lse, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_merge(P, O_part, lse_part, O, lse, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_layer_fwd(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                               void* O, float* lse, void* workspace, size_t ws_bytes,
                               spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (!Q || !K || !V || !O || !lse) return SPAVA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < P.ws_total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPAVA_ERR_WORKSPACE;
  auto* ws = static_cast<uint8_t*>(workspace);
  float* qsum = reinterpret_cast<float*>(ws + P.ws_qsum);
  float* scores = reinterpret_cast<float*>(ws + P.ws_scores);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + P.ws_idx);
  void* Kp = ws + P.ws_kp;
  void* Vp = ws + P.ws_vp;
  float* O_part = reinterpret_cast<float*>(ws + P.ws_opart);
  float* lse_part = reinterpret_cast<float*>(ws + P.ws_lsepart);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (P.lp > 0 && compress_fits(P)) {   // steps 1-3 in one launch
    if ((s = run_compress(P, Q, K, V, qsum, scores, idx, Kp, Vp, st)) != SPAVA_OK) return s;
  } else if (P.lp > 0) {   // with lp = 0 no later host receives anything: skip the compression
    if ((s = run_score(P, Q, K, qsum, scores, st)) != SPAVA_OK) return s;
    if ((s = run_topk(P, scores, idx, st)) != SPAVA_OK) return s;
    if ((s = run_gather(P, K, V, idx, Kp, Vp, st)) != SPAVA_OK) return s;
  }
  if ((s = run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, st)) != SPAVA_OK) return s;
  return run_merge(P, O_part, lse_part, O, lse, st);
}

spava_status_t spava_device_error(uint32_t* code) {
  if (!code) return SPAVA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return SPAVA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return SPAVA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return SPAVA_ERR_CUDA;
  *code = v;
  return SPAVA_OK;
}

const char* spava_status_string(spava_status_t status) {
  switch (status) {
    case SPAVA_OK: return "SPAVA_OK";
    case SPAVA_ERR_INVALID_ARG: return "SPAVA_ERR_INVALID_ARG";
    case SPAVA_ERR_UNSUPPORTED: return "SPAVA_ERR_UNSUPPORTED";
    case SPAVA_ERR_WORKSPACE: return "SPAVA_ERR_WORKSPACE";
    case SPAVA_ERR_CUDA: return "SPAVA_ERR_CUDA";
    case SPAVA_ERR_DEVICE: return "SPAVA_ERR_DEVICE";
  }
  return "SPAVA_ERR_UNKNOWN";
}

}  // extern "C"

// ======================================================= no-allocation entry
// A copy of the layer's sequencing whose intermediates live in a fixed
// device array of this library instead of a caller-provided workspace.
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB per device
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_static_scratch on the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current)
// and keeps it; later calls reuse it.
spava_status_t static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPAVA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxScratchDevices) return SPAVA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SPAVA_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return SPAVA_OK;
}

}  // namespace

extern "C" spava_status_t spava_layer_fwd_noalloc(const spava_problem_t* prob, const void* Q,
                                                  const void* K, const void* V, void* O, float* lse,
                                                  spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (P.ws_total > kStaticScratchBytes) return SPAVA_ERR_WORKSPACE;   // problem too large for it
  if (!Q || !K || !V || !O || !lse) return SPAVA_ERR_INVALID_ARG;
  void* base = nullptr;
  if ((s = static_scratch_address(&base)) != SPAVA_OK) return s;
  // Every byte the steps below read from the scratch is written earlier in
  // the same call, so nothing has to be cleared between calls.
  auto* ws = static_cast<uint8_t*>(base);
  float* qsum = reinterpret_cast<float*>(ws + P.ws_qsum);
  float* scores = reinterpret_cast<float*>(ws + P.ws_scores);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + P.ws_idx);
  void* Kp = ws + P.ws_kp;
  void* Vp = ws + P.ws_vp;
  float* O_part = reinterpret_cast<float*>(ws + P.ws_opart);
  float* lse_part = reinterpret_cast<float*>(ws + P.ws_lsepart);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (P.lp > 0 && compress_fits(P)) {
    if ((s = run_compress(P, Q, K, V, qsum, scores, idx, Kp, Vp, st)) != SPAVA_OK) return s;
  } else if (P.lp > 0) {
    if ((s = run_score(P, Q, K, qsum, scores, st)) != SPAVA_OK) return s;
    if ((s = run_topk(P, scores, idx, st)) != SPAVA_OK) return s;
    if ((s = run_gather(P, K, V, idx, Kp, Vp, st)) != SPAVA_OK) return s;
  }
  if ((s = run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, st)) != SPAVA_OK) return s;
  return run_merge(P, O_part, lse_part, O, lse, st);
}
