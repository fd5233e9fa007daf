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
#include "score_variants.cuh"
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

spava_status_t last_launch() {
  return cudaGetLastError() == cudaSuccess ? SPAVA_OK : SPAVA_ERR_CUDA;
}

// ------------------------------------------------------ once per device
// Kernel attributes (dynamic shared memory limits) and the register check of
// the attention kernels are set up the first time a device is used, not on
// every call.
constexpr int kMaxDevices = 64;

struct DeviceSetup {
  bool done = false;
  spava_status_t status = SPAVA_OK;
  int sm_count = 148;
  int smem_per_sm = 228 * 1024;      // shared memory of one SM
  int smem_optin = 227 * 1024;       // largest dynamic + static shared memory of one CTA
  int smem_reserved = 1024;          // shared memory the system reserves per CTA
  int compress_static[2] = {0, 0};   // static shared memory of compress_kernel<64>, <128>
  int select_static = 0;             // ... of its select-only form
  // cudaOccupancyMaxActiveClusters of the cluster kernels, by (kernel, nc, dynamic smem)
  struct ClusterFit { const void* fn; int nc, smem, clusters; };
  std::vector<ClusterFit> compress_fit;
};
std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

template <int D>
spava_status_t setup_attn() {
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
  return SPAVA_OK;
}

// The current device's setup (done on first use).  Returns its status.
spava_status_t device_setup(const DeviceSetup** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPAVA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SPAVA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  DeviceSetup& s = g_setup[dev];
  if (!s.done) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) s.sm_count = n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess && n > 0)
      s.smem_per_sm = n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && n > 0)
      s.smem_optin = n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrReservedSharedMemoryPerBlock, dev) == cudaSuccess && n >= 0)
      s.smem_reserved = n;
    spava_status_t st = setup_attn<128>();
    if (st == SPAVA_OK) st = setup_attn<64>();
    if (st == SPAVA_OK &&
        (cudaFuncSetAttribute(colsum_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ColsumCfg<128>::kSmemBytes) != cudaSuccess ||
         cudaFuncSetAttribute(colsum_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ColsumCfg<64>::kSmemBytes) != cudaSuccess))
      st = SPAVA_ERR_CUDA;
    // compress_kernel may ask for up to the whole per-CTA limit (a launch that
    // wants one CTA per SM pads its request)
    cudaFuncAttributes fa;
    if (st == SPAVA_OK && cudaFuncGetAttributes(&fa, compress_kernel<64>) == cudaSuccess)
      s.compress_static[0] = static_cast<int>(fa.sharedSizeBytes);
    if (st == SPAVA_OK && cudaFuncGetAttributes(&fa, compress_kernel<128>) == cudaSuccess)
      s.compress_static[1] = static_cast<int>(fa.sharedSizeBytes);
    if (st == SPAVA_OK && cudaFuncGetAttributes(&fa, compress_kernel<128, true>) == cudaSuccess)
      s.select_static = static_cast<int>(fa.sharedSizeBytes);
    if (st == SPAVA_OK &&
        (cudaFuncSetAttribute(compress_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              s.smem_optin - s.compress_static[0]) != cudaSuccess ||
         cudaFuncSetAttribute(compress_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              s.smem_optin - s.compress_static[1]) != cudaSuccess ||
         cudaFuncSetAttribute(compress_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              s.smem_optin - s.select_static) != cudaSuccess ||
         cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, s.smem_optin) !=
             cudaSuccess ||
         cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, s.smem_optin) !=
             cudaSuccess))
      st = SPAVA_ERR_CUDA;
    s.status = st;
    s.done = true;
  }
  *out = &s;
  return s.status;
}

int sm_count() {
  const DeviceSetup* s = nullptr;
  return device_setup(&s) == SPAVA_OK ? s->sm_count : 148;
}

// ------------------------------------------------------ attention launch cache
// The attention launch's parameter block holds the work list (every 128-row
// tile pair sorted by cost) and five tensor maps; both depend only on the
// problem and the input pointers.  A small cache keyed by them lets repeated
// calls on the same buffers (the common case for a layer run many times)
// skip the sort and the encoding.
struct AttnKey {
  int device;
  int tag;   // which regions: 0 the layer's, else the first pass of selector `tag`
  int32_t H, la, lq, lp, Hq, Hkv, d;
  float scale;
  uint64_t hmask;
  int32_t L[kMaxV];
  const void *Q, *K, *V, *Kp, *Vp;
  bool operator==(const AttnKey& o) const { return std::memcmp(this, &o, sizeof(AttnKey)) == 0; }
};

struct AttnEntry {
  AttnKey key;
  std::unique_ptr<AttnParams> prm;
  int grid = 0;
  uint64_t last_use = 0;
};

constexpr int kAttnCacheSize = 8;
std::mutex g_attn_mu;
AttnEntry g_attn_cache[kAttnCacheSize];
uint64_t g_attn_clock = 0;

AttnKey attn_key(const Plan& P, int dev, int tag, const void* Q, const void* K, const void* V,
                 const void* Kp, const void* Vp) {
  AttnKey k;
  std::memset(&k, 0, sizeof(k));   // padding included, for the byte-wise compare
  k.device = dev;
  k.tag = tag;
  k.H = P.H;
  k.la = P.la;
  k.lq = P.lq;
  k.lp = P.lp;
  k.Hq = P.Hq;
  k.Hkv = P.Hkv;
  k.d = P.d;
  k.scale = P.scale;
  k.hmask = P.hmask;
  for (int h = 0; h < P.V; ++h) k.L[h] = P.L[h];
  k.Q = Q;
  k.K = K;
  k.V = V;
  k.Kp = P.passing_rows > 0 ? Kp : nullptr;
  k.Vp = P.passing_rows > 0 ? Vp : nullptr;
  return k;
}

// Build the input-dependent part of the attention launch (work list, tensor
// maps, regions).  Output pointers are filled in per call.
spava_status_t build_attn(const Plan& P, const void* Q, const void* K, const void* V, const void* Kp,
                          const void* Vp, AttnParams* prm, int* grid) {
  std::vector<uint32_t> items;
  spava_status_t s = make_items(P, &items);
  if (s != SPAVA_OK) return s;
  const int64_t g = static_cast<int64_t>(items.size()) * P.Hq;
  if (g > 0x7FFFFFFF) return SPAVA_ERR_UNSUPPORTED;
  std::memset(prm, 0, sizeof(AttnParams));
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
  prm->n = static_cast<int32_t>(P.n);
  prm->Hq = P.Hq;
  prm->G = P.G;
  prm->lq = P.lq;
  prm->qs = static_cast<int32_t>(P.qs);
  prm->V = P.V;
  prm->scale_log2 = P.scale * 1.44269504088896340736f;
  prm->nregions = P.nregions;
  prm->nitems = static_cast<int32_t>(items.size());
  for (int r = 0; r < P.nregions; ++r) prm->regions[r] = P.regions[r];
  std::memcpy(prm->items, items.data(), items.size() * sizeof(uint32_t));
  *grid = static_cast<int>(g);
  return SPAVA_OK;
}

// The cached parameter block for these inputs, built on a miss.  The caller
// holds g_attn_mu while it uses the returned entry.
spava_status_t attn_entry(const Plan& P, int tag, const void* Q, const void* K, const void* V,
                          const void* Kp, const void* Vp, AttnEntry** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPAVA_ERR_CUDA;
  const AttnKey key = attn_key(P, dev, tag, Q, K, V, Kp, Vp);
  AttnEntry* victim = &g_attn_cache[0];
  for (AttnEntry& e : g_attn_cache) {
    if (e.prm && e.key == key) {
      e.last_use = ++g_attn_clock;
      *out = &e;
      return SPAVA_OK;
    }
    if (!e.prm || e.last_use < victim->last_use) victim = &e;
  }
  if (!victim->prm) victim->prm = std::make_unique<AttnParams>();
  victim->last_use = 0;
  victim->key = AttnKey{};   // invalid until the build succeeds
  spava_status_t s = build_attn(P, Q, K, V, Kp, Vp, victim->prm.get(), &victim->grid);
  if (s != SPAVA_OK) {
    victim->prm.reset();
    return s;
  }
  victim->key = key;
  victim->last_use = ++g_attn_clock;
  *out = victim;
  return SPAVA_OK;
}

}  // namespace

namespace {

// ----------------------------------------------------------------- stages
int cluster_fit(const DeviceSetup* ds, const void* fn, int nc, int smem);
bool compress_params(const Plan& P, CompressParams* cp);

spava_status_t run_score(const Plan& P, const void* Q, const void* K, float* qsum, float* scores,
                         cudaStream_t st) {
  if (!Q || !K || !qsum || !scores || !aligned16(Q) || !aligned16(K)) return SPAVA_ERR_INVALID_ARG;
  const DeviceSetup* ds = nullptr;
  spava_status_t s = device_setup(&ds);
  if (s != SPAVA_OK) return s;
  const int smem = score_smem_bytes(P.Hkv, P.d);   // the ring + the query sums of every KV head
  if (smem > ds->smem_optin) return SPAVA_ERR_UNSUPPORTED;
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  dim3 qgrid(kQsumSplit, P.Hkv);
  if (P.d == 128)
    qsum_kernel<128><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  else
    qsum_kernel<64><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  if (last_launch() != SPAVA_OK) return SPAVA_ERR_CUDA;
  const int64_t items = (P.score_cols * P.Hkv * (P.d / 8) + kScoreThreads - 1) / kScoreThreads;
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(items, static_cast<int64_t>(ds->sm_count) * 2));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kScoreThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int64_t key0 = P.la, nkeys = P.score_cols;
  const int hkv = P.Hkv;
  const cudaError_t e = P.d == 128
                            ? cudaLaunchKernelEx(&cfg, score_kernel<128>, k, static_cast<const float*>(qsum), scores,
                                                 key0, nkeys, hkv)
                            : cudaLaunchKernelEx(&cfg, score_kernel<64>, k, static_cast<const float*>(qsum), scores,
                                                 key0, nkeys, hkv);
  if (e != cudaSuccess) return SPAVA_ERR_CUDA;
  return last_launch();
}

// Top-lp of every compressed block.  The cluster select of the fused
// compression (compress_kernel's select-only form: each CTA holds one slice
// of the block's scores) when a slice fits in shared memory; else one CTA per
// (block, KV head) reading the scores from global memory (topk_kernel).
spava_status_t run_topk(const Plan& P, const float* scores, int32_t* idx, cudaStream_t st) {
  if (P.lp == 0) return SPAVA_OK;
  if (!scores || !idx) return SPAVA_ERR_INVALID_ARG;
  const DeviceSetup* ds = nullptr;
  spava_status_t s = device_setup(&ds);
  if (s != SPAVA_OK) return s;
  CompressParams cp;
  if (!compress_params(P, &cp)) return SPAVA_OK;
  const void* fn = reinterpret_cast<const void*>(compress_kernel<128, true>);
  const int pairs = P.ncblk * P.Hkv;
  int nc = 0;
  for (int c = kCompressMaxCtas; c >= kCompressMinCtas; c /= 2) {   // the first that fits one wave
    const int b = select_smem_bytes(cp.lmax, c);
    if (b + ds->select_static <= ds->smem_optin && cluster_fit(ds, fn, c, b) >= pairs) {
      nc = c;
      break;
    }
  }
  if (nc == 0 && select_smem_bytes(cp.lmax, kCompressMaxCtas) + ds->select_static <= ds->smem_optin)
    nc = kCompressMaxCtas;   // more than one wave
  if (nc > 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(nc);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(nc), static_cast<unsigned>(P.ncblk), static_cast<unsigned>(P.Hkv));
    cfg.blockDim = dim3(kCompressThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(select_smem_bytes(cp.lmax, nc));
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __nv_bfloat16* none = nullptr;
    __nv_bfloat16* none_w = nullptr;
    const float* no_qsum = nullptr;
    if (cudaLaunchKernelEx(&cfg, compress_kernel<128, true>, none, none, no_qsum, const_cast<float*>(scores), idx,
                           none_w, none_w, cp) != cudaSuccess)
      return SPAVA_ERR_CUDA;
    return last_launch();
  }
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

// Clusters of nc CTAs of the cluster kernel `fn` (compress_kernel in either
// form) with `smem` dynamic bytes that can be resident at once (0 when the
// query fails); cached per device.
int cluster_fit(const DeviceSetup* ds, const void* fn, int nc, int smem) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  auto& fit = const_cast<DeviceSetup*>(ds)->compress_fit;
  for (const auto& f : fit)
    if (f.fn == fn && f.nc == nc && f.smem == smem) return f.clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(nc);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(nc), 1, 1);
  cfg.blockDim = dim3(kCompressThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();   // a failed query is not a launch error
    n = 0;
  }
  if (fit.size() >= 256) fit.clear();   // the key includes the block length: bound the cache
  fit.push_back({fn, nc, smem, n});
  return n;
}

// The launch parameters of the cluster kernels for the blocks the plan
// compresses (all h < V-1, or a host mask's); false when there are none.
bool compress_params(const Plan& P, CompressParams* cp) {
  std::memset(cp, 0, sizeof(*cp));
  for (int h = 0; h < P.V; ++h) {
    cp->start[h] = P.start[h];
    cp->L[h] = P.L[h];
    cp->k[h] = P.lpe[h];
  }
  for (int h = 0; h <= P.V; ++h) cp->poff[h] = P.poff[h];
  cp->Hkv = P.Hkv;
  cp->lp = P.lp;
  cp->la = P.la;
  cp->score_cols = P.score_cols;
  for (int i = 0; i < P.ncblk; ++i) {
    cp->blk[i] = P.cblk[i];
    cp->lmax = std::max(cp->lmax, P.L[P.cblk[i]]);
  }
  return P.ncblk > 0;
}

bool compress_fits(const Plan& P) {
  for (int h = 0; h < P.V - 1; ++h)
    if (P.L[h] > kCompressMaxBlock) return false;
  return true;
}

// Steps 1-3 in two launches: the query-block sum (qsum_kernel, the same
// kernel as the scoring stage's), then one cluster of nc CTAs per (block, KV
// head), launched as the sum's programmatic dependent: it starts its K stream
// at once and waits for the sum before its first score.  merge_count (may be
// null): the following attention launch's merge counters, zeroed by the
// second launch.
//
// The launch shape is the first of: 8-CTA clusters with one CTA per SM,
// 4-CTA clusters with one CTA per SM, 8-CTA clusters packed two per SM, 4-CTA
// clusters packed, that fits the GPU in one wave (cudaOccupancyMaxActiveClusters,
// which knows how clusters fill the GPCs); 4-CTA clusters packed when none
// does.  One CTA per SM is forced by padding the shared-memory request: two
// CTAs on one SM share its load bandwidth and set the launch's span.
spava_status_t run_compress(const Plan& P, const void* Q, const void* K, const void* V, float* qsum,
                            float* scores, int32_t* idx, void* Kp, void* Vp, int32_t* merge_count,
                            cudaStream_t st) {
  if (P.lp == 0) return SPAVA_OK;
  if (!Q || !K || !V || !qsum || !scores || !idx || !Kp || !Vp) return SPAVA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Kp) || !aligned16(Vp))
    return SPAVA_ERR_INVALID_ARG;
  if (!compress_fits(P)) return SPAVA_ERR_UNSUPPORTED;
  const DeviceSetup* ds = nullptr;
  spava_status_t s = device_setup(&ds);
  if (s != SPAVA_OK) return s;
  CompressParams cp;
  if (!compress_params(P, &cp)) return SPAVA_OK;   // a host mask that selects no compressed block
  cp.merge_count = merge_count;
  cp.n_merge = merge_count ? P.n_merge : 0;
  const int pairs = P.ncblk * P.Hkv;
  const int stat = ds->compress_static[P.d == 128 ? 1 : 0];
  // dynamic bytes above which two CTAs (dynamic + static + what the system
  // reserves per CTA) no longer fit one SM
  const int spread = (ds->smem_per_sm / 2 - stat - ds->smem_reserved + 16) / 16 * 16;
  int nc = kCompressMinCtas, smem = compress_smem_bytes(cp.lmax, kCompressMinCtas);
  const struct { int nc; bool spread; } shapes[4] = {{8, true}, {4, true}, {8, false}, {4, false}};
  for (const auto& sh : shapes) {
    int b = compress_smem_bytes(cp.lmax, sh.nc);
    if (sh.spread) b = std::max(b, spread);
    if (b + stat > ds->smem_optin) continue;
    const void* fn = P.d == 128 ? reinterpret_cast<const void*>(compress_kernel<128>)
                                : reinterpret_cast<const void*>(compress_kernel<64>);
    if (cluster_fit(ds, fn, sh.nc, b) >= pairs) {
      nc = sh.nc;
      smem = b;
      break;
    }
  }
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  const auto* v = static_cast<const __nv_bfloat16*>(V);
  auto* kp = static_cast<__nv_bfloat16*>(Kp);
  auto* vp = static_cast<__nv_bfloat16*>(Vp);
  const dim3 qgrid(kQsumSplit, P.Hkv);
  if (P.d == 128)
    qsum_kernel<128><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  else
    qsum_kernel<64><<<qgrid, kQsumThreads, 0, st>>>(q, qsum, P.qs, P.lq, P.Hq, P.G, P.scale);
  if (last_launch() != SPAVA_OK) return SPAVA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(nc);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(nc), static_cast<unsigned>(P.ncblk), static_cast<unsigned>(P.Hkv));
  cfg.blockDim = dim3(kCompressThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = P.d == 128
                            ? cudaLaunchKernelEx(&cfg, compress_kernel<128>, k, v, qsum, scores, idx, kp, vp, cp)
                            : cudaLaunchKernelEx(&cfg, compress_kernel<64>, k, v, qsum, scores, idx, kp, vp, cp);
  if (e != cudaSuccess) return SPAVA_ERR_CUDA;
  return last_launch();
}

// Attention over every row kind in one launch.  merge_count non-null: the
// query partials are merged in the same launch (counters must be zero).
// dependent: launched as a programmatic dependent of the kernel just before
// it on the stream (the layer's compression), so that it can start while
// that kernel runs; it waits for it before reading the passing buffer or the
// counters.
spava_status_t run_attn(const Plan& P, const void* Q, const void* K, const void* V, const void* Kp,
                        const void* Vp, void* O, float* lse, float* O_part, float* lse_part,
                        int32_t* merge_count, bool dependent, cudaStream_t st, int tag = 0,
                        int skip_k_tile = -1, uint64_t wait_limit_ns = kWaitLimitNs) {
  if (!Q || !K || !V || !O || !lse || !O_part || !lse_part) return SPAVA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(O_part))
    return SPAVA_ERR_INVALID_ARG;
  if (P.passing_rows > 0 && (!Kp || !Vp || !aligned16(Kp) || !aligned16(Vp))) return SPAVA_ERR_INVALID_ARG;
  if (P.items > kMaxItems) return SPAVA_ERR_UNSUPPORTED;
  const DeviceSetup* ds = nullptr;
  spava_status_t s = device_setup(&ds);
  if (s != SPAVA_OK) return s;
  std::lock_guard<std::mutex> lock(g_attn_mu);
  AttnEntry* e = nullptr;
  if ((s = attn_entry(P, tag, Q, K, V, Kp, Vp, &e)) != SPAVA_OK) return s;
  AttnParams& prm = *e->prm;
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.lse = lse;
  prm.O_part = O_part;
  prm.lse_part = lse_part;
  prm.merge_count = merge_count;
  prm.pdl_wait = dependent ? 1 : 0;
  prm.skip_k_tile = skip_k_tile;
  prm.wait_limit_ns = wait_limit_ns;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(e->grid));
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  if (P.d == 128) {
    cfg.blockDim = dim3(AttnCfg<128>::kThreads);
    cfg.dynamicSmemBytes = AttnCfg<128>::kSmemBytes;
    if (cudaLaunchKernelEx(&cfg, attn_kernel<128>, prm) != cudaSuccess) return SPAVA_ERR_CUDA;
  } else {
    cfg.blockDim = dim3(AttnCfg<64>::kThreads);
    cfg.dynamicSmemBytes = AttnCfg<64>::kSmemBytes;
    if (cudaLaunchKernelEx(&cfg, attn_kernel<64>, prm) != cudaSuccess) return SPAVA_ERR_CUDA;
  }
  return last_launch();
}

spava_status_t run_merge(const Plan& P, const float* O_part, const float* lse_part, void* O, float* lse,
                         cudaStream_t st) {
  if (!O_part || !lse_part || !O || !lse || !aligned16(O_part) || !aligned16(O)) return SPAVA_ERR_INVALID_ARG;
  if (P.V > 32) return SPAVA_ERR_UNSUPPORTED;   // one lane per partial
  const int64_t pairs = static_cast<int64_t>(P.lq) * P.Hq;   // one warp per (row, head), 8 per block
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((pairs + 7) / 8, sm_count() * 16));
  auto* o = static_cast<__nv_bfloat16*>(O);
  if (P.d == 128)
    merge_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(O_part, lse_part, o, lse, P.V, P.lq, P.Hq,
                                                                    P.qs, P.n);
  else
    merge_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(O_part, lse_part, o, lse, P.V, P.lq, P.Hq,
                                                                   P.qs, P.n);
  return last_launch();
}

// Step 1 under a selector variant (P.score_kind != linear), two passes:
// the attention kernel on the variant's regions gives every scoring row's
// lse over the block (softmax: into the query-partial slots; context: into
// the workspace's row outputs), then colsum_kernel sums the probabilities
// per key.  `ws` is the layer's workspace.
spava_status_t run_score_variant(const Plan& P, const void* Q, const void* K, float* scores, uint8_t* ws,
                                 cudaStream_t st) {
  if (!Q || !K || !scores || !aligned16(Q) || !aligned16(K)) return SPAVA_ERR_INVALID_ARG;
  if (P.V < 2 || P.score_cols == 0) return SPAVA_OK;
  Plan PV = P;
  make_variant_regions(&PV);
  if (PV.items > kMaxItems) return SPAVA_ERR_UNSUPPORTED;
  const bool ctx = P.score_kind == kScoreContext;
  float* O_part = reinterpret_cast<float*>(ws + P.ws_opart);
  float* lse_part = reinterpret_cast<float*>(ws + P.ws_lsepart);
  void* vo = ctx ? static_cast<void*>(ws + P.ws_vo) : static_cast<void*>(O_part);
  float* vlse = ctx ? reinterpret_cast<float*>(ws + P.ws_vlse) : lse_part;
  spava_status_t s = run_attn(PV, Q, K, K, nullptr, nullptr, vo, vlse, O_part, lse_part, nullptr, false, st,
                              P.score_kind);
  if (s != SPAVA_OK) return s;
  auto prm = std::make_unique<ColsumParams>();
  std::memset(prm.get(), 0, sizeof(ColsumParams));
  if (!make_tmap(&prm->tm_q, Q, P.d, P.Hq, P.n) || !make_tmap(&prm->tm_k, K, P.d, P.Hkv, P.n)) return SPAVA_ERR_CUDA;
  prm->scores = scores;
  prm->lse = ctx ? vlse : lse_part;
  prm->kind = P.score_kind;
  prm->Hq = P.Hq;
  prm->G = P.G;
  prm->lq = P.lq;
  prm->qs = static_cast<int32_t>(P.qs);
  prm->n = static_cast<int32_t>(P.n);
  prm->la = P.la;
  prm->V = P.V;
  prm->score_cols = P.score_cols;
  prm->scale_log2 = P.scale * 1.44269504088896340736f;
  prm->nblocks = P.V - 1;
  int tiles = 0;
  for (int h = 0; h < P.V - 1; ++h) {
    prm->start[h] = P.start[h];
    prm->L[h] = P.L[h];
    prm->tile0[h] = tiles;
    tiles += (P.L[h] + 127) / 128;
  }
  prm->tile0[P.V - 1] = tiles;
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(P.Hkv));
  if (P.d == 128)
    colsum_kernel<128><<<grid, ColsumCfg<128>::kThreads, ColsumCfg<128>::kSmemBytes, st>>>(*prm);
  else
    colsum_kernel<64><<<grid, ColsumCfg<64>::kThreads, ColsumCfg<64>::kSmemBytes, st>>>(*prm);
  return last_launch();
}

// The whole layer with its intermediates carved from `ws` (P.ws_total bytes,
// 256-byte aligned): compression (qsum + one cluster launch, or the stage kernels for
// blocks too long for it), then attention with the query-partial merge in
// the same launch, started as a programmatic dependent of the compression.
// The work list is built (and checked) before anything is launched.
spava_status_t run_layer(const Plan& P, uint8_t* ws, const void* Q, const void* K, const void* V, void* O,
                         float* lse, cudaStream_t st) {
  float* qsum = reinterpret_cast<float*>(ws + P.ws_qsum);
  float* scores = reinterpret_cast<float*>(ws + P.ws_scores);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + P.ws_idx);
  void* Kp = ws + P.ws_kp;
  void* Vp = ws + P.ws_vp;
  float* O_part = reinterpret_cast<float*>(ws + P.ws_opart);
  float* lse_part = reinterpret_cast<float*>(ws + P.ws_lsepart);
  int32_t* count = reinterpret_cast<int32_t*>(ws + P.ws_count);
  spava_status_t s;
  if (P.items > kMaxItems) return SPAVA_ERR_UNSUPPORTED;   // before any CUDA call
  {   // validate the attention launch first (work list, tensor maps)
    const DeviceSetup* ds = nullptr;
    if ((s = device_setup(&ds)) != SPAVA_OK) return s;
    std::lock_guard<std::mutex> lock(g_attn_mu);
    AttnEntry* e = nullptr;
    if ((s = attn_entry(P, 0, Q, K, V, Kp, Vp, &e)) != SPAVA_OK) return s;
  }
  bool dependent = false;
  if (P.lp > 0 && P.score_kind != kScoreLinear) {   // a selector variant: two scoring passes, top-lp, gather
    if ((s = run_score_variant(P, Q, K, scores, ws, st)) != SPAVA_OK) return s;
    if ((s = run_topk(P, scores, idx, st)) != SPAVA_OK) return s;
    if ((s = run_gather(P, K, V, idx, Kp, Vp, st)) != SPAVA_OK) return s;
    if (cudaMemsetAsync(count, 0, sizeof(int32_t) * static_cast<size_t>(P.n_merge), st) != cudaSuccess)
      return SPAVA_ERR_CUDA;
  } else if (P.lp > 0 && compress_fits(P)) {   // steps 1-3 in two launches; the second zeroes the merge counters
    if ((s = run_compress(P, Q, K, V, qsum, scores, idx, Kp, Vp, count, st)) != SPAVA_OK) return s;
    dependent = true;
  } else {
    if (P.lp > 0) {   // with lp = 0 no later host receives anything: no compression
      if ((s = run_score(P, Q, K, qsum, scores, st)) != SPAVA_OK) return s;
      if ((s = run_topk(P, scores, idx, st)) != SPAVA_OK) return s;
      if ((s = run_gather(P, K, V, idx, Kp, Vp, st)) != SPAVA_OK) return s;
    }
    if (cudaMemsetAsync(count, 0, sizeof(int32_t) * static_cast<size_t>(P.n_merge), st) != cudaSuccess)
      return SPAVA_ERR_CUDA;
  }
  return run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, count, dependent, st);
}

}  // namespace


namespace {

// Test hook: one thread waits on an mbarrier that nothing will complete, with
// the kernels' own bounded waits and a short limit.  out[0] = what mbar_wait
// returned, out[1] = the abort flag it left, out[2] = what mbar_wait_drain
// returned, out[3] = nanoseconds the two waits took.
__global__ void wait_timeout_kernel(int64_t* out, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  fence_barrier_init();
  const uint64_t t0 = globaltimer_ns();
  const bool w = mbar_wait(b, 0, &abort_flag, limit_ns);
  const bool d = mbar_wait_drain(b, 0, limit_ns);
  out[0] = w;
  out[1] = abort_flag;
  out[2] = d;
  out[3] = static_cast<int64_t>(globaltimer_ns() - t0);
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
  if (P.score_kind != kScoreLinear) return SPAVA_ERR_UNSUPPORTED;   // spava_score_variant
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;
  return run_score(P, Q, K, qsum, scores, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_score_variant(const spava_problem_t* prob, const void* Q, const void* K, float* scores,
                                   void* workspace, size_t ws_bytes, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;
  if (P.score_kind == kScoreLinear) {   // the pages' selector needs no workspace
    if (!workspace || ws_bytes < P.ws_total) return SPAVA_ERR_WORKSPACE;
    float* qsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + P.ws_qsum);
    return run_score(P, Q, K, qsum, scores, reinterpret_cast<cudaStream_t>(stream));
  }
  if (!workspace || ws_bytes < P.ws_total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPAVA_ERR_WORKSPACE;
  return run_score_variant(P, Q, K, scores, static_cast<uint8_t*>(workspace),
                           reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_select_topk(const spava_problem_t* prob, const float* scores, int32_t* idx,
                                 spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;
  return run_topk(P, scores, idx, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_gather_passing(const spava_problem_t* prob, const void* K, const void* V,
                                    const int32_t* idx, void* Kp, void* Vp, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;
  return run_gather(P, K, V, idx, Kp, Vp, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_compress(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                              float* qsum, float* scores, int32_t* idx, void* Kp, void* Vp,
                              spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_compress(P, Q, K, V, qsum, scores, idx, Kp, Vp, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

spava_status_t spava_attn_fwd(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                              const void* Kp, const void* Vp, void* O, float* lse, float* O_part,
                              float* lse_part, spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  return run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, nullptr, false,
                  reinterpret_cast<cudaStream_t>(stream));
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
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;   // needs the other hosts' passing rows
  if (!Q || !K || !V || !O || !lse) return SPAVA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < P.ws_total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SPAVA_ERR_WORKSPACE;
  return run_layer(P, static_cast<uint8_t*>(workspace), Q, K, V, O, lse, reinterpret_cast<cudaStream_t>(stream));
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

spava_status_t spava_debug_attn_abort(const spava_problem_t* prob, const void* Q, const void* K, const void* V,
                                      const void* Kp, const void* Vp, void* O, float* lse, float* O_part,
                                      float* lse_part, int32_t skip_k_tile, uint64_t limit_ns,
                                      spava_stream_t stream) {
  Plan P;
  spava_status_t s = make_plan(prob, &P);
  if (s != SPAVA_OK) return s;
  if (skip_k_tile < 0 || limit_ns == 0 || limit_ns > kWaitLimitNs) return SPAVA_ERR_INVALID_ARG;
  return run_attn(P, Q, K, V, Kp, Vp, O, lse, O_part, lse_part, nullptr, false,
                  reinterpret_cast<cudaStream_t>(stream), 0, skip_k_tile, limit_ns);
}

spava_status_t spava_debug_wait_timeout(int64_t* out, uint64_t limit_ns, spava_stream_t stream) {
  if (!out || limit_ns == 0 || limit_ns > kWaitLimitNs) return SPAVA_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(out, limit_ns);
  return last_launch();
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
// The layer with its intermediates in a fixed device array of this library
// instead of a caller-provided workspace (same sequencing: run_layer).
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;   // 64 MiB per device
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current)
// and keeps it; later calls reuse it.
spava_status_t static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPAVA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SPAVA_ERR_UNSUPPORTED;
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
  if (P.partial) return SPAVA_ERR_UNSUPPORTED;
  if (P.ws_total > kStaticScratchBytes) return SPAVA_ERR_WORKSPACE;   // problem too large for it
  if (!Q || !K || !V || !O || !lse) return SPAVA_ERR_INVALID_ARG;
  void* base = nullptr;
  if ((s = static_scratch_address(&base)) != SPAVA_OK) return s;
  // Every byte the layer reads from the scratch is written earlier in the
  // same call (the merge counters are zeroed by the call itself), so nothing
  // has to be cleared between calls.
  return run_layer(P, static_cast<uint8_t*>(base), Q, K, V, O, lse, reinterpret_cast<cudaStream_t>(stream));
}
