// bitlinear_api.cu -- the C ABI declared in include/bitlinear.h: argument
// checks, path selection, TMA descriptor encoding and kernel launches.  One
// translation unit holds every kernel so the device status word is a plain
// __device__ variable.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/bitlinear.h"
#include "gemm_skinny.cuh"
#include "gemm_tc2.cuh"

namespace bl {

__device__ int32_t g_device_status;

namespace {

// The kernel variant of the last successful call on this thread; assigning it
// also logs the name to stderr when BITLINEAR_LOG is set (read once).
bool log_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("BITLINEAR_LOG");
    return v != nullptr && v[0] != '\0' && std::strcmp(v, "0") != 0;
  }();
  return on;
}

struct LastKernel {
  const char* name = "";
  LastKernel& operator=(const char* n) {
    name = n;
    if (log_enabled()) std::fprintf(stderr, "bitlinear: %s\n", n);
    return *this;
  }
};

thread_local LastKernel t_last_kernel;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  int32_t* status = nullptr;
  int sk_clusters[kSkMaxCluster + 1] = {};  // clusters of each size the few-token kernel fits at once (0: not asked)
  int t2_pairs[3][4] = {};  // CTA pairs of the pair GEMM resident at once ([dense, 2:4, n:8][BN 128 .. 224]; 0: not asked)
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

bitlinear_status current_device(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BITLINEAR_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    if (d.supported) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return BITLINEAR_ERR_CUDA;
      d.status = static_cast<int32_t*>(p);
    }
    d.probed = true;
  }
  if (!d.supported) return BITLINEAR_ERR_DEVICE;
  *out = &d;
  return BITLINEAR_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A tensor map depends only on the address, extents, stride, box and swizzle
// it was encoded from, so encoded maps are kept per host thread (a small
// round-robin table) and reused by later calls with the same key: repeated
// calls on the same weights and buffers skip the driver's encoding.
struct MapKey {
  const void* base;
  uint64_t inner, outer, stride;
  uint32_t box_inner, box_outer, swizzle;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && outer == o.outer && stride == o.stride &&
           box_inner == o.box_inner && box_outer == o.box_outer && swizzle == o.swizzle;
  }
};

constexpr int kMapCache = 256;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  bool used[kMapCache] = {};
  int next = 0;
};
thread_local MapCache t_maps;

// 2-D uint8 tensor map: inner extent `inner` bytes, `outer` rows of `stride`
// bytes, box {box_inner, box_outer}; out-of-range elements read as zero.
// swizzle: 0 (none), 32, 64 or 128 (the shared-memory swizzle of the landed box, in bytes).
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t stride,
                 uint32_t box_inner, uint32_t box_outer, int swizzle) {
  const MapKey k{base, inner, outer, stride, box_inner, box_outer, static_cast<uint32_t>(swizzle)};
  MapCache& c = t_maps;
  for (int i = 0; i < kMapCache; ++i)
    if (c.used[i] && c.key[i] == k) {
      *map = c.map[i];
      return true;
    }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                  : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                  : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  c.key[c.next] = k;
  c.map[c.next] = *map;
  c.used[c.next] = true;
  c.next = (c.next + 1) % kMapCache;
  return true;
}

// Largest dynamic shared memory already granted to a kernel on a device
// (per host thread): the attribute is set only when a launch needs more.
struct SmemGrant {
  int dev;
  const void* fn;
  size_t bytes;
};
constexpr int kSmemGrants = 128;
thread_local SmemGrant t_grants[kSmemGrants];
thread_local int t_ngrants = 0;

bool ensure_smem(const void* fn, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  for (int i = 0; i < t_ngrants; ++i)
    if (t_grants[i].dev == dev && t_grants[i].fn == fn) {
      if (t_grants[i].bytes >= smem) return true;
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
          cudaSuccess)
        return false;
      t_grants[i].bytes = smem;
      return true;
    }
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return false;
  if (t_ngrants < kSmemGrants) t_grants[t_ngrants++] = SmemGrant{dev, fn, smem};
  return true;
}

template <typename Kern, typename... Args>
bitlinear_status launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, int cluster_x,
                           Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  // the 48 KB default covers static and dynamic shared memory together: opt in well below it
  if (smem > 32 * 1024 && !ensure_smem(reinterpret_cast<const void*>(kern), smem)) return BITLINEAR_ERR_CUDA;
  return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

template <typename Kern, typename... Args>
bitlinear_status launch(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, Args... args) {
  return launch_ex(kern, grid, block, smem, s, pdl, 1, args...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline int64_t dense_ld(int K) { return 16 * ((static_cast<int64_t>(K) + 63) / 64); }
inline int64_t k16(int K) { return (static_cast<int64_t>(K) + 15) / 16 * 16; }

bool pattern_ok(int n, int m) { return (n == 0 && m == 0) || (n == 2 && m == 4) || (m == 8 && n >= 1 && n <= 7); }

bitlinear_status check_nk(int N, int K) {
  if (N < 1 || N > BITLINEAR_MAX_N || K < 1 || K > BITLINEAR_MAX_K) return BITLINEAR_ERR_SHAPE;
  return BITLINEAR_OK;
}

// ---------------------------------------------------------------- tensor-core path
int pick_bn(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// Tiling of one tensor-core GEMM.  When the (weight-row tile, token tile)
// pairs leave SMs idle, each tile's K range is cut into ksplit slices (at
// least two k-blocks each, none empty) so that about one unit runs per SM.
struct TcPlan {
  int bn, row_tiles, tok_tiles, kblocks, ksplit, kbs;
};

TcPlan tc_plan(int M, int N, int K, int nm, int sm_count) {
  TcPlan p;
  p.bn = pick_bn(M);
  p.row_tiles = (N + kTcRows - 1) / kTcRows;
  // narrower token tiles while the tiles would fill fewer than half the SMs
  while (p.bn > 32 && p.row_tiles * ((M + p.bn - 1) / p.bn) < sm_count / 2) p.bn >>= 1;
  p.tok_tiles = (M + p.bn - 1) / p.bn;
  p.kblocks = (K + tc_bk(nm, p.bn) - 1) / tc_bk(nm, p.bn);
  const int tiles = p.row_tiles * p.tok_tiles;
  int ks = 1;
  if (tiles < sm_count) ks = std::max(1, std::min(std::min(sm_count / tiles, p.kblocks / 2), 16));
  p.kbs = (p.kblocks + ks - 1) / ks;
  p.ksplit = (p.kblocks + p.kbs - 1) / p.kbs;
  return p;
}

int plan_sm_count() {
  DeviceState* d = nullptr;
  return current_device(&d) == BITLINEAR_OK ? d->sm_count : 148;
}

// Workspace: codes [M, k16(K)] | gamma [M] | code sums [M] | (split only)
// arrival counters [sm_count] | fp32 sums [M][N].
size_t tc_base_bytes(int M, int K) {
  return align256(static_cast<size_t>(M) * k16(K)) + 2 * align256(4 * static_cast<size_t>(M));
}
size_t tc_cnt_bytes(int sm_count) { return align256(4 * static_cast<size_t>(sm_count)); }

// Workspace of bitlinear_forward_q8: only the split-K counters and sums (none without a split).
size_t tc_workspace_q8(int M, int N, int K, int nm, int sm_count) {
  const TcPlan p = tc_plan(M, N, K, nm, sm_count);
  return p.ksplit > 1 ? tc_cnt_bytes(sm_count) + align256(static_cast<size_t>(M) * N * 4) : 0;
}
bool workspace_ok_q8(const void* ws, size_t bytes, int M, int N, int K, int nm, int sm_count) {
  const size_t need = tc_workspace_q8(M, N, K, nm, sm_count);
  return need == 0 || (ws && bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 15u) == 0);
}

size_t tc_workspace(int M, int N, int K, int nm, int sm_count) {
  const TcPlan p = tc_plan(M, N, K, nm, sm_count);
  size_t b = tc_base_bytes(M, K);
  if (p.ksplit > 1) b += tc_cnt_bytes(sm_count) + align256(static_cast<size_t>(M) * N * 4);
  return b;
}

template <int BN, int NM>
bitlinear_status launch_tc_bn(const CUtensorMap& mB, const CUtensorMap& mA, const CUtensorMap& mMeta, TcArgs ta,
                              int sm_count, cudaStream_t s) {
  const size_t smem = tc_smem_bytes(BN, NM, ta.vbox);
  const int units = ta.row_tiles * ta.tok_tiles * ta.ksplit;
  const int grid = std::min(sm_count, units);
  return launch(tc_gemm_kernel<BN, NM>, dim3(grid), dim3(kTcThreads), smem, s, true, mB, mA, mMeta, ta);
}

template <int NM>
bitlinear_status launch_tc(int bn, const CUtensorMap& mB, const CUtensorMap& mA, const CUtensorMap& mMeta,
                           const TcArgs& ta, int sm_count, cudaStream_t s) {
  switch (bn) {
    case 16: return launch_tc_bn<16, NM>(mB, mA, mMeta, ta, sm_count, s);
    case 32: return launch_tc_bn<32, NM>(mB, mA, mMeta, ta, sm_count, s);
    case 64: return launch_tc_bn<64, NM>(mB, mA, mMeta, ta, sm_count, s);
    default: return launch_tc_bn<128, NM>(mB, mA, mMeta, ta, sm_count, s);
  }
}

// CTA pairs of the pair GEMM resident at once (one CTA per SM), asked once per device and variant.
template <int NM, int BN>
int t2_active_pairs(DeviceState* dev) {
  int& slot = dev->t2_pairs[NM == 0 ? 0 : NM == 3 ? 1 : 2][(BN - 128) / 32];
  std::lock_guard<std::mutex> lk(g_mu);
  if (slot == 0) {
    int n = -1;
    if (ensure_smem(reinterpret_cast<const void*>(tc2_gemm_kernel<NM, BN>), T2<NM, BN>::SMEM)) {
      cudaLaunchConfig_t cfg;
      std::memset(&cfg, 0, sizeof cfg);
      cfg.gridDim = dim3(2 * 64);
      cfg.blockDim = dim3(kTcThreads);
      cfg.dynamicSmemBytes = T2<NM, BN>::SMEM;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, tc2_gemm_kernel<NM, BN>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = -1;
      }
    }
    slot = n;
  }
  return slot;
}

const char* tc_name(int nm, int bn) {
  static const char* names[4][4] = {
      {"tc_gemm_dense_bn16", "tc_gemm_dense_bn32", "tc_gemm_dense_bn64", "tc_gemm_dense_bn128"},
      {"tc_gemm_nm24_bn16", "tc_gemm_nm24_bn32", "tc_gemm_nm24_bn64", "tc_gemm_nm24_bn128"},
      {"tc_gemm_n8_bn16", "tc_gemm_n8_bn32", "tc_gemm_n8_bn64", "tc_gemm_n8_bn128"},
      {"tc_gemm_sp24_bn16", "tc_gemm_sp24_bn32", "tc_gemm_sp24_bn64", "tc_gemm_sp24_bn128"}};
  const int i = bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : 3;
  return names[nm][i];
}

// ---------------------------------------------------------------- few-token path
// Plan of the fused few-token kernel (gemm_skinny.cuh): token tile BN, K
// slices per cluster and chunks per slice.  Not eligible (ok = false) for more
// than 64 tokens or a K too long for eight resident slices.
struct SkPlan {
  bool ok;
  int bn, cs, per, row_tiles, kchunks;
  size_t smem;
};

// Clusters of cs CTAs of the few-token kernel resident at once on the device
// (one CTA per SM), asked once per device and size.
int sk_active_clusters(DeviceState* dev, int cs, size_t smem) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev->sk_clusters[cs] == 0) {
    int n = -1;
    if (ensure_smem(reinterpret_cast<const void*>(skinny_kernel<16>), smem)) {
      cudaLaunchConfig_t cfg;
      std::memset(&cfg, 0, sizeof cfg);
      cfg.gridDim = dim3(cs * 64);
      cfg.blockDim = dim3(kSkThreads);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = static_cast<unsigned>(cs);
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, skinny_kernel<16>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = -1;
      }
    }
    dev->sk_clusters[cs] = n;
  }
  return dev->sk_clusters[cs];
}

SkPlan sk_plan(int M, int N, int K, DeviceState* dev) {
  SkPlan p;
  std::memset(&p, 0, sizeof p);
  if (M < 1 || M > 64) return p;
  p.bn = M <= 16 ? 16 : M <= 32 ? 32 : 64;
  p.row_tiles = (N + kTcRows - 1) / kTcRows;
  p.kchunks = (K + 127) / 128;
  const size_t budget = 227 * 1024;
  const int maxch = static_cast<int>(std::min<size_t>(kSkMaxChunks, (budget - sk_fixed_bytes(p.bn)) /
                                                                        sk_chunk_bytes(p.bn)));
  const int cs_min = (p.kchunks + maxch - 1) / maxch;
  if (cs_min > kSkMaxCluster) return p;
  // as many K slices as keep the whole grid in one wave of clusters (one CTA per SM)
  int cs = std::max(1, std::min(std::min(dev->sm_count / p.row_tiles, kSkMaxCluster), p.kchunks));
  cs = std::max(cs, cs_min);
  for (; cs > cs_min; --cs) {
    const int per = (p.kchunks + cs - 1) / cs;
    const int n = sk_active_clusters(dev, cs, std::max(sk_smem_bytes(p.bn, per), kSkMinSmem));
    if (n >= p.row_tiles) break;
  }
  p.per = (p.kchunks + cs - 1) / cs;
  p.cs = (p.kchunks + p.per - 1) / p.per;  // no empty slice
  if (sk_band_rows(p.cs, p.cs - 1) <= 0) return p;  // every CTA owns some rows of the tile
  p.smem = std::max(sk_smem_bytes(p.bn, p.per), kSkMinSmem);
  if (sk_active_clusters(dev, p.cs, p.smem) <= 0) return p;  // this cluster size cannot be launched here
  p.ok = true;
  return p;
}

bitlinear_status skinny_launch(const bitlinear_weights* w, const uint16_t* x, int M, uint16_t* y, int32_t* acc,
                               bool pdl, cudaStream_t s, DeviceState* dev, const SkPlan& p) {
  const int N = w->N, K = w->K;
  const int64_t ld = dense_ld(K);
  CUtensorMap mW;
  if (!make_map_u8(&mW, w->codes, static_cast<uint64_t>(ld), static_cast<uint64_t>(N), static_cast<uint64_t>(ld), 32,
                   kTcRows, 0))
    return BITLINEAR_ERR_CUDA;
  SkArgs sa;
  sa.x = x;
  sa.M = M;
  sa.N = N;
  sa.K = K;
  sa.kchunks = p.kchunks;
  sa.per = p.per;
  sa.cs = p.cs;
  sa.alpha = w->alpha;
  sa.y = y;
  sa.acc = acc;
  sa.status = dev->status;
  const dim3 grid(static_cast<unsigned>(p.row_tiles * p.cs));
  bitlinear_status st;
  switch (p.bn) {
    case 16: st = launch_ex(skinny_kernel<16>, grid, dim3(kSkThreads), p.smem, s, pdl, p.cs, mW, sa); break;
    case 32: st = launch_ex(skinny_kernel<32>, grid, dim3(kSkThreads), p.smem, s, pdl, p.cs, mW, sa); break;
    default: st = launch_ex(skinny_kernel<64>, grid, dim3(kSkThreads), p.smem, s, pdl, p.cs, mW, sa); break;
  }
  if (st == BITLINEAR_OK) t_last_kernel = p.bn == 16 ? "tc_skinny_bn16" : p.bn == 32 ? "tc_skinny_bn32" : "tc_skinny_bn64";
  return st;
}

// Token-side scratch of the tensor-core path: the codes in contraction order,
// gamma and the code sums.  One quantisation serves every matrix that
// multiplies the same x.
struct QuantWs {
  int8_t* q;        // [M, ldq] natural K order
  int ldq;          // row stride of q in bytes (k16(K) in the workspace)
  float* gamma;     // [M]
  int32_t* rowsum;  // [M]
  uint32_t* cnt;    // [ncnt] split-K arrival counters (zeroed by the quantisation kernel)
  int ncnt;         // 0 when no GEMM of the call splits K
  float* part;      // split-K fp32 sums [M][max N] (zeroed by the quantisation kernel)
  size_t part_words;
};

QuantWs tc_ws_layout(void* ws, int M, int K, int ncnt, int max_n) {
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  QuantWs r;
  r.q = reinterpret_cast<int8_t*>(wsb);
  r.ldq = static_cast<int>(k16(K));
  r.gamma = reinterpret_cast<float*>(wsb + align256(static_cast<size_t>(M) * k16(K)));
  r.rowsum = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(r.gamma) + align256(4 * static_cast<size_t>(M)));
  r.cnt = reinterpret_cast<uint32_t*>(wsb + tc_base_bytes(M, K));
  r.ncnt = ncnt;
  r.part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(r.cnt) + tc_cnt_bytes(ncnt > 0 ? ncnt : 0));
  r.part_words = ncnt > 0 ? static_cast<size_t>(M) * max_n : 0;
  return r;
}

// The quant_act_kernel instantiation for G k-groups per lane in registers.
template <bool kPermute, bool kNorm>
auto quant_kernel(int G) {
  return G == 2 ? quant_act_kernel<kPermute, kNorm, 2>
                : G == 3 ? quant_act_kernel<kPermute, kNorm, 3> : quant_act_kernel<kPermute, kNorm, 8>;
}

bitlinear_status tc_quant(const uint16_t* x, int M, int K, const QuantWs& qw, bool pdl, cudaStream_t s,
                          const float* gnorm = nullptr, float eps = 0.0f) {
  const QuantShape qs = quant_shape(M, K, gnorm != nullptr, plan_sm_count());
  const int wpr = qs.wpr;
  const int rows_per_cta = kQuantWarps / wpr;
  const int qblocks = (M + rows_per_cta - 1) / rows_per_cta;
  // extra CTAs clear the split-K sums, 16 bytes per thread and step, at most four steps each
  const size_t vec4 = (qw.part_words + 3) / 4;
  const int zblocks = static_cast<int>(std::min<size_t>(1024, (vec4 + 4 * 32 * kQuantWarps - 1) /
                                                                   (4 * 32 * kQuantWarps)));
  uint32_t* cnt = qw.ncnt > 0 ? qw.cnt : static_cast<uint32_t*>(nullptr);
  // natural K order, rows zero-padded to a multiple of 16 (the order every tensor-core GEMM reads;
  // the structured-sparse MMA's metadata names positions inside runs of four consecutive k)
  auto go = [&](auto kern, const float* g, float e) {
    return launch(kern, dim3(qblocks + zblocks), dim3(32 * kQuantWarps), 0, s, pdl, x, M, K, static_cast<int>(k16(K)),
                  qw.q, qw.gamma, qw.rowsum, cnt, qw.ncnt, qw.part, vec4, qblocks, wpr, g, e);
  };
  if (gnorm) return go(quant_kernel<false, true>(qs.G), gnorm, eps);
  return go(quant_kernel<false, false>(qs.G), static_cast<const float*>(nullptr), 0.0f);
}

template <int NM, int BN>
bitlinear_status tc2_launch(const bitlinear_weights* w, int M, const QuantWs& qw, uint16_t* y, int32_t* acc,
                            cudaStream_t s, DeviceState* dev, float qb, const TcPlan& plan, int pairs) {
  using C = T2<NM, BN>;
  const int N = w->N, K = w->K;
  CUtensorMap mB, mA, mMeta;
  if (!make_map_u8(&mB, qw.q, static_cast<uint64_t>(k16(K)), static_cast<uint64_t>(M), static_cast<uint64_t>(qw.ldq),
                   kTcSubK, static_cast<uint32_t>(C::HALF), 128))
    return BITLINEAR_ERR_CUDA;
  if (NM == 0) {
    const int64_t ld = dense_ld(K);
    // packed rows land swizzled (128-byte rows at 512 k a stage, 64-byte rows at 256 k)
    if (!make_map_u8(&mA, w->codes, ld, N, ld, 32 * C::KSUB, kTcRows, 32 * C::KSUB)) return BITLINEAR_ERR_CUDA;
    mMeta = mA;
  } else {
    int64_t ldv = 0, ldm = 0;
    if (bitlinear_packed_layout(N, K, w->nm_n, w->nm_m, &ldv, &ldm, nullptr, nullptr) != BITLINEAR_OK)
      return BITLINEAR_ERR_PATTERN;
    // n:8: the kept codes (4 n bytes per 128 k) and the masks (16 bytes per 128 k) of a stage per row
    const uint32_t vbox = static_cast<uint32_t>(NM == 2 ? 4 * C::KSUB * w->nm_n : 16 * C::KSUB);
    const uint32_t mbox = static_cast<uint32_t>(16 * C::KSUB);
    if (NM == 2 && vbox % 16 != 0) return BITLINEAR_ERR_DEVICE;  // odd n runs 512-k stages only
    if (ldv < vbox || ldm < mbox) return BITLINEAR_ERR_DEVICE;  // rows shorter than one stage's box
    if (!make_map_u8(&mA, w->codes, ldv, N, ldv, vbox, kTcRows, 0)) return BITLINEAR_ERR_CUDA;
    if (!make_map_u8(&mMeta, w->meta, ldm, N, ldm, mbox, kTcRows, 0)) return BITLINEAR_ERR_CUDA;
  }
  TcArgs ta;
  std::memset(&ta, 0, sizeof ta);
  ta.M = M;
  ta.N = N;
  ta.K = K;
  ta.kblocks = (K + kTcSubK * C::KSUB - 1) / (kTcSubK * C::KSUB);  // the pair GEMM's own k-block
  ta.row_tiles = (N + kT2Rows - 1) / kT2Rows;
  ta.tok_tiles = (M + BN - 1) / BN;
  ta.ksplit = 1;
  ta.kbs = ta.kblocks;
  ta.gamma = qw.gamma;
  ta.alpha = w->alpha;
  ta.rowsum = NM == 3 ? nullptr : qw.rowsum;
  ta.nm_n = w->nm_n;
  ta.y = y;
  ta.acc = acc;
  ta.qb = qb;
  ta.status = dev->status;
  ta.vec_store = aligned16(y) && (!acc || aligned16(acc)) && (N % 8) == 0;
  pairs = std::min(pairs, ta.row_tiles * ta.tok_tiles);
  const bitlinear_status st =
      launch_ex(tc2_gemm_kernel<NM, BN>, dim3(2 * pairs), dim3(kTcThreads), C::SMEM, s, true, 2, mB, mA, mMeta, ta);
  static const char* names[3][4] = {
      {"tc2_gemm_dense_bn128", "tc2_gemm_dense_bn160", "tc2_gemm_dense_bn192", "tc2_gemm_dense_bn224"},
      {"tc2_gemm_sp24_bn128", "tc2_gemm_sp24_bn160", "tc2_gemm_sp24_bn192", "tc2_gemm_sp24_bn224"},
      {"tc2_gemm_n8_bn128", "tc2_gemm_n8_bn160", "tc2_gemm_n8_bn192", "tc2_gemm_n8_bn224"}};
  if (st == BITLINEAR_OK) t_last_kernel = names[NM == 0 ? 0 : NM == 3 ? 1 : 2][(BN - 128) / 32];
  return st;
}

// Token tile of the pair GEMM: the fewest (rounds of the pairs) x (time of one
// tile).  A wider tile does more work per k-block but may leave the last round
// of pairs half idle.  A tile's time is modelled as a + b x (K / 256) ns: a =
// 3.5 ns per token (epilogue and pipeline fill), b fitted to measured GEMM
// times of 2048 -> 11008 and 11008 -> 2048 at M = 4096 on 148 SMs.  Dense b
// grows with the tile (the codes in shared memory are read by every MMA, and
// BN = 128 keeps them in TMEM instead); 2:4 b barely does; n:8 b is set by
// the expansion of kept codes and masks.
constexpr int kT2Bn[4] = {128, 160, 192, 224};
// [dense, 2:4, n:8][BN]: ns per 256 k (n:8 measured on 6:8)
constexpr int kT2B[3][4] = {{418, 577, 600, 633}, {456, 511, 511, 514}, {793, 833, 832, 860}};

int t2_pick_bn(int nm, int row_tiles, int M, int K, const int pairs[4]) {
  int best = 0;
  int64_t best_cost = -1;
  for (int v = 0; v < 4; ++v) {
    if (pairs[v] < 1) continue;
    const int64_t units = static_cast<int64_t>(row_tiles) * ((M + kT2Bn[v] - 1) / kT2Bn[v]);
    const int64_t tile_ns = (7 * kT2Bn[v]) / 2 + static_cast<int64_t>(kT2B[nm == 0 ? 0 : nm == 3 ? 1 : 2][v]) * K / 256;
    const int64_t cost = (units + pairs[v] - 1) / pairs[v] * tile_ns;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = kT2Bn[v];
    }
  }
  return best;
}

// The pair GEMM (gemm_tc2.cuh) for a plan of 128-token tiles without a K split
// (the pair kernel then picks its own token tile, 128 to 224).
// DEVICE: no pair fits at once.  (Dense token tiles of 96 and 64 were measured
// too: a k-block's cost is mostly per instruction and per hand-off, so a
// narrower tile did less work in nearly the same time.)
template <int NM>
bitlinear_status tc2_gemm(const bitlinear_weights* w, int M, const QuantWs& qw, uint16_t* y, int32_t* acc,
                          cudaStream_t s, DeviceState* dev, float qb, const TcPlan& plan) {
  if (NM == 2 && (w->nm_n & 1)) {  // odd n: 128-token tiles (512-k stages keep the kept codes 16-byte aligned)
    const int pairs = t2_active_pairs<NM, 128>(dev);
    if (pairs < 1) return BITLINEAR_ERR_DEVICE;
    return tc2_launch<NM, 128>(w, M, qw, y, acc, s, dev, qb, plan, pairs);
  } else {
    const int pairs[4] = {t2_active_pairs<NM, 128>(dev), t2_active_pairs<NM, 160>(dev),
                          t2_active_pairs<NM, 192>(dev), t2_active_pairs<NM, 224>(dev)};
    switch (t2_pick_bn(NM, (w->N + kT2Rows - 1) / kT2Rows, M, w->K, pairs)) {
      case 128: return tc2_launch<NM, 128>(w, M, qw, y, acc, s, dev, qb, plan, pairs[0]);
      case 160: return tc2_launch<NM, 160>(w, M, qw, y, acc, s, dev, qb, plan, pairs[1]);
      case 192: return tc2_launch<NM, 192>(w, M, qw, y, acc, s, dev, qb, plan, pairs[2]);
      case 224: return tc2_launch<NM, 224>(w, M, qw, y, acc, s, dev, qb, plan, pairs[3]);
      default: return BITLINEAR_ERR_DEVICE;
    }
  }
}

// sparse24: 2:4 weights on the structured-sparse MMA (otherwise expanded for the dense one).
bitlinear_status tc_gemm(const bitlinear_weights* w, int M, const QuantWs& qw, uint16_t* y, int32_t* acc,
                         cudaStream_t s, DeviceState* dev, float qb = kQb, bool sparse24 = true) {
  const int N = w->N, K = w->K;
  const int nm = (w->nm_m == 0) ? 0 : (w->nm_m == 4 ? (sparse24 ? 3 : 1) : 2);
  const TcPlan plan = tc_plan(M, N, K, nm, dev->sm_count);
  if ((nm == 0 || nm == 2 || nm == 3) && plan.bn == 128 && plan.ksplit == 1) {
    const bitlinear_status st = nm == 0   ? tc2_gemm<0>(w, M, qw, y, acc, s, dev, qb, plan)
                                : nm == 3 ? tc2_gemm<3>(w, M, qw, y, acc, s, dev, qb, plan)
                                          : tc2_gemm<2>(w, M, qw, y, acc, s, dev, qb, plan);
    if (st != BITLINEAR_ERR_DEVICE) return st;  // DEVICE: no pair fits at once, take the one-CTA kernel
  }
  const int bn = plan.bn;
  CUtensorMap mB, mA, mMeta;
  if (!make_map_u8(&mB, qw.q, static_cast<uint64_t>(k16(K)), static_cast<uint64_t>(M), static_cast<uint64_t>(qw.ldq),
                   kTcSubK, static_cast<uint32_t>(bn), 128))
    return BITLINEAR_ERR_CUDA;
  TcArgs ta;
  ta.M = M;
  ta.N = N;
  ta.K = K;
  ta.kblocks = plan.kblocks;
  ta.row_tiles = plan.row_tiles;
  ta.tok_tiles = plan.tok_tiles;
  ta.ksplit = plan.ksplit;
  ta.kbs = plan.kbs;
  ta.part = plan.ksplit > 1 ? qw.part : nullptr;
  ta.cnt = plan.ksplit > 1 ? qw.cnt : nullptr;
  if (plan.ksplit > 1 && (qw.ncnt < plan.row_tiles * plan.tok_tiles)) return BITLINEAR_ERR_WORKSPACE;
  ta.gamma = qw.gamma;
  ta.alpha = w->alpha;
  ta.rowsum = nm == 3 ? nullptr : qw.rowsum;  // signed kept weights: no code-sum correction
  ta.y = y;
  ta.acc = acc;
  ta.nm_n = w->nm_n;
  ta.vbox = 0;
  ta.qb = qb;
  ta.status = dev->status;
  ta.vec_store = aligned16(y) && (!acc || aligned16(acc)) && (N % 8) == 0;
  if (nm == 0) {
    const int64_t ld = dense_ld(K);
    if (!make_map_u8(&mA, w->codes, ld, N, ld, 32 * tc_ksub(0, bn), kTcRows, 0)) return BITLINEAR_ERR_CUDA;
    mMeta = mA;
  } else {
    int64_t ldv = 0, ldm = 0;
    if (bitlinear_packed_layout(N, K, w->nm_n, w->nm_m, &ldv, &ldm, nullptr, nullptr) != BITLINEAR_OK)
      return BITLINEAR_ERR_PATTERN;
    const uint32_t vbox = nm != 2 ? static_cast<uint32_t>(16 * tc_ksub(nm, bn))
                                  : static_cast<uint32_t>((4 * w->nm_n + 12 + 15) / 16 * 16);
    ta.vbox = static_cast<int>(vbox);
    if (!make_map_u8(&mA, w->codes, ldv, N, ldv, vbox, kTcRows, 0)) return BITLINEAR_ERR_CUDA;
    if (!make_map_u8(&mMeta, w->meta, ldm, N, ldm, static_cast<uint32_t>(16 * tc_ksub(nm, bn)), kTcRows, 0))
      return BITLINEAR_ERR_CUDA;
  }
  bitlinear_status st;
  if (nm == 0)
    st = launch_tc<0>(bn, mB, mA, mMeta, ta, dev->sm_count, s);
  else if (nm == 1)
    st = launch_tc<1>(bn, mB, mA, mMeta, ta, dev->sm_count, s);
  else if (nm == 3)
    st = launch_tc<3>(bn, mB, mA, mMeta, ta, dev->sm_count, s);
  else
    st = launch_tc<2>(bn, mB, mA, mMeta, ta, dev->sm_count, s);
  if (st == BITLINEAR_OK) t_last_kernel = tc_name(nm, bn);
  return st;
}

// H-BitLinear activations for the tensor-core GEMM: Hadamard transform and
// 4-bit codes in contraction order (plus the split-K clearing of tc_quant).
bitlinear_status hbit_quant(const uint16_t* x, int M, int K, int8_t* q, int ldq, bool permute, float* gamma,
                            int32_t* rowsum, uint32_t* cnt, int ncnt, float* part, size_t part_words, bool pdl,
                            cudaStream_t s) {
  const int B = hbit_block(K);
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(B)));
  const size_t vec4 = (part_words + 3) / 4;
  const int zblocks = static_cast<int>(std::min<size_t>(1024, (vec4 + 4 * kHbitThreads - 1) / (4 * kHbitThreads)));
  const size_t smem = static_cast<size_t>(K) * 4;
  const dim3 grid(static_cast<unsigned>(M + zblocks)), block(kHbitThreads);
  auto go = [&](auto kern) {
    return launch(kern, grid, block, smem, s, pdl, x, M, K, B, scale, ldq, q, gamma, rowsum, cnt, ncnt, part, vec4);
  };
  switch (hbit_vals_per_lane(B)) {
    case 1: return permute ? go(hbit_quant_kernel<true, 1>) : go(hbit_quant_kernel<false, 1>);
    case 2: return permute ? go(hbit_quant_kernel<true, 2>) : go(hbit_quant_kernel<false, 2>);
    case 4: return permute ? go(hbit_quant_kernel<true, 4>) : go(hbit_quant_kernel<false, 4>);
    case 8: return permute ? go(hbit_quant_kernel<true, 8>) : go(hbit_quant_kernel<false, 8>);
    case 16: return permute ? go(hbit_quant_kernel<true, 16>) : go(hbit_quant_kernel<false, 16>);
    case 32: return permute ? go(hbit_quant_kernel<true, 32>) : go(hbit_quant_kernel<false, 32>);
    case 64: return permute ? go(hbit_quant_kernel<true, 64>) : go(hbit_quant_kernel<false, 64>);
    default: return permute ? go(hbit_quant_kernel<true, 0>) : go(hbit_quant_kernel<false, 0>);
  }
}

// Activation quantisation feeding the tensor-core GEMM.
enum class ActKind { kInt8, kInt8Norm, kHbit4 };

bitlinear_status forward_tc(const bitlinear_weights* w, const uint16_t* x, int M, uint16_t* y, int32_t* acc,
                            void* ws, size_t ws_bytes, bool pdl, cudaStream_t s, DeviceState* dev,
                            const float* gnorm = nullptr, float eps = 0.0f, ActKind act = ActKind::kInt8,
                            bool nm24_expand = false) {
  const int nm = w->nm_m == 0 ? 0 : (w->nm_m == 4 ? 1 : 2);
  const bool sparse24 = !nm24_expand;  // 2:4 weights on the structured-sparse MMA
  if (!ws || ws_bytes < tc_workspace(M, w->N, w->K, nm, dev->sm_count) || !aligned16(ws))
    return BITLINEAR_ERR_WORKSPACE;
  const bool split = tc_plan(M, w->N, w->K, nm, dev->sm_count).ksplit > 1;
  const QuantWs qw = tc_ws_layout(ws, M, w->K, split ? dev->sm_count : 0, w->N);
  bitlinear_status st;
  if (act == ActKind::kHbit4) {
    st = hbit_quant(x, M, w->K, qw.q, static_cast<int>(k16(w->K)), false, qw.gamma, qw.rowsum,
                    qw.ncnt > 0 ? qw.cnt : nullptr, qw.ncnt, qw.part, qw.part_words, pdl, s);
    if (st != BITLINEAR_OK) return st;
    return tc_gemm(w, M, qw, y, acc, s, dev, kQb4, sparse24);
  }
  st = tc_quant(x, M, w->K, qw, pdl, s, act == ActKind::kInt8Norm ? gnorm : nullptr, eps);
  if (st != BITLINEAR_OK) return st;
  return tc_gemm(w, M, qw, y, acc, s, dev, kQb, sparse24);
}

// ---------------------------------------------------------------- GEMV path
// Shared-memory budget for one CTA's weight rows in the decode GEMV: small
// enough that the next kernel's CTA (launched early under PDL) fits beside it.
constexpr int64_t kGemvWeightSmem = 96 * 1024;

// Splits about one CTA per SM over the matrices of a group in proportion to
// their rows, then doubles every share until one CTA's rows fit the
// shared-memory budget and a TMA box (at most 256 rows).  Returns the box
// height; fills cta_begin, rows_base, rows_rem and the total CTA count.
int gemv_split(GemvDense& g, const int* N, int count, int sm_count, int* grid) {
  int64_t R = 0;
  for (int i = 0; i < count; ++i) R += N[i];
  int share[kGemvGroup];
  int used = 0;
  for (int i = 0; i < count; ++i) {
    share[i] = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(N[i], sm_count * static_cast<int64_t>(N[i]) / R)));
    used += share[i];
  }
  // hand the CTAs left over to the matrices with the most rows per CTA
  while (used < sm_count) {
    int best = -1;
    for (int i = 0; i < count; ++i)
      if (share[i] < N[i] && (best < 0 || static_cast<int64_t>(N[i]) * share[best] > static_cast<int64_t>(N[best]) * share[i]))
        best = i;
    if (best < 0) break;
    ++share[best];
    ++used;
  }
  auto box = [&]() {
    int b = 0;
    for (int i = 0; i < count; ++i) b = std::max(b, N[i] / share[i] + 1);
    return b;
  };
  auto fits = [&](int rows_box) {
    return rows_box <= 256 && gemv_smem_bytes(rows_box, g.ld, g.C) <= static_cast<size_t>(kGemvWeightSmem) + 16 * 1024;
  };
  for (;;) {
    if (fits(box())) break;
    bool grew = false;
    for (int i = 0; i < count; ++i)
      if (share[i] < N[i]) {
        share[i] = std::min(N[i], share[i] * 2);
        grew = true;
      }
    if (!grew) break;
  }
  int begin = 0;
  for (int i = 0; i < count; ++i) {
    g.mat[i].cta_begin = begin;
    g.mat[i].rows_base = N[i] / share[i];
    g.mat[i].rows_rem = N[i] % share[i];
    begin += share[i];
  }
  g.count = count;
  *grid = begin;
  return box();
}

// One launch of the dense decode GEMV over `count` matrices sharing x.
bitlinear_status gemv_dense_launch(const bitlinear_weights* const* w, uint16_t* const* y, int32_t* const* acc,
                                   int count, const uint16_t* x, bool pdl, cudaStream_t s, DeviceState* dev,
                                   const float* gnorm = nullptr, float eps = 0.0f) {
  GemvDense g;
  std::memset(&g, 0, sizeof g);
  g.gnorm = gnorm;
  g.eps = eps;
  const int K = w[0]->K;
  g.ld = dense_ld(K);
  g.C = static_cast<int>(g.ld / 16);
  g.K = K;
  g.x = x;
  g.status = dev->status;
  int N[kGemvGroup];
  for (int i = 0; i < count; ++i) N[i] = w[i]->N;
  int grid = 0;
  g.rows_box = gemv_split(g, N, count, dev->sm_count, &grid);
  CUtensorMap map[kGemvGroup];
  for (int i = 0; i < count; ++i) {
    g.mat[i].alpha = w[i]->alpha;
    g.mat[i].y = y[i];
    g.mat[i].acc = acc ? acc[i] : nullptr;
    if (!make_map_u8(&map[i], w[i]->codes, static_cast<uint64_t>(g.ld), static_cast<uint64_t>(N[i]),
                     static_cast<uint64_t>(g.ld), 128, static_cast<uint32_t>(g.rows_box), 128))
      return BITLINEAR_ERR_CUDA;
  }
  for (int i = count; i < kGemvGroup; ++i) map[i] = map[0];  // never selected
  bitlinear_status st;
  if (gnorm) {
    const size_t smem = gemv_smem_bytes(g.rows_box, g.ld, g.C) + 4 * static_cast<size_t>(K);
    st = launch(gemv_dense_kernel<true>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, map[0], map[1], map[2], map[3],
                g);
  } else {
    const size_t smem = gemv_smem_bytes(g.rows_box, g.ld, g.C);
    st = launch(gemv_dense_kernel<false>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, map[0], map[1], map[2], map[3],
                g);
  }
  if (st == BITLINEAR_OK) t_last_kernel = "gemv_m1_dense";
  return st;
}

// Rows per CTA of the fused one-token kernel: about one CTA per SM, doubled
// until both matrices' rows fit the shared-memory budget and a box of at most
// 128 rows (a multiple of 8).  False: no such split (very long K).
bool glu_split(int N, int64_t ld, int C, int sm_count, int* ctas, int* rows_box) {
  int c = std::max(1, std::min(N, sm_count));
  for (;;) {
    const int rows = (N + c - 1) / c;
    const int box = (rows + 7) / 8 * 8;
    if (box <= 128 && gemv_glu_smem_bytes(box, ld, C) <= static_cast<size_t>(kGemvWeightSmem) + 16 * 1024) {
      *ctas = c;
      *rows_box = box;
      return true;
    }
    if (c >= N) return false;
    c = std::min(N, 2 * c);
  }
}


// The lookup-table variant of the dense decode GEMV (one matrix).
bitlinear_status gemv_lut_launch(const bitlinear_weights* w, uint16_t* y, int32_t* acc, const uint16_t* x, bool pdl,
                                 cudaStream_t s, DeviceState* dev) {
  GemvDense g;
  std::memset(&g, 0, sizeof g);
  const int N = w->N, K = w->K;
  g.ld = dense_ld(K);
  g.C = static_cast<int>(g.ld / 16);
  g.K = K;
  g.x = x;
  g.status = dev->status;
  g.count = 1;
  int grid = std::min(dev->sm_count, N);
  auto fits = [&](int gr) {
    const int rows_box = N / gr + 1;
    return rows_box <= 256 && gemv_lut_smem_bytes(rows_box, g.ld, g.C) <= 200 * 1024;
  };
  while (!fits(grid) && grid < N) grid = std::min(N, grid * 2);
  if (!fits(grid)) return BITLINEAR_ERR_SHAPE;
  g.mat[0].alpha = w->alpha;
  g.mat[0].y = y;
  g.mat[0].acc = acc;
  g.mat[0].rows_base = N / grid;
  g.mat[0].rows_rem = N % grid;
  g.rows_box = g.mat[0].rows_base + 1;
  CUtensorMap map;
  if (!make_map_u8(&map, w->codes, static_cast<uint64_t>(g.ld), static_cast<uint64_t>(N), static_cast<uint64_t>(g.ld),
                   128, static_cast<uint32_t>(g.rows_box), 128))
    return BITLINEAR_ERR_CUDA;
  bitlinear_status st = launch(gemv_lut_kernel, dim3(grid), dim3(kGemvThreads),
                               gemv_lut_smem_bytes(g.rows_box, g.ld, g.C), s, pdl, map, g);
  if (st == BITLINEAR_OK) t_last_kernel = "gemv_m1_dense_lut";
  return st;
}

bitlinear_status forward_gemv(const bitlinear_weights* w, const uint16_t* x, uint16_t* y, int32_t* acc, bool pdl,
                              cudaStream_t s, DeviceState* dev, bool lut = false) {
  const int N = w->N, K = w->K;
  if (w->nm_m == 0 && lut) return gemv_lut_launch(w, y, acc, x, pdl, s, dev);
  if (w->nm_m == 0) return gemv_dense_launch(&w, &y, &acc, 1, x, pdl, s, dev);
  int64_t ldv = 0, ldm = 0;
  if (bitlinear_packed_layout(N, K, w->nm_n, w->nm_m, &ldv, &ldm, nullptr, nullptr) != BITLINEAR_OK)
    return BITLINEAR_ERR_PATTERN;
  GemvNmArgs na;
  std::memset(&na, 0, sizeof na);
  na.x = x;
  na.alpha = w->alpha;
  na.y = y;
  na.acc = acc;
  na.status = dev->status;
  na.ld_v = ldv;
  na.ld_m = ldm;
  na.K = K;
  na.C = (K + 127) / 128;
  const bool nm_lut = w->nm_m == 4;
  // about one CTA per SM; more while a CTA's rows exceed a TMA box or the shared-memory budget
  int grid = std::min(dev->sm_count, N);
  auto fits = [&](int g) {
    const int rows_box = N / g + 1;
    return rows_box <= 256 && gemv_nm_smem_bytes(rows_box, ldv, ldm, na.C, nm_lut) <= 160 * 1024;
  };
  while (!fits(grid) && grid < N) grid = std::min(N, grid * 2);
  na.rows_base = N / grid;
  na.rows_rem = N % grid;
  na.rows_box = na.rows_base + 1;
  CUtensorMap mv, mm;
  if (!make_map_u8(&mv, w->codes, static_cast<uint64_t>(ldv), static_cast<uint64_t>(N), static_cast<uint64_t>(ldv), 128,
                   static_cast<uint32_t>(na.rows_box), 128) ||
      !make_map_u8(&mm, w->meta, static_cast<uint64_t>(ldm), static_cast<uint64_t>(N), static_cast<uint64_t>(ldm), 128,
                   static_cast<uint32_t>(na.rows_box), 128))
    return BITLINEAR_ERR_CUDA;
  const size_t smem = gemv_nm_smem_bytes(na.rows_box, ldv, ldm, na.C, nm_lut);
  bitlinear_status st;
  switch (w->nm_m == 4 ? 0 : w->nm_n) {
    case 0: st = launch(gemv_nm_kernel<0>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 1: st = launch(gemv_nm_kernel<1>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 2: st = launch(gemv_nm_kernel<2>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 3: st = launch(gemv_nm_kernel<3>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 4: st = launch(gemv_nm_kernel<4>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 5: st = launch(gemv_nm_kernel<5>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    case 6: st = launch(gemv_nm_kernel<6>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
    default: st = launch(gemv_nm_kernel<7>, dim3(grid), dim3(kGemvThreads), smem, s, pdl, mv, mm, na); break;
  }
  if (st == BITLINEAR_OK) t_last_kernel = w->nm_m == 4 ? "gemv_m1_nm24" : "gemv_m1_n8";
  return st;
}

// Checks one matrix and its outputs (x and the flags are checked by the caller).
bitlinear_status check_matrix(const bitlinear_weights* w, const uint16_t* y, const int32_t* acc) {
  if (!w || !y || !w->codes || !w->alpha) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_nk(w->N, w->K);
  if (st != BITLINEAR_OK) return st;
  if (!pattern_ok(w->nm_n, w->nm_m)) return BITLINEAR_ERR_PATTERN;
  const bool is_nm = w->nm_m != 0;
  if (is_nm && !w->meta) return BITLINEAR_ERR_NULL;
  if (is_nm && w->K % w->nm_m != 0) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(w->codes) || (is_nm && !aligned16(w->meta))) return BITLINEAR_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(y) & 1u) || (acc && (reinterpret_cast<uintptr_t>(acc) & 3u)) ||
      (reinterpret_cast<uintptr_t>(w->alpha) & 3u))
    return BITLINEAR_ERR_ALIGN;
  return BITLINEAR_OK;
}

bitlinear_status check_flags(uint32_t flags, int M) {
  const uint32_t known = BITLINEAR_FLAG_PDL | BITLINEAR_FLAG_PATH_GEMV | BITLINEAR_FLAG_PATH_TC |
                         BITLINEAR_FLAG_DECODE_LUT | BITLINEAR_FLAG_PATH_PERSISTENT | BITLINEAR_FLAG_NM24_EXPAND;
  if (flags & ~known) return BITLINEAR_ERR_FLAGS;
  if ((flags & BITLINEAR_FLAG_PATH_GEMV) && ((flags & BITLINEAR_FLAG_PATH_TC) || M != 1)) return BITLINEAR_ERR_FLAGS;
  if ((flags & BITLINEAR_FLAG_DECODE_LUT) && ((flags & BITLINEAR_FLAG_PATH_TC) || M != 1)) return BITLINEAR_ERR_FLAGS;
  if ((flags & BITLINEAR_FLAG_PATH_PERSISTENT) && (flags & (BITLINEAR_FLAG_PATH_GEMV | BITLINEAR_FLAG_DECODE_LUT)))
    return BITLINEAR_ERR_FLAGS;
  return BITLINEAR_OK;
}

bitlinear_status forward_common(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y, int32_t* acc,
                                void* ws, size_t ws_bytes, uint32_t flags, void* stream, bool want_nm) {
  if (!w || !x || !y) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_matrix(w, y, acc);
  if (st != BITLINEAR_OK) return st;
  if (M < 1 || M > BITLINEAR_MAX_M) return BITLINEAR_ERR_SHAPE;
  if ((w->nm_m != 0) != want_nm) return BITLINEAR_ERR_PATTERN;
  if (!aligned16(x)) return BITLINEAR_ERR_ALIGN;
  st = check_flags(flags, M);
  if (st != BITLINEAR_OK) return st;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const bool pdl = (flags & BITLINEAR_FLAG_PDL) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tc = (flags & BITLINEAR_FLAG_PATH_TC) || M > 1;
  if (tc && w->nm_m == 0 && !(flags & BITLINEAR_FLAG_PATH_PERSISTENT)) {
    const SkPlan p = sk_plan(M, w->N, w->K, dev);
    if (p.ok) return skinny_launch(w, x, M, y, acc, pdl, s, dev, p);
  }
  if (tc)
    return forward_tc(w, x, M, y, acc, ws, ws_bytes, pdl, s, dev, nullptr, 0.0f, ActKind::kInt8,
                      (flags & BITLINEAR_FLAG_NM24_EXPAND) != 0);
  if ((flags & BITLINEAR_FLAG_DECODE_LUT) && want_nm) return BITLINEAR_ERR_FLAGS;
  return forward_gemv(w, x, y, acc, pdl, s, dev, (flags & BITLINEAR_FLAG_DECODE_LUT) != 0);
}

bitlinear_status forward_group(const bitlinear_weights* w, int count, const uint16_t* x, int M, uint16_t* const* y,
                               int32_t* const* acc, void* ws, size_t ws_bytes, uint32_t flags, void* stream) {
  if (!w || !x || !y) return BITLINEAR_ERR_NULL;
  if (count < 1 || count > BITLINEAR_MAX_GROUP) return BITLINEAR_ERR_SHAPE;
  if (M < 1 || M > BITLINEAR_MAX_M) return BITLINEAR_ERR_SHAPE;
  for (int i = 0; i < count; ++i) {
    bitlinear_status st = check_matrix(&w[i], y[i], acc ? acc[i] : nullptr);
    if (st != BITLINEAR_OK) return st;
    if (w[i].K != w[0].K) return BITLINEAR_ERR_SHAPE;
  }
  if (!aligned16(x)) return BITLINEAR_ERR_ALIGN;
  bitlinear_status st = check_flags(flags, M);
  if (st != BITLINEAR_OK) return st;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const bool pdl = (flags & BITLINEAR_FLAG_PDL) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tc = (flags & BITLINEAR_FLAG_PATH_TC) || M > 1;
  if (tc && !(flags & BITLINEAR_FLAG_PATH_PERSISTENT)) {
    // few tokens, dense weights: one fused launch per matrix (each quantises its own K slices)
    SkPlan plans[BITLINEAR_MAX_GROUP];
    bool all = true;
    for (int i = 0; i < count && all; ++i) {
      all = w[i].nm_m == 0;
      if (all) {
        plans[i] = sk_plan(M, w[i].N, w[i].K, dev);
        all = plans[i].ok;
      }
    }
    if (all) {
      for (int i = 0; i < count && st == BITLINEAR_OK; ++i)
        st = skinny_launch(&w[i], x, M, y[i], acc ? acc[i] : nullptr, i == 0 ? pdl : true, s, dev, plans[i]);
      return st;
    }
  }
  if (tc) {
    size_t need = 0;
    bool split = false;
    int max_n = 0;
    for (int i = 0; i < count; ++i) {
      const int nm = w[i].nm_m == 0 ? 0 : (w[i].nm_m == 4 ? 1 : 2);
      need = std::max(need, tc_workspace(M, w[i].N, w[i].K, nm, dev->sm_count));
      if (tc_plan(M, w[i].N, w[i].K, nm, dev->sm_count).ksplit > 1) {
        split = true;
        max_n = std::max(max_n, w[i].N);
      }
    }
    if (!ws || ws_bytes < need || !aligned16(ws)) return BITLINEAR_ERR_WORKSPACE;
    const QuantWs qw = tc_ws_layout(ws, M, w[0].K, split ? dev->sm_count : 0, max_n);
    // one quantisation serves every matrix
    const bool sparse24 = !(flags & BITLINEAR_FLAG_NM24_EXPAND);
    st = tc_quant(x, M, w[0].K, qw, pdl, s);
    for (int i = 0; i < count && st == BITLINEAR_OK; ++i)
      st = tc_gemm(&w[i], M, qw, y[i], acc ? acc[i] : nullptr, s, dev, kQb, sparse24);
    return st;
  }
  // decode: the dense matrices share one launch; each N:M matrix has its own
  const bitlinear_weights* dw[kGemvGroup];
  uint16_t* dy[kGemvGroup];
  int32_t* dacc[kGemvGroup];
  int nd = 0;
  for (int i = 0; i < count; ++i)
    if (w[i].nm_m == 0) {
      dw[nd] = &w[i];
      dy[nd] = y[i];
      dacc[nd] = acc ? acc[i] : nullptr;
      ++nd;
    }
  bool first = true;
  if (nd) {
    st = gemv_dense_launch(dw, dy, dacc, nd, x, pdl, s, dev);
    first = false;
  }
  for (int i = 0; i < count && st == BITLINEAR_OK; ++i)
    if (w[i].nm_m != 0) {
      // a later kernel of the group may start early: it reads only its weights before waiting
      st = forward_gemv(&w[i], x, y[i], acc ? acc[i] : nullptr, first ? pdl : true, s, dev);
      first = false;
    }
  return st;
}

}  // namespace
}  // namespace bl

using namespace bl;

extern "C" {

bitlinear_status bitlinear_packed_layout(int32_t N, int32_t K, int32_t nm_n, int32_t nm_m, int64_t* ld_codes,
                                         int64_t* ld_meta, size_t* codes_bytes, size_t* meta_bytes) {
  bitlinear_status st = check_nk(N, K);
  if (st != BITLINEAR_OK) return st;
  if (!pattern_ok(nm_n, nm_m)) return BITLINEAR_ERR_PATTERN;
  int64_t ldc, ldm = 0;
  if (nm_m == 0) {
    ldc = dense_ld(K);
  } else {
    if (K % nm_m != 0) return BITLINEAR_ERR_SHAPE;
    const int64_t kept = static_cast<int64_t>(K) / nm_m * nm_n;
    ldc = 16 * ((kept + 63) / 64);
    ldm = 16 * ((static_cast<int64_t>(K) + 127) / 128);
  }
  if (ld_codes) *ld_codes = ldc;
  if (ld_meta) *ld_meta = ldm;
  if (codes_bytes) *codes_bytes = static_cast<size_t>(ldc) * N;
  if (meta_bytes) *meta_bytes = static_cast<size_t>(ldm) * N;
  return BITLINEAR_OK;
}

size_t bitlinear_pack_workspace_bytes(int32_t N, int32_t K) {
  (void)N;
  (void)K;
  return 1024 * sizeof(double);
}

bitlinear_status bitlinear_pack_weights(const float* W, int32_t N, int32_t K, int32_t nm_n, int32_t nm_m,
                                        uint8_t* codes, uint8_t* meta, float* alpha, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!W || !codes || !alpha) return BITLINEAR_ERR_NULL;
  int64_t ldc = 0, ldm = 0;
  bitlinear_status st = bitlinear_packed_layout(N, K, nm_n, nm_m, &ldc, &ldm, nullptr, nullptr);
  if (st != BITLINEAR_OK) return st;
  if (nm_m != 0 && !meta) return BITLINEAR_ERR_NULL;
  if (!aligned16(codes) || (nm_m != 0 && !aligned16(meta)) || (reinterpret_cast<uintptr_t>(W) & 3u) ||
      (reinterpret_cast<uintptr_t>(alpha) & 3u))
    return BITLINEAR_ERR_ALIGN;
  if (!workspace || workspace_bytes < bitlinear_pack_workspace_bytes(N, K) ||
      (reinterpret_cast<uintptr_t>(workspace) & 7u))
    return BITLINEAR_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t count = static_cast<int64_t>(N) * K;
  const int nparts = static_cast<int>(std::min<int64_t>(1024, (count + 255) / 256));
  double* partial = static_cast<double*>(workspace);
  st = launch(absmean_partial_kernel, dim3(nparts), dim3(256), 0, s, false, W, count, partial);
  if (st != BITLINEAR_OK) return st;
  st = launch(absmean_final_kernel, dim3(1), dim3(256), 0, s, false, static_cast<const double*>(partial), nparts,
              count, alpha);
  if (st != BITLINEAR_OK) return st;
  if (nm_m == 0) {
    const int64_t units = (ldc / 16) * N;
    st = launch(pack_dense_kernel<true>, dim3(static_cast<unsigned>((units + 255) / 256)), dim3(256), 0, s, false, W,
                static_cast<const int8_t*>(nullptr), N, K, ldc, static_cast<const float*>(alpha), codes);
    if (st == BITLINEAR_OK) t_last_kernel = "pack_dense";
  } else {
    const int spans = (K / nm_m + 63) / 64;
    const int64_t threads = static_cast<int64_t>(spans) * N;
    st = launch(pack_nm_kernel, dim3(static_cast<unsigned>((threads + 127) / 128)), dim3(128), 0, s, false, W, N, K,
                nm_n, nm_m, ldc, ldm, static_cast<const float*>(alpha), codes, meta);
    if (st == BITLINEAR_OK) t_last_kernel = "pack_nm";
  }
  return st;
}

bitlinear_status bitlinear_pack_ternary(const int8_t* Wt, int32_t N, int32_t K, float alpha, uint8_t* codes,
                                        float* alpha_out, void* stream) {
  if (!Wt || !codes || !alpha_out) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_nk(N, K);
  if (st != BITLINEAR_OK) return st;
  if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(alpha_out) & 3u)) return BITLINEAR_ERR_ALIGN;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t ld = dense_ld(K);
  const int64_t units = (ld / 16) * N;
  st = launch(write_alpha_kernel, dim3(1), dim3(32), 0, s, false, alpha_out, alpha);
  if (st != BITLINEAR_OK) return st;
  st = launch(pack_dense_kernel<false>, dim3(static_cast<unsigned>((units + 255) / 256)), dim3(256), 0, s, false,
              static_cast<const float*>(nullptr), Wt, N, K, ld, static_cast<const float*>(nullptr), codes);
  if (st == BITLINEAR_OK) t_last_kernel = "pack_ternary";
  return st;
}

bitlinear_status bitlinear_quant_act(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* gamma,
                                     int32_t* rowsum, void* stream) {
  if (!x || !q || !gamma) return BITLINEAR_ERR_NULL;
  if (M < 1 || M > BITLINEAR_MAX_M || K < 1 || K > BITLINEAR_MAX_K) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(gamma) & 3u) ||
      (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
    return BITLINEAR_ERR_ALIGN;
  DeviceState* dev = nullptr;
  bitlinear_status st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const QuantShape qs = quant_shape(M, K, false, plan_sm_count());
  const int wpr = qs.wpr;
  const int qblocks = (M + kQuantWarps / wpr - 1) / (kQuantWarps / wpr);
  st = launch(quant_kernel<false, false>(qs.G), dim3(qblocks), dim3(32 * kQuantWarps), 0,
              static_cast<cudaStream_t>(stream), false, x, M, K, K, q, gamma, rowsum, static_cast<uint32_t*>(nullptr), 0,
              static_cast<float*>(nullptr), static_cast<size_t>(0), qblocks, wpr, static_cast<const float*>(nullptr),
              0.0f);
  if (st == BITLINEAR_OK) t_last_kernel = "quant_act";
  return st;
}

bitlinear_status bitlinear_rmsnorm_quant_act(const uint16_t* x, int32_t M, int32_t K, const float* g, float eps,
                                             int8_t* q, float* gamma, int32_t* rowsum, void* stream) {
  if (!x || !g || !q || !gamma) return BITLINEAR_ERR_NULL;
  if (M < 1 || M > BITLINEAR_MAX_M || K < 1 || K > BITLINEAR_MAX_K) return BITLINEAR_ERR_SHAPE;
  if (!(eps >= 0.0f) || eps > 1.0f) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(g) & 3u) || (reinterpret_cast<uintptr_t>(gamma) & 3u) ||
      (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
    return BITLINEAR_ERR_ALIGN;
  DeviceState* dev = nullptr;
  bitlinear_status st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const QuantShape qs = quant_shape(M, K, true, plan_sm_count());
  const int wpr = qs.wpr;
  const int qblocks = (M + kQuantWarps / wpr - 1) / (kQuantWarps / wpr);
  st = launch(quant_kernel<false, true>(qs.G), dim3(qblocks), dim3(32 * kQuantWarps), 0,
              static_cast<cudaStream_t>(stream), false, x, M, K, K, q, gamma, rowsum, static_cast<uint32_t*>(nullptr), 0,
              static_cast<float*>(nullptr), static_cast<size_t>(0), qblocks, wpr, g, eps);
  if (st == BITLINEAR_OK) t_last_kernel = "rmsnorm_quant_act";
  return st;
}

bitlinear_status bitlinear_forward_norm(const bitlinear_weights* w, const uint16_t* x, int32_t M, const float* g,
                                        float eps, uint16_t* y, int32_t* acc, void* workspace, size_t workspace_bytes,
                                        uint32_t flags, void* stream) {
  if (!w || !x || !y || !g) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_matrix(w, y, acc);
  if (st != BITLINEAR_OK) return st;
  if (M < 1 || M > BITLINEAR_MAX_M) return BITLINEAR_ERR_SHAPE;
  if (!(eps >= 0.0f) || eps > 1.0f) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(g) & 3u)) return BITLINEAR_ERR_ALIGN;
  if (flags & ~static_cast<uint32_t>(BITLINEAR_FLAG_PDL | BITLINEAR_FLAG_PATH_TC | BITLINEAR_FLAG_NM24_EXPAND))
    return BITLINEAR_ERR_FLAGS;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const bool pdl = (flags & BITLINEAR_FLAG_PDL) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 1 && w->nm_m == 0 && !(flags & BITLINEAR_FLAG_PATH_TC)) {
    // decode: every GEMV CTA normalises and quantises the token itself
    return gemv_dense_launch(&w, &y, &acc, 1, x, pdl, s, dev, g, eps);
  }
  return forward_tc(w, x, M, y, acc, workspace, workspace_bytes, pdl, s, dev, g, eps, ActKind::kInt8Norm,
                    (flags & BITLINEAR_FLAG_NM24_EXPAND) != 0);
}

bitlinear_status bitlinear_hadamard_quant_act4(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* gamma,
                                               int32_t* rowsum, void* stream) {
  if (!x || !q || !gamma) return BITLINEAR_ERR_NULL;
  if (M < 1 || M > BITLINEAR_MAX_M || K < 1 || K > BITLINEAR_HBIT_MAX_K) return BITLINEAR_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (reinterpret_cast<uintptr_t>(gamma) & 3u) ||
      (rowsum && (reinterpret_cast<uintptr_t>(rowsum) & 3u)))
    return BITLINEAR_ERR_ALIGN;
  DeviceState* dev = nullptr;
  bitlinear_status st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  st = hbit_quant(x, M, K, q, K, false, gamma, rowsum, nullptr, 0, nullptr, 0, false,
                  static_cast<cudaStream_t>(stream));
  if (st == BITLINEAR_OK) t_last_kernel = "hadamard_quant_act4";
  return st;
}

bitlinear_status bitlinear_forward_hbit(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                        int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                        void* stream) {
  if (!w || !x || !y) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_matrix(w, y, acc);
  if (st != BITLINEAR_OK) return st;
  if (M < 1 || M > BITLINEAR_MAX_M || w->K > BITLINEAR_HBIT_MAX_K) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(x)) return BITLINEAR_ERR_ALIGN;
  if (flags & ~static_cast<uint32_t>(BITLINEAR_FLAG_PDL | BITLINEAR_FLAG_PATH_TC | BITLINEAR_FLAG_NM24_EXPAND))
    return BITLINEAR_ERR_FLAGS;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  return forward_tc(w, x, M, y, acc, workspace, workspace_bytes, (flags & BITLINEAR_FLAG_PDL) != 0,
                    static_cast<cudaStream_t>(stream), dev, nullptr, 0.0f, ActKind::kHbit4,
                    (flags & BITLINEAR_FLAG_NM24_EXPAND) != 0);
}

bitlinear_status bitlinear_forward_q8(const bitlinear_weights* w, const int8_t* q, int32_t ldq, const float* gamma,
                                      const int32_t* rowsum, int32_t M, uint16_t* y, int32_t* acc, void* workspace,
                                      size_t workspace_bytes, uint32_t flags, void* stream) {
  if (!w || !q || !gamma || !rowsum || !y) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_matrix(w, y, acc);
  if (st != BITLINEAR_OK) return st;
  if (M < 1 || M > BITLINEAR_MAX_M || ldq < w->K || (ldq % 16) != 0) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(q) || (reinterpret_cast<uintptr_t>(gamma) & 3u) || (reinterpret_cast<uintptr_t>(rowsum) & 3u))
    return BITLINEAR_ERR_ALIGN;
  if (flags & ~static_cast<uint32_t>(BITLINEAR_FLAG_PDL | BITLINEAR_FLAG_PATH_TC | BITLINEAR_FLAG_NM24_EXPAND))
    return BITLINEAR_ERR_FLAGS;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nm = w->nm_m == 0 ? 0 : (w->nm_m == 4 ? 1 : 2);
  if (!workspace_ok_q8(workspace, workspace_bytes, M, w->N, w->K, nm, dev->sm_count)) return BITLINEAR_ERR_WORKSPACE;
  const bool split = tc_plan(M, w->N, w->K, nm, dev->sm_count).ksplit > 1;
  QuantWs qw;
  std::memset(&qw, 0, sizeof qw);
  qw.q = const_cast<int8_t*>(q);
  qw.ldq = ldq;
  qw.gamma = const_cast<float*>(gamma);
  qw.rowsum = const_cast<int32_t*>(rowsum);
  if (split) {
    // the K slices' sums and arrival counters start from zero (the quantisation launch clears them otherwise)
    qw.cnt = static_cast<uint32_t*>(workspace);
    qw.ncnt = dev->sm_count;
    qw.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + tc_cnt_bytes(dev->sm_count));
    qw.part_words = static_cast<size_t>(M) * w->N;
    if (cudaMemsetAsync(workspace, 0, tc_cnt_bytes(dev->sm_count) + 4 * qw.part_words, s) != cudaSuccess)
      return BITLINEAR_ERR_CUDA;
  }
  (void)(flags & BITLINEAR_FLAG_PDL);  // the GEMM always launches as a programmatic dependent
  return tc_gemm(w, M, qw, y, acc, s, dev, kQb, (flags & BITLINEAR_FLAG_NM24_EXPAND) == 0);
}

size_t bitlinear_forward_workspace_bytes(int32_t M, int32_t N, int32_t K, uint32_t flags) {
  if (M < 1 || K < 1 || N < 1) return 0;
  const bool tc = (flags & BITLINEAR_FLAG_PATH_TC) || (M > 1 && !(flags & BITLINEAR_FLAG_PATH_GEMV));
  if (!tc) return 0;
  // enough for dense and for N:M weights (their k-blocks differ, and with them the K split)
  const int sm = plan_sm_count();
  return std::max({tc_workspace(M, N, K, 0, sm), tc_workspace(M, N, K, 1, sm), tc_workspace(M, N, K, 2, sm)});
}

// ---------------------------------------------------------------- FFN gate/up with squared ReLU

size_t bitlinear_forward_relu2_glu_workspace_bytes(int32_t M, int32_t N, int32_t K, uint32_t flags) {
  if (M < 1 || K < 1 || N < 1) return 0;
  // the two BitLinear outputs, then the forward's own workspace (none for the fused one-token kernel)
  return 2 * align256(static_cast<size_t>(M) * N * 2) + bitlinear_forward_workspace_bytes(M, N, K, flags);
}

bitlinear_status bitlinear_forward_relu2_glu(const bitlinear_weights* w_gate, const bitlinear_weights* w_up,
                                             const uint16_t* x, int32_t M, uint16_t* h, void* workspace,
                                             size_t workspace_bytes, uint32_t flags, void* stream) {
  if (!w_gate || !w_up || !x || !h) return BITLINEAR_ERR_NULL;
  bitlinear_status st = check_matrix(w_gate, h, nullptr);
  if (st != BITLINEAR_OK) return st;
  st = check_matrix(w_up, h, nullptr);
  if (st != BITLINEAR_OK) return st;
  if (w_gate->N != w_up->N || w_gate->K != w_up->K) return BITLINEAR_ERR_SHAPE;
  if (M < 1 || M > BITLINEAR_MAX_M) return BITLINEAR_ERR_SHAPE;
  if (!aligned16(x)) return BITLINEAR_ERR_ALIGN;
  st = check_flags(flags, M);
  if (st != BITLINEAR_OK) return st;
  if (flags & BITLINEAR_FLAG_DECODE_LUT) return BITLINEAR_ERR_FLAGS;
  DeviceState* dev = nullptr;
  st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  const bool pdl = (flags & BITLINEAR_FLAG_PDL) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int N = w_gate->N, K = w_gate->K;
  // one token, dense weights: both BitLinears and h in one launch
  if (M == 1 && !(flags & BITLINEAR_FLAG_PATH_TC) && w_gate->nm_m == 0 && w_up->nm_m == 0) {
    GemvGlu g;
    std::memset(&g, 0, sizeof g);
    g.ld = dense_ld(K);
    g.C = static_cast<int>(g.ld / 16);
    g.K = K;
    g.x = x;
    g.h = h;
    g.alpha_g = w_gate->alpha;
    g.alpha_u = w_up->alpha;
    g.status = dev->status;
    int ctas = 0;
    if (glu_split(N, g.ld, g.C, dev->sm_count, &ctas, &g.rows_box)) {
      g.rows_base = N / ctas;
      g.rows_rem = N % ctas;
      CUtensorMap mg, mu;
      if (!make_map_u8(&mg, w_gate->codes, static_cast<uint64_t>(g.ld), static_cast<uint64_t>(N),
                       static_cast<uint64_t>(g.ld), 128, static_cast<uint32_t>(g.rows_box), 128) ||
          !make_map_u8(&mu, w_up->codes, static_cast<uint64_t>(g.ld), static_cast<uint64_t>(N),
                       static_cast<uint64_t>(g.ld), 128, static_cast<uint32_t>(g.rows_box), 128))
        return BITLINEAR_ERR_CUDA;
      st = launch(gemv_glu_kernel, dim3(ctas), dim3(kGemvThreads), gemv_glu_smem_bytes(g.rows_box, g.ld, g.C), s, pdl,
                  mg, mu, g);
      if (st == BITLINEAR_OK) t_last_kernel = "gemv_m1_relu2_glu";
      return st;
    }
  }
  // otherwise: the two BitLinears as one grouped call into the workspace, then h elementwise
  const size_t yb = align256(static_cast<size_t>(M) * N * 2);
  if (!workspace || !aligned16(workspace) || workspace_bytes < 2 * yb) return BITLINEAR_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  uint16_t* ys[2] = {reinterpret_cast<uint16_t*>(wsb), reinterpret_cast<uint16_t*>(wsb + yb)};
  const bitlinear_weights pair[2] = {*w_gate, *w_up};
  st = forward_group(pair, 2, x, M, ys, nullptr, wsb + 2 * yb, workspace_bytes - 2 * yb, flags, stream);
  if (st != BITLINEAR_OK) return st;
  const size_t count = static_cast<size_t>(M) * N;
  const bool vec = aligned16(h);  // the workspace halves are 256-byte aligned
  const int blocks = static_cast<int>(std::min<size_t>(static_cast<size_t>(4 * dev->sm_count), (count / 8 + 255) / 256 + 1));
  st = launch(relu2_glu_kernel, dim3(blocks), dim3(256), 0, s, true, ys[0], ys[1], h, count, vec);
  if (st == BITLINEAR_OK) t_last_kernel = "relu2_glu";
  return st;
}

size_t bitlinear_forward_q8_workspace_bytes(int32_t M, int32_t N, int32_t K) {
  if (M < 1 || K < 1 || N < 1) return 0;
  const int sm = plan_sm_count();
  return std::max({tc_workspace_q8(M, N, K, 0, sm), tc_workspace_q8(M, N, K, 1, sm), tc_workspace_q8(M, N, K, 2, sm)});
}

bitlinear_status bitlinear_forward_group(const bitlinear_weights* w, int32_t count, const uint16_t* x, int32_t M,
                                         uint16_t* const* y, int32_t* const* acc, void* workspace,
                                         size_t workspace_bytes, uint32_t flags, void* stream) {
  return forward_group(w, count, x, M, y, acc, workspace, workspace_bytes, flags, stream);
}

bitlinear_status bitlinear_forward(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                   int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                   void* stream) {
  return forward_common(w, x, M, y, acc, workspace, workspace_bytes, flags, stream, false);
}

bitlinear_status bitlinear_forward_nm(const bitlinear_weights* w, const uint16_t* x, int32_t M, uint16_t* y,
                                      int32_t* acc, void* workspace, size_t workspace_bytes, uint32_t flags,
                                      void* stream) {
  return forward_common(w, x, M, y, acc, workspace, workspace_bytes, flags, stream, true);
}

bitlinear_status bitlinear_device_status(void* stream, int32_t* code, int32_t clear) {
  if (!code) return BITLINEAR_ERR_NULL;
  DeviceState* dev = nullptr;
  bitlinear_status st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, dev->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  *code = v;
  if (clear) {
    const int32_t z = 0;
    if (cudaMemcpy(dev->status, &z, sizeof z, cudaMemcpyHostToDevice) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  }
  return BITLINEAR_OK;
}

const char* bitlinear_last_kernel(void) { return t_last_kernel.name; }

int32_t bitlinear_layout_version(void) { return BITLINEAR_LAYOUT_VERSION; }

const char* bitlinear_status_string(bitlinear_status s) {
  switch (s) {
    case BITLINEAR_OK: return "ok";
    case BITLINEAR_ERR_NULL: return "null pointer";
    case BITLINEAR_ERR_SHAPE: return "unsupported shape";
    case BITLINEAR_ERR_ALIGN: return "misaligned pointer";
    case BITLINEAR_ERR_PATTERN: return "unsupported N:M pattern";
    case BITLINEAR_ERR_WORKSPACE: return "workspace missing or too small";
    case BITLINEAR_ERR_CUDA: return "CUDA error";
    case BITLINEAR_ERR_DEVICE: return "device is not sm_100";
    case BITLINEAR_ERR_FLAGS: return "bad flags";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation entry point
// Scratch for callers that cannot allocate: one fixed array per device,
// shared by every bitlinear_forward_noalloc call on that device.
namespace bl {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[BITLINEAR_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  The host-side
// name is only a stand-in, so the address is looked up once per device, with
// that device current, and cached.
bitlinear_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BITLINEAR_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BITLINEAR_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BITLINEAR_OK;
}

}  // namespace
}  // namespace bl

extern "C" bitlinear_status bitlinear_forward_noalloc(const bitlinear_weights* w, const uint16_t* x, int32_t M,
                                                      uint16_t* y, int32_t* acc, uint32_t flags, void* stream) {
  if (!w) return BITLINEAR_ERR_NULL;
  if (M >= 1 && bitlinear_forward_workspace_bytes(M, w->N, w->K, flags) > BITLINEAR_NOALLOC_SCRATCH_BYTES)
    return BITLINEAR_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  if (w->N >= 1 && w->K >= 1 && M >= 1) {  // let the shared checks report bad shapes first
    bitlinear_status st = current_device(&dev);
    if (st != BITLINEAR_OK) return st;
  }
  void* scratch = nullptr;
  if (dev) {
    bitlinear_status st = noalloc_scratch(&scratch);
    if (st != BITLINEAR_OK) return st;
  }
  // The quantisation kernel rewrites every scratch byte the GEMM reads, so
  // nothing has to be cleared between calls.
  return forward_common(w, x, M, y, acc, scratch, BITLINEAR_NOALLOC_SCRATCH_BYTES, flags, stream, w->nm_m != 0);
}

#ifdef BITLINEAR_TEST_HOOKS
// ---------------------------------------------------------------- test builds only
#include "../../include/bitlinear_test_hooks.h"

extern "C" bitlinear_status bitlinear_test_set_wait_fault(uint64_t wait_limit_ns, uint32_t extra_tx_bytes) {
  DeviceState* dev = nullptr;
  bitlinear_status st = current_device(&dev);
  if (st != BITLINEAR_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return BITLINEAR_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_test_wait_limit_ns, &wait_limit_ns, sizeof wait_limit_ns) != cudaSuccess ||
      cudaMemcpyToSymbol(g_test_extra_tx, &extra_tx_bytes, sizeof extra_tx_bytes) != cudaSuccess)
    return BITLINEAR_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? BITLINEAR_OK : BITLINEAR_ERR_CUDA;
}

extern "C" int32_t bitlinear_test_timeline(uint64_t* records, int32_t max_records) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  uint32_t seq = 0;
  if (cudaMemcpyFromSymbol(&seq, g_timeline_seq, sizeof seq) != cudaSuccess) return -1;
  const int32_t n = static_cast<int32_t>(std::min<uint32_t>(seq, static_cast<uint32_t>(kTlSlots)));
  if (records && max_records > 0 &&
      cudaMemcpyFromSymbol(records, g_timeline, sizeof(uint64_t) * kTlWords * std::min(n, max_records)) != cudaSuccess)
    return -1;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_timeline_seq, &zero, sizeof zero) != cudaSuccess) return -1;
  return static_cast<int32_t>(seq);
}
#endif
