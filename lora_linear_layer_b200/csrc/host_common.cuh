// host_common.cuh - host-side foundations of the library: limits and
// constants, argument validation helpers, the per-device state (device
// probe, primary-context set-up, tensor-map encoder), the per-thread
// tensor-map cache, kernel attribute set-up and the launch helper (cluster
// shape, programmatic dependent launch, error reporting).
// Part of the single translation unit built from lora_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/lora.h"
#include "common.cuh"

namespace {

using namespace lora;

constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s: far above any legitimate wait
constexpr uint32_t kSmemMax = 232448;             // 227 KB opt-in dynamic shared memory
constexpr uint32_t kSmemPerSM = 233472;           // shared memory per SM (228 KB)
constexpr uint32_t kBwdFlags = LORA_BWD_FP32_GRADS | LORA_BWD_T_SAVED;  // known backward flag bits

// ------------------------------------------------------------ validation ----

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range range_of(const void* p, uint64_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return Range{a, a + bytes};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

lora_status_t check_sizes(int64_t M, int64_t d_in, int64_t d_out, int32_t r) {
  if (M < 0 || d_in <= 0 || d_out <= 0) return LORA_ERR_SHAPE;
  if ((d_in % 8) != 0 || (d_out % 8) != 0) return LORA_ERR_SHAPE;
  if (M > (int64_t(1) << 30) || d_in > (int64_t(1) << 30) || d_out > (int64_t(1) << 30)) return LORA_ERR_SHAPE;
  if (r < 8 || r > 128 || (r % 8) != 0) return LORA_ERR_RANK;
  return LORA_OK;
}

int r_pad_of(int r) { return (r + 15) / 16 * 16; }
int rcw_of(int r_pad) { return r_pad <= 16 ? 16 : r_pad <= 32 ? 32 : 64; }

// ---------------------------------------------------------- device state ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[64];
EncodeTiledFn g_encode = nullptr;

lora_status_t device_info(DeviceInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  // The tensor-map encoder is a driver call and needs a current context.  A
  // thread that has not used the runtime yet (PyTorch's autograd worker, for
  // one) has none: cudaSetDevice makes the device's primary context current.
  thread_local int t_ctx_dev = -1;
  if (t_ctx_dev != dev) {
    if (cudaSetDevice(dev) != cudaSuccess) return LORA_ERR_CUDA;
    t_ctx_dev = dev;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LORA_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.sm_count = sms;
    d.probed = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return LORA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  out = d;
  return d.supported ? LORA_OK : LORA_ERR_UNSUPPORTED_DEVICE;
}

CUtensorMapSwizzle swz_enum(uint32_t span_bytes) {
  return span_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : span_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                            : CU_TENSOR_MAP_SWIZZLE_32B;
}

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows,
// row pitch `ld` elements, box {box_inner, box_outer}.  Encoded maps are
// kept in a per-thread hash table keyed by every encoding input, so a layer
// (or a batched merge of hundreds of matrices) called again on the same
// buffers skips the driver call.  The table is emptied when it reaches
// kMapCache entries.
struct MapKey {
  const void* ptr;
  uint64_t inner, outer, ld;
  uint32_t bi, bo, swz;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && inner == o.inner && outer == o.outer && ld == o.ld && bi == o.bi && bo == o.bo &&
           swz == o.swz;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = reinterpret_cast<uintptr_t>(k.ptr) * 0x9E3779B97F4A7C15ull;
    for (uint64_t v : {k.inner, k.outer, k.ld, uint64_t(k.bi) << 32 | k.bo, uint64_t(k.swz)})
      h = (h ^ v) * 0x100000001B3ull + (h >> 29);
    return size_t(h);
  }
};
constexpr size_t kMapCache = 8192;
thread_local std::unordered_map<MapKey, CUtensorMap, MapKeyHash> t_maps;

bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld, uint32_t box_inner,
              uint32_t box_outer, uint32_t swz_span_bytes) {
  const MapKey k{ptr, inner, outer, ld, box_inner, box_outer, swz_span_bytes};
  const auto it = t_maps.find(k);
  if (it != t_maps.end()) {
    *m = it->second;
    return true;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult rc = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz_enum(swz_span_bytes),
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) {
    std::fprintf(stderr, "lora_b200: cuTensorMapEncodeTiled failed (%d) dims=%llu,%llu box=%u,%u\n", int(rc),
                 (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return false;
  }
  if (t_maps.size() >= kMapCache) t_maps.clear();
  t_maps.emplace(k, *m);
  return true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel, device
// and size (the attribute only grows).
std::mutex g_attr_mu;
std::vector<std::pair<std::pair<const void*, int>, int>> g_attr_done;

template <typename Kern>
bool ensure_smem_attr(Kern kern, uint32_t smem) {
  int dev = 0;
  cudaGetDevice(&dev);
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lk(g_attr_mu);
  for (auto& e : g_attr_done)
    if (e.first.first == fn && e.first.second == dev && e.second >= int(smem)) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return false;
  for (auto& e : g_attr_done)
    if (e.first.first == fn && e.first.second == dev) {
      e.second = int(smem);
      return true;
    }
  g_attr_done.push_back({{fn, dev}, int(smem)});
  return true;
}

lora_status_t launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    std::fprintf(stderr, "lora_b200: launch failed: %s\n", cudaGetErrorString(e));
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

// Programmatic dependent launch (PDL) on every launch unless
// LORA_B200_PDL=0: a kernel's prologue (barrier init, TMEM allocation,
// descriptor prefetch) then overlaps the tail of the kernel before it on the
// stream.  Every kernel waits (griddepcontrol.wait) before its first global
// memory access, so results do not depend on this setting.
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("LORA_B200_PDL");
    return !(e != nullptr && e[0] == '0');
  }();
  return on;
}

// cudaLaunchKernelEx with an optional cluster shape and the PDL attribute.
template <typename... KArgs, typename... Args>
lora_status_t launch_ex(const char* what, void (*kern)(KArgs...), dim3 grid, dim3 block, uint32_t smem,
                        cudaStream_t st, const dim3* cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster != nullptr) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster->x;
    attr[n].val.clusterDim.y = cluster->y;
    attr[n].val.clusterDim.z = cluster->z;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    std::fprintf(stderr, "lora_b200: %s launch failed: %s\n", what, cudaGetErrorString(e));
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace
