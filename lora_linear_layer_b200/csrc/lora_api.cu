// lora_api.cu - the extern "C" entry points declared in include/lora.h.
//
// Host side of the library: argument validation, TMA tensor-map encoding,
// tile / pipeline configuration and kernel launches on the caller's stream.
// All arithmetic of the layer runs in the kernels of fused.cuh, skinny.cuh
// and merge.cuh.
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
#include "fused.cuh"
#include "merge.cuh"
#include "skinny.cuh"
#include "splitk.cuh"

namespace lora {

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(smem_addr(&bar), 0u, &abort_flag, limit_ns, SITE_SELFTEST);
  __syncthreads();
}

}  // namespace lora

namespace {

using namespace lora;

constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s: far above any legitimate wait
constexpr uint32_t kSmemMax = 232448;             // 227 KB opt-in dynamic shared memory
constexpr int kSplitSMs = 148;                    // B200 SM count used to size split-M work
constexpr uint32_t kSmemPerSM = 233472;           // shared memory per SM (228 KB)

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

// ------------------------------------------------------------ fused GEMM ----

struct FusedCfg {
  int BN, CG, RCW, r_pad, n_rchunks, stages, ep_bufs;
  uint32_t smem;
  FusedArgs args;
};

// Pipeline stages that fit in shared memory for (BN, CG), capped at 8.
int fused_stages(int BN, int CG, bool mn, int RCW, int r_pad, int n_rchunks, int ep_bufs) {
  const FusedLayout L0(BN, CG, mn, RCW, r_pad, n_rchunks, 0, ep_bufs);
  const uint32_t fixed = L0.total + 1024;
  if (fixed >= kSmemMax) return 0;
  return std::min(int((kSmemMax - fixed) / L0.stage_bytes), 8);
}

// Optional tile override "BN,CG" from LORA_B200_FUSED_TILE (e.g. "256,1"),
// used to measure or test one configuration; 0,0 = choose per problem.
void tile_override(int& BN, int& CG) {
  BN = 0;
  CG = 0;
  const char* e = std::getenv("LORA_B200_FUSED_TILE");
  if (e == nullptr) return;
  int b = 0, g = 0;
  if (std::sscanf(e, "%d,%d", &b, &g) == 2 && (b == 128 || b == 256) && (g == 1 || g == 2)) {
    BN = b;
    CG = g;
  }
}

// Optional schedule override from LORA_B200_FUSED_RUN (-1 = choose).
int run_override() {
  const char* e = std::getenv("LORA_B200_FUSED_RUN");
  if (e == nullptr) return -1;
  const int v = std::atoi(e);
  return v >= 0 && v <= 4096 ? v : -1;
}

bool pick_fused(int64_t M, int64_t N, int64_t K, int r, bool mn, int sm_count, FusedCfg& c) {
  c.r_pad = r_pad_of(r);
  c.RCW = rcw_of(c.r_pad);
  c.n_rchunks = (c.r_pad + c.RCW - 1) / c.RCW;
  int fBN, fCG;
  tile_override(fBN, fCG);
  // Candidates in order of preference: 256-wide tiles first (least operand
  // traffic per flop); CTA pairs first for long contractions, single CTAs
  // first for K <= 1024 (measured faster there: 8192x512x512 16.4 vs
  // 18.4 us, 4096x1024x1024 21.2 vs 22.6 us).  Take the first that fits in
  // shared memory with tiles for at least 80% of its clusters (fewer,
  // larger tiles beat more, smaller ones: 2048x2048x2048 28.7 us with 64
  // pair tiles of 256 x 256 against 38.9 us with 128 of 256 x 128), else
  // 128-wide single-CTA tiles (128-wide pairs measured slower in every
  // case: 512x4096x4096 43.0 vs 41.0 us).  LORA_B200_FUSED_TILE can still
  // force a 128-wide pair.
  const bool short_k = K <= 1024;
  const int cands[4][2] = {{256, short_k ? 1 : 2}, {256, short_k ? 2 : 1}, {128, 1}, {128, 2}};
  c.BN = 0;
  for (int pass = 0; pass < 2 && c.BN == 0; ++pass) {  // pass 1 ignores an infeasible override
    for (int i = 0; i < 4; ++i) {
      const int BN = cands[i][0], CG = cands[i][1];
      const bool forced = pass == 0 && fBN != 0;
      if (forced && (BN != fBN || CG != fCG)) continue;
      if (!forced && i == 3) break;  // the 128-wide pair only when forced
      const int S = fused_stages(BN, CG, mn, c.RCW, c.r_pad, c.n_rchunks, 1);
      if (S < (BN == 256 ? 3 : 2)) continue;
      const int64_t tiles = ((M + 128 * CG - 1) / (128 * CG)) * ((N + BN - 1) / BN);
      const bool fills = double(tiles) >= 0.8 * double(sm_count / CG);
      if (forced || fills || i == 2) {
        c.BN = BN;
        c.CG = CG;
        c.stages = S;
        break;
      }
    }
  }
  if (c.BN == 0) return false;
  const int num_m = int((M + 128 * c.CG - 1) / (128 * c.CG));
  const int num_n = int((N + c.BN - 1) / c.BN);
  // a second output staging buffer per epilogue warp when it costs no stage
  c.ep_bufs = fused_stages(c.BN, c.CG, mn, c.RCW, c.r_pad, c.n_rchunks, 2) >= c.stages ? 2 : 1;
  const FusedLayout L(c.BN, c.CG, mn, c.RCW, c.r_pad, c.n_rchunks, c.stages, c.ep_bufs);
  c.smem = L.total + 1024;
  FusedArgs& a = c.args;
  a.M = int32_t(M);
  a.N = int32_t(N);
  a.K = int32_t(K);
  a.r_pad = c.r_pad;
  a.n_rchunks = c.n_rchunks;
  a.stages = c.stages;
  a.ep_bufs = c.ep_bufs;
  a.num_m = num_m;
  a.num_n = num_n;
  // Column bands keep the operands the whole GPU touches at once well
  // inside the 126 MB L2 when the full problem is larger than that.
  const double footprint = double(M + N) * double(K) * 2.0;
  if (footprint > 96.0e6) {
    const double per_ntile = double(c.BN) * double(K) * 2.0;
    a.band_w = std::max(1, std::min(num_n, int(40.0e6 / per_ntile)));
    // a band must still hold two tiles per cluster: with few M blocks the
    // operands are not reused across the band anyway
    const int want = int((2 * (sm_count / c.CG) + num_m - 1) / num_m);
    a.band_w = std::max(a.band_w, std::min(num_n, want));
  } else {
    a.band_w = num_n;
  }
  a.n_bands = (num_n + a.band_w - 1) / a.band_w;
  // Runs of L N tiles of one M block, dealt round-robin: the clusters walk
  // the same W tiles at the same time, so the operands they share stay in
  // L2, and T is computed once per run.  L in [2, 8] minimises the modelled
  // makespan ceil(runs / clusters) * (L + 0.5) (a T computation costs about
  // half a tile), over runs that keep at least 80% of the clusters busy;
  // ties go to the longer run (runs of 16 measured no faster than 8).  Without such a run length: contiguous ranges inside
  // column bands.  (Measured, same box: 8192x4096x4096 forward 202.8 ->
  // 192.5 us at L = 8; 16384x4096x14336 forward 1708 -> 1329 us at L = 7.)
  // The dX form computes no T, so single-tile runs: the round-robin order
  // alone keeps the tiles in flight on a few M blocks, and the makespan is
  // ceil(tiles / clusters).  (Measured on 8192x4096x4096 without T products:
  // runs of 8 on 64 clusters 186 us, single tiles on 74 clusters 168 us.)
  const int64_t clusters = sm_count / c.CG;
  int best_l = mn ? 1 : 0;
  double best_cost = 0.0;
  for (int l = 2; !mn && l <= std::min(num_n, 8); ++l) {
    const int64_t runs = int64_t(num_m) * ((num_n + l - 1) / l);
    if (runs * 5 < clusters * 4) continue;
    const double cost = double((runs + clusters - 1) / clusters) * (l + 0.5);
    if (best_l == 0 || cost < best_cost - 1e-9 || (cost < best_cost + 1e-9 && l > best_l)) {
      best_l = l;
      best_cost = cost;
    }
  }
  const int ro = run_override();
  a.run_l = ro >= 0 ? ro : best_l;
  a.wait_limit_ns = kWaitLimitNs;
  return true;
}

struct ClusterCap {
  const void* fn;
  uint32_t smem;
  int dev;
  int clusters;
};
std::mutex g_cap_mu;
std::vector<ClusterCap> g_caps;

// How many clusters of `cg` CTAs of this kernel can be resident at once.
template <typename Kern>
int max_clusters(Kern kern, int cg, uint32_t smem, int sm_count) {
  if (cg == 1) return sm_count;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_cap_mu);
  for (const ClusterCap& cc : g_caps)
    if (cc.fn == (const void*)kern && cc.smem == smem && cc.dev == dev) return cc.clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(sm_count / cg * cg));
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(cg);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count / cg;
  }
  g_caps.push_back(ClusterCap{(const void*)kern, smem, dev, n});
  return n;
}

template <int BN, bool MN, int RCW, int CG>
lora_status_t launch_fused_t(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  auto kern = fused_lora_kernel<BN, MN, RCW, CG>;
  if (!ensure_smem_attr(kern, c.smem)) return LORA_ERR_CUDA;
  const int64_t tiles = int64_t(c.args.num_m) * c.args.num_n;
  const int clusters = int(std::min<int64_t>(tiles, max_clusters(kern, CG, c.smem, sm_count)));
  const dim3 cl(unsigned(CG), 1, 1);
  return launch_ex("fused", kern, dim3(unsigned(clusters * CG)), dim3(kFusedThreads), c.smem, st, &cl, maps[0],
                   maps[1], maps[2], maps[3], maps[4], c.args);
}

template <bool MN, int CG>
lora_status_t launch_fused_cg(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  if constexpr (MN) {  // the dX form has no rank chunks in shared memory
    return c.BN == 256 ? launch_fused_t<256, true, 64, CG>(maps, c, sm_count, st)
                       : launch_fused_t<128, true, 64, CG>(maps, c, sm_count, st);
  }
  if (c.BN == 256) {
    if (c.RCW == 16) return launch_fused_t<256, MN, 16, CG>(maps, c, sm_count, st);
    if (c.RCW == 32) return launch_fused_t<256, MN, 32, CG>(maps, c, sm_count, st);
    return launch_fused_t<256, MN, 64, CG>(maps, c, sm_count, st);
  }
  if (c.RCW == 16) return launch_fused_t<128, MN, 16, CG>(maps, c, sm_count, st);
  if (c.RCW == 32) return launch_fused_t<128, MN, 32, CG>(maps, c, sm_count, st);
  return launch_fused_t<128, MN, 64, CG>(maps, c, sm_count, st);
}

template <bool MN>
lora_status_t launch_fused(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  return c.CG == 2 ? launch_fused_cg<MN, 2>(maps, c, sm_count, st) : launch_fused_cg<MN, 1>(maps, c, sm_count, st);
}

// ------------------------------------------------- split-K fused forward ----

constexpr int kGroupMaxJobs = 40;  // problems per grouped launch (kernel parameter space)

struct SplitkPlan {
  int RCW, r_pad, n_rchunks, stages, splits;
  uint32_t smem;
};

// LORA_B200_SPLITK=0 turns the split-K forward off, =1 uses it whenever it
// applies at all (S >= 2); unset: automatic.  A forced fused tile
// (LORA_B200_FUSED_TILE) also turns it off.
int splitk_mode() {
  const char* e = std::getenv("LORA_B200_SPLITK");
  if (e != nullptr && (e[0] == '0' || e[0] == '1')) return e[0] - '0';
  return std::getenv("LORA_B200_FUSED_TILE") != nullptr ? 0 : -1;
}

// Split count and pipeline depth for a launch of `tiles` 128 x 128 tiles
// whose shortest contraction has `min_nk` K blocks: S CTAs (at most 8, the
// portable cluster size) per tile, as many as fill the SMs, with at least 8
// K blocks each (shorter K loops do not pay for the reduction: measured
// slower at K = 512 and at 4 K blocks per split).  From r_pad = 64 on, whose
// T reduction costs more, contractions under 32 K blocks are not split: at
// r = 64 two splits took 20.5 us on 128 x 1024 x 1024 and 512 x 1024 x 1024
// against 16.4 us for one 128 x 128 tile per CTA (at K = 2048 four splits
// and one tile per CTA tie, 20.5 us, and two splits take 22.6 us).
// With more tiles than SMs (a grouped launch), three stages, so that two
// CTAs fit on an SM.
void plan_splitk(int64_t tiles, int min_nk, int r, int sm_count, SplitkPlan& pl) {
  pl.r_pad = r_pad_of(r);
  pl.RCW = rcw_of(pl.r_pad);
  pl.n_rchunks = (pl.r_pad + pl.RCW - 1) / pl.RCW;
  pl.splits = int(std::max<int64_t>(1, std::min<int64_t>({8, sm_count / std::max<int64_t>(1, tiles), min_nk / 8})));
  if (pl.r_pad >= 64 && min_nk < 32) pl.splits = 1;
  int stages = tiles > sm_count ? 3 : 6;
  while (stages > 1 && SplitkLayout(pl.RCW, pl.r_pad, pl.n_rchunks, stages).total + 1024 > kSmemMax) --stages;
  pl.stages = stages;
  pl.smem = SplitkLayout(pl.RCW, pl.r_pad, pl.n_rchunks, stages).total + 1024;
}

// The single-problem split-K forward is used when 128 x 128 tiles would fill
// at most half of the SMs, S >= 2, and r <= 64 (at r = 128 the T reduction
// costs more than the split saves).
bool use_splitk(int64_t M, int64_t N, int64_t K, int r, int sm_count, SplitkPlan& pl) {
  const int mode = splitk_mode();
  if (mode == 0) return false;
  const int64_t tiles = ((M + 127) / 128) * ((N + 127) / 128);
  if (tiles > 65535) return false;
  if (mode < 0 && (tiles * 2 > sm_count || r_pad_of(r) > 64)) return false;
  plan_splitk(tiles, int((K + 63) / 64), r, sm_count, pl);
  return pl.splits >= 2;
}

// Fill one job of a split-K table (the caller validated the arguments).
bool splitk_job(SplitkJob& j, const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                int64_t d_in, int64_t d_out, int32_t r, const SplitkPlan& pl, int tile_begin) {
  if (!make_map(&j.p, X, d_in, M, d_in, 64, 128, 128) || !make_map(&j.q, W, d_in, d_out, d_in, 64, 128, 128) ||
      !make_map(&j.u, A, d_in, r, d_in, 64, uint32_t(pl.r_pad), 128) ||
      !make_map(&j.v, B, r, d_out, r, pl.RCW, 128, pl.RCW * 2))
    return false;
  j.M = int32_t(M);
  j.N = int32_t(d_out);
  j.K = int32_t(d_in);
  j.num_n = int32_t((d_out + 127) / 128);
  j.tile_begin = tile_begin;
  const int nk = int((d_in + 63) / 64);
  j.kb_per_split = (nk + pl.splits - 1) / pl.splits;
  j.out = reinterpret_cast<__nv_bfloat16*>(Y);
  return true;
}

template <int NJ>
void splitk_table_common(SplitkTable<NJ>& t, int n_jobs, const SplitkPlan& pl, float scale) {
  t.n_jobs = n_jobs;
  t.r_pad = pl.r_pad;
  t.n_rchunks = pl.n_rchunks;
  t.stages = pl.stages;
  t.splits = pl.splits;
  t.scale = scale;
  t.wait_limit_ns = kWaitLimitNs;
}

template <int RCW, int NJ>
lora_status_t launch_splitk_t(const SplitkTable<NJ>& t, int tiles, const SplitkPlan& pl, cudaStream_t st) {
  auto kern = fused_splitk_kernel<RCW, NJ>;
  if (!ensure_smem_attr(kern, pl.smem)) return LORA_ERR_CUDA;
  const dim3 cl(unsigned(pl.splits), 1, 1);
  return launch_ex("split-K forward", kern, dim3(unsigned(pl.splits), unsigned(tiles)), dim3(192), pl.smem, st, &cl,
                   t);
}

template <int NJ>
lora_status_t launch_splitk(const SplitkTable<NJ>& t, int tiles, const SplitkPlan& pl, cudaStream_t st) {
  if (pl.RCW == 16) return launch_splitk_t<16, NJ>(t, tiles, pl, st);
  if (pl.RCW == 32) return launch_splitk_t<32, NJ>(t, tiles, pl, st);
  return launch_splitk_t<64, NJ>(t, tiles, pl, st);
}

// ----------------------------------------------------------- skinny GEMM ----

struct SkinnyCfg {
  int RCW, r_pad, n_rchunks, stages, splits;
  uint32_t smem;
  SkinnyArgs args;
};

// Split the contraction so that about two CTAs per SM run; the splits of a
// row tile form one cluster (at most 8, the portable cluster size), and
// every split keeps at least 4 K blocks.
// `launch_tiles` is the number of 128-row tiles of the whole launch (both
// jobs when dB and dA share one), which sets the split count: as many
// splits as keep every resident CTA slot of the GPU busy, at most 8 (the
// portable cluster size) and at least 4 K blocks per split.
void pick_skinny(int64_t rows, int64_t K, int r, bool r_mn, int out_mode, int64_t launch_tiles, SkinnyCfg& c) {
  c.r_pad = r_pad_of(r);
  c.RCW = rcw_of(c.r_pad);
  c.n_rchunks = (c.r_pad + c.RCW - 1) / c.RCW;
  c.stages = 4;
  const SkinnyLayout L(r_mn, c.RCW, c.r_pad, c.n_rchunks, c.stages);
  c.smem = L.total + 1024;
  const int per_sm = std::max(1, std::min<int>(int(kSmemPerSM / (c.smem + 1024)),
                                               int(512 / tmem_cols_for(c.r_pad))));
  const int slots = per_sm * kSplitSMs;
  const int tiles = int(std::max<int64_t>(1, launch_tiles));
  const int nk = int((K + 63) / 64);
  int splits = std::max(1, std::min({slots / tiles, 8, std::max(1, nk / 4)}));
  const int kb_per = std::max(1, (nk + splits - 1) / splits);
  splits = std::max(1, (nk + kb_per - 1) / kb_per);
  c.splits = splits;
  SkinnyArgs& a = c.args;
  std::memset(&a, 0, sizeof(a));
  a.rows = int32_t(rows);
  a.K = int32_t(K);
  a.r_pad = c.r_pad;
  a.r = r;
  a.n_rchunks = c.n_rchunks;
  a.stages = c.stages;
  a.kb_per_split = kb_per;
  a.splits = splits;
  a.out_mode = out_mode;
  a.r_mn = r_mn ? 1 : 0;
  a.scale = 1.0f;
  a.wait_limit_ns = kWaitLimitNs;
}

// Re-split a job's contraction into exactly `splits` ranges (a launch's
// two jobs share one cluster shape); trailing ranges may be empty.
void resplit_skinny(SkinnyCfg& c, int splits) {
  const int nk = int((int64_t(c.args.K) + 63) / 64);
  c.splits = splits;
  c.args.splits = splits;
  c.args.kb_per_split = std::max(1, (nk + splits - 1) / splits);
}

// One launch of one job (c1 == nullptr) or of two jobs with the same P
// layout, RCW and split count; the launch takes the larger shared-memory
// size of the two.
template <bool P_MN, int RCW>
lora_status_t launch_skinny_t(const CUtensorMap& p0, const CUtensorMap& r0, const SkinnyCfg& c0,
                              const CUtensorMap* p1, const CUtensorMap* r1, const SkinnyCfg* c1, cudaStream_t st) {
  auto kern = skinny_kernel<P_MN, RCW>;
  const uint32_t smem = c1 != nullptr ? std::max(c0.smem, c1->smem) : c0.smem;
  if (!ensure_smem_attr(kern, smem)) return LORA_ERR_CUDA;
  const int t0 = (c0.args.rows + 127) / 128;
  const int t1 = c1 != nullptr ? (c1->args.rows + 127) / 128 : 0;
  const dim3 cl(1, unsigned(c0.splits), 1);
  return launch_ex("skinny", kern, dim3(unsigned(t0 + t1), unsigned(c0.splits)), dim3(192), smem, st, &cl, p0, r0,
                   p1 != nullptr ? *p1 : p0, r1 != nullptr ? *r1 : r0, c0.args, c1 != nullptr ? c1->args : c0.args,
                   int32_t(t0));
}

template <bool P_MN>
lora_status_t launch_skinny(const CUtensorMap& p0, const CUtensorMap& r0, const SkinnyCfg& c0, cudaStream_t st,
                            const CUtensorMap* p1 = nullptr, const CUtensorMap* r1 = nullptr,
                            const SkinnyCfg* c1 = nullptr) {
  if (c0.RCW == 16) return launch_skinny_t<P_MN, 16>(p0, r0, c0, p1, r1, c1, st);
  if (c0.RCW == 32) return launch_skinny_t<P_MN, 32>(p0, r0, c0, p1, r1, c1, st);
  return launch_skinny_t<P_MN, 64>(p0, r0, c0, p1, r1, c1, st);
}

// --------------------------------------------------------- bwd workspace ----

struct BwdPlan {
  SkinnyCfg dt_cfg, t_cfg, db_cfg, da_cfg;
  size_t off_t, off_dt, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

void plan_bwd(int64_t M, int64_t d_in, int64_t d_out, int32_t r, BwdPlan& p) {
  // dT (contraction d_out) and T (contraction d_in) share the first launch
  // and its split count, which the longer contraction sets for the row
  // tiles of both jobs; the longer job goes first in the grid
  const int64_t both_tiles = 2 * ((M + 127) / 128);
  pick_skinny(M, d_out, r, true, OUT_ROWS_RPAD, both_tiles, p.dt_cfg);
  pick_skinny(M, d_in, r, false, OUT_ROWS_RPAD, both_tiles, p.t_cfg);
  const int s1 = d_out >= d_in ? p.dt_cfg.splits : p.t_cfg.splits;
  resplit_skinny(p.dt_cfg, s1);
  resplit_skinny(p.t_cfg, s1);
  // dB and dA share one launch, so they share its split count
  const int64_t dbda_tiles = (d_out + 127) / 128 + (d_in + 127) / 128;
  pick_skinny(d_out, M, r, true, OUT_ROWS_R, dbda_tiles, p.db_cfg);
  pick_skinny(d_in, M, r, true, OUT_COLS_R, dbda_tiles, p.da_cfg);
  const int r_pad = r_pad_of(r);
  const size_t tb = align256(size_t(M) * r_pad * 2);
  p.off_t = 0;                                         // T   bf16 [M, r_pad]
  p.off_dt = tb;                                       // dT  bf16 [M, r_pad]
  p.total = 2 * tb;
}

// -------------------------------------------------------- merge batching ----

struct MergeItem {
  const void* W_src;
  const void* A;
  const void* B;
  void* W_dst;
  int64_t d_out, d_in;
};

lora_status_t check_merge_item(const MergeItem& it, int32_t r) {
  if (!it.W_src || !it.A || !it.B || !it.W_dst) return LORA_ERR_NULL;
  lora_status_t s = check_sizes(0, it.d_in, it.d_out, r);
  if (s != LORA_OK) return s;
  if (!aligned16(it.W_src) || !aligned16(it.A) || !aligned16(it.B) || !aligned16(it.W_dst)) return LORA_ERR_ALIGN;
  const Range dst = range_of(it.W_dst, uint64_t(it.d_out) * it.d_in * 2);
  if (overlaps(dst, range_of(it.A, uint64_t(r) * it.d_in * 2)) ||
      overlaps(dst, range_of(it.B, uint64_t(it.d_out) * r * 2)))
    return LORA_ERR_ALIAS;
  if (it.W_dst != it.W_src && overlaps(dst, range_of(it.W_src, uint64_t(it.d_out) * it.d_in * 2)))
    return LORA_ERR_ALIAS;
  return LORA_OK;
}

// `per_sm` persistent CTAs per SM (at most one per tile).
template <int RCW>
lora_status_t launch_merge_t(const MergeTable& tab, int sm_count, int per_sm, uint32_t smem, cudaStream_t st) {
  auto kern = merge_kernel<RCW>;
  if (!ensure_smem_attr(kern, smem)) return LORA_ERR_CUDA;
  const int grid = std::max(1, std::min(tab.n_tiles, per_sm * sm_count));
  return launch_ex("merge", kern, dim3(unsigned(grid)), dim3(kMergeThreads), smem, st, nullptr, tab);
}

lora_status_t run_merge(const MergeItem* items, int n, int32_t r, float alpha, int sm_count, cudaStream_t st) {
  if (n <= 0) return LORA_OK;
  const int r_pad = r_pad_of(r);
  const int rcw = rcw_of(r_pad);
  const int n_rchunks = (r_pad + rcw - 1) / rcw;
  // One CTA per SM with as many stages as fit, at most kMergeMaxStages, and
  // at least two: a stage is given back one tile after its store is issued.
  // (Two CTAs per SM with two stages each measured slower: 4.2 vs 3.2 ms on
  // the 252-matrix refresh.)
  const MergeLayout L0(rcw, r_pad, n_rchunks, 0);
  const int per_sm = 1;
  const int stages = std::min<int>(kMergeMaxStages, int((kSmemMax - L0.total - 1024) / L0.stage_bytes));
  if (stages < 2) return LORA_ERR_RANK;
  const MergeLayout L(rcw, r_pad, n_rchunks, stages);
  const uint32_t smem = L.total + 1024;
  static thread_local MergeTable tab;  // ~28 KB, kept off the stack
  int i = 0;
  while (i < n) {
    std::memset(&tab, 0, sizeof(tab));
    tab.r_pad = r_pad;
    tab.n_rchunks = n_rchunks;
    tab.stages = stages;
    tab.scale = alpha / float(r);
    tab.wait_limit_ns = kWaitLimitNs;
    int tiles = 0, nj = 0;
    for (; i < n && nj < kMergeMaxJobs; ++i) {
      const MergeItem& it = items[i];
      MergeJob& j = tab.job[nj];
      if (!make_map(&j.w_src, it.W_src, it.d_in, it.d_out, it.d_in, 64, 128, 128) ||
          !make_map(&j.w_dst, it.W_dst, it.d_in, it.d_out, it.d_in, 64, 32, 128) ||
          !make_map(&j.a, it.A, it.d_in, r, it.d_in, 64, r_pad, 128) ||
          !make_map(&j.b, it.B, r, it.d_out, r, rcw, 128, rcw * 2))
        return LORA_ERR_CUDA;
      j.tiles_n = int32_t((it.d_in + kMergeBN - 1) / kMergeBN);
      j.tile_begin = tiles;
      j.rows = int32_t(it.d_out);
      j.cols = int32_t(it.d_in);
      tiles += j.tiles_n * int32_t((it.d_out + 127) / 128);
      ++nj;
    }
    tab.n_jobs = nj;
    tab.n_tiles = tiles;
    lora_status_t s = rcw == 16 ? launch_merge_t<16>(tab, sm_count, per_sm, smem, st)
                      : rcw == 32 ? launch_merge_t<32>(tab, sm_count, per_sm, smem, st)
                                  : launch_merge_t<64>(tab, sm_count, per_sm, smem, st);
    if (s != LORA_OK) return s;
  }
  return LORA_OK;
}

lora_status_t zero_bytes(void* p, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return LORA_OK;
  if ((bytes % 16) != 0 || !aligned16(p)) return LORA_ERR_ALIGN;
  const size_t n16 = bytes / 16;
  const int blocks = int(std::min<size_t>((n16 + 255) / 256, 4096));
  return launch_ex("zero", zero16_kernel, dim3(unsigned(blocks)), dim3(256), 0, st, nullptr,
                   reinterpret_cast<uint4*>(p), n16);
}

}  // namespace

// ================================================================ C ABI ====

extern "C" {

int lora_abi_version(void) { return LORA_ABI_VERSION; }

const char* lora_status_string(lora_status_t s) {
  switch (s) {
    case LORA_OK: return "LORA_OK";
    case LORA_ERR_NULL: return "LORA_ERR_NULL: a required pointer is NULL";
    case LORA_ERR_SHAPE: return "LORA_ERR_SHAPE: bad size (d_in, d_out must be positive multiples of 8)";
    case LORA_ERR_ALIGN: return "LORA_ERR_ALIGN: pointer not 16-byte aligned";
    case LORA_ERR_RANK: return "LORA_ERR_RANK: r must be a multiple of 8 in [8, 128]";
    case LORA_ERR_WORKSPACE: return "LORA_ERR_WORKSPACE: workspace missing or too small";
    case LORA_ERR_CUDA: return "LORA_ERR_CUDA: a CUDA call failed";
    case LORA_ERR_TIMEOUT: return "LORA_ERR_TIMEOUT: a kernel gave up on a bounded wait";
    case LORA_ERR_UNSUPPORTED_DEVICE: return "LORA_ERR_UNSUPPORTED_DEVICE: needs an sm_100 (B200) device";
    case LORA_ERR_ALIAS: return "LORA_ERR_ALIAS: an output overlaps an input";
    case LORA_ERR_FLAGS: return "LORA_ERR_FLAGS: unknown bit in a flags argument";
  }
  return "LORA_ERR_UNKNOWN";
}

static lora_status_t check_bwd_args(const void* const* ptrs, int32_t n_ptrs, int64_t M, int64_t d_in, int64_t d_out,
                                    int32_t r, size_t workspace_bytes, size_t need, int grad_bytes = 2);

lora_status_t lora_check_args(int32_t op, const void* const* ptrs, int32_t n_ptrs, int64_t M, int64_t d_in,
                              int64_t d_out, int32_t r, size_t workspace_bytes) {
  if (op == 0) {
    // X and Y may be NULL only when M == 0 (nothing is read or written).
    if (ptrs == nullptr || n_ptrs != 5) return LORA_ERR_NULL;
    for (int i = 0; i < 5; ++i) {
      const bool needed = (i >= 1 && i <= 3) || M != 0;
      if (needed && ptrs[i] == nullptr) return LORA_ERR_NULL;
    }
    lora_status_t s = check_sizes(M, d_in, d_out, r);
    if (s != LORA_OK) return s;
    for (int i = 0; i < 5; ++i)
      if (!aligned16(ptrs[i])) return LORA_ERR_ALIGN;
    const Range y = range_of(ptrs[4], uint64_t(M) * d_out * 2);
    if (overlaps(y, range_of(ptrs[0], uint64_t(M) * d_in * 2)) ||
        overlaps(y, range_of(ptrs[1], uint64_t(d_out) * d_in * 2)) ||
        overlaps(y, range_of(ptrs[2], uint64_t(r) * d_in * 2)) ||
        overlaps(y, range_of(ptrs[3], uint64_t(d_out) * r * 2)))
      return LORA_ERR_ALIAS;
    return LORA_OK;
  }
  if (op == 1) return check_bwd_args(ptrs, n_ptrs, M, d_in, d_out, r, workspace_bytes,
                                     lora_bwd_workspace_size(M, d_in, d_out, r), 2);
  if (op == 2) {
    if (ptrs == nullptr || n_ptrs != 4) return LORA_ERR_NULL;
    MergeItem it{ptrs[0], ptrs[1], ptrs[2], const_cast<void*>(ptrs[3]), d_out, d_in};
    return check_merge_item(it, r);
  }
  return LORA_ERR_SHAPE;
}

// The backward's argument rules with `need` bytes of workspace required and
// dA, dB of `grad_bytes` per element.
static lora_status_t check_bwd_args(const void* const* ptrs, int32_t n_ptrs, int64_t M, int64_t d_in, int64_t d_out,
                                    int32_t r, size_t workspace_bytes, size_t need, int grad_bytes) {
  {
    // X, dY, dX (and the workspace) may be NULL only when M == 0; dA and dB
    // are always written (zeros when M == 0).
    if (ptrs == nullptr || n_ptrs != 9) return LORA_ERR_NULL;
    for (int i = 0; i < 8; ++i) {
      const bool needed = (i >= 1 && i <= 3) || i == 6 || i == 7 || M != 0;
      if (needed && ptrs[i] == nullptr) return LORA_ERR_NULL;
    }
    lora_status_t s = check_sizes(M, d_in, d_out, r);
    if (s != LORA_OK) return s;
    for (int i = 0; i < 8; ++i)
      if (!aligned16(ptrs[i])) return LORA_ERR_ALIGN;
    if (M > 0) {
      if (ptrs[8] == nullptr || workspace_bytes < need) return LORA_ERR_WORKSPACE;
      if ((reinterpret_cast<uintptr_t>(ptrs[8]) & 255u) != 0) return LORA_ERR_ALIGN;
    }
    const Range in[5] = {range_of(ptrs[0], uint64_t(M) * d_in * 2), range_of(ptrs[1], uint64_t(d_out) * d_in * 2),
                         range_of(ptrs[2], uint64_t(r) * d_in * 2), range_of(ptrs[3], uint64_t(d_out) * r * 2),
                         range_of(ptrs[4], uint64_t(M) * d_out * 2)};
    const Range out[4] = {range_of(ptrs[5], uint64_t(M) * d_in * 2),
                          range_of(ptrs[6], uint64_t(r) * d_in * uint64_t(grad_bytes)),
                          range_of(ptrs[7], uint64_t(d_out) * r * uint64_t(grad_bytes)), range_of(ptrs[8], need)};
    for (int o = 0; o < 4; ++o) {
      for (int i = 0; i < 5; ++i)
        if (overlaps(out[o], in[i])) return LORA_ERR_ALIAS;
      for (int o2 = o + 1; o2 < 4; ++o2)
        if (overlaps(out[o], out[o2])) return LORA_ERR_ALIAS;
    }
    return LORA_OK;
  }
}

lora_status_t lora_fwd(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                       int64_t d_in, int64_t d_out, int32_t r, float alpha, void* stream) {
  const void* ptrs[5] = {X, W, A, B, Y};
  lora_status_t s = lora_check_args(0, ptrs, 5, M, d_in, d_out, r, 0);
  if (s != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  if (M == 0) return LORA_OK;
  {
    SplitkPlan pl;
    if (use_splitk(M, d_out, d_in, r, dev.sm_count, pl)) {
      SplitkTable<1> t;
      std::memset(&t, 0, sizeof(t));
      splitk_table_common(t, 1, pl, alpha / float(r));
      if (!splitk_job(t.job[0], X, W, A, B, Y, M, d_in, d_out, r, pl, 0)) return LORA_ERR_CUDA;
      const int tiles = int(((M + 127) / 128) * ((d_out + 127) / 128));
      return launch_splitk(t, tiles, pl, reinterpret_cast<cudaStream_t>(stream));
    }
  }
  FusedCfg c;
  if (!pick_fused(M, d_out, d_in, r, false, dev.sm_count, c)) return LORA_ERR_RANK;
  c.args.scale = alpha / float(r);
  c.args.out = reinterpret_cast<__nv_bfloat16*>(Y);
  CUtensorMap maps[5];
  const uint32_t bnc = uint32_t(c.BN / c.CG);
  if (!make_map(&maps[0], X, d_in, M, d_in, 64, 128, 128) ||
      !make_map(&maps[1], W, d_in, d_out, d_in, 64, bnc, 128) ||
      !make_map(&maps[2], A, d_in, r, d_in, 64, uint32_t(c.r_pad / c.CG), 128) ||
      !make_map(&maps[3], B, r, d_out, r, c.RCW, bnc, c.RCW * 2) ||
      !make_map(&maps[4], Y, d_out, M, d_out, kEpCols, 32, kEpCols * 2))
    return LORA_ERR_CUDA;
  return launch_fused<false>(maps, c, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_fwd_batched(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float alpha, void* stream) {
  if (n < 0) return LORA_ERR_SHAPE;
  if (n == 0) return LORA_OK;
  if (descs == nullptr) return LORA_ERR_NULL;
  for (int32_t i = 0; i < n; ++i) {
    const lora_fwd_desc_t& d = descs[i];
    const void* ptrs[5] = {d.X, d.W, d.A, d.B, d.Y};
    const lora_status_t s = lora_check_args(0, ptrs, 5, d.M, d.d_in, d.d_out, r, 0);
    if (s != LORA_OK) return s;
  }
  // no problem's output may overlap another problem's inputs or output
  for (int32_t i = 0; i < n; ++i) {
    const lora_fwd_desc_t& di = descs[i];
    if (di.M == 0) continue;
    const Range yi = range_of(di.Y, uint64_t(di.M) * di.d_out * 2);
    for (int32_t j = 0; j < n; ++j) {
      if (j == i) continue;
      const lora_fwd_desc_t& dj = descs[j];
      if (overlaps(yi, range_of(dj.X, uint64_t(dj.M) * dj.d_in * 2)) ||
          overlaps(yi, range_of(dj.W, uint64_t(dj.d_out) * dj.d_in * 2)) ||
          overlaps(yi, range_of(dj.A, uint64_t(r) * dj.d_in * 2)) ||
          overlaps(yi, range_of(dj.B, uint64_t(dj.d_out) * r * 2)) ||
          overlaps(yi, range_of(dj.Y, uint64_t(dj.M) * dj.d_out * 2)))
        return LORA_ERR_ALIAS;
    }
  }
  DeviceInfo dev;
  lora_status_t s = device_info(dev);
  if (s != LORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // A problem with at least four 128 x 128 tiles per SM runs through lora_fwd
  // (the CTA-pair kernel); the others share grouped split-K launches (two
  // CTAs per SM), longest contraction first so that the long tiles start in
  // the first wave.  (The seven targets of a hidden-2560 layer, CUDA-graph
  // replay, grouped vs separate lora_fwd calls: M = 256 94 vs 166 us,
  // M = 1024 ~260 vs 403 us, M = 2048 385 vs 436 us, M = 4096 698 vs 717 us.)
  std::vector<int32_t> group;
  for (int32_t i = 0; i < n; ++i) {
    const lora_fwd_desc_t& d = descs[i];
    if (d.M == 0) continue;
    const int64_t tj = ((d.M + 127) / 128) * ((d.d_out + 127) / 128);
    if (tj >= 4 * int64_t(dev.sm_count) || tj > 65535) {
      if ((s = lora_fwd(d.X, d.W, d.A, d.B, d.Y, d.M, d.d_in, d.d_out, r, alpha, stream)) != LORA_OK) return s;
    } else {
      group.push_back(i);
    }
  }
  std::stable_sort(group.begin(), group.end(),
                   [&](int32_t x, int32_t y) { return descs[x].d_in > descs[y].d_in; });
  static thread_local SplitkTable<kGroupMaxJobs> t;  // ~23 KB, kept off the stack
  size_t g = 0;
  while (g < group.size()) {
    // one launch: up to kGroupMaxJobs problems and 65535 tiles
    size_t end = g;
    int64_t tiles = 0;
    int min_nk = 1 << 30;
    while (end < group.size() && end - g < size_t(kGroupMaxJobs)) {
      const lora_fwd_desc_t& d = descs[group[end]];
      const int64_t tj = ((d.M + 127) / 128) * ((d.d_out + 127) / 128);
      if (tiles + tj > 65535) break;
      tiles += tj;
      min_nk = std::min(min_nk, int((d.d_in + 63) / 64));
      ++end;
    }
    SplitkPlan pl;
    plan_splitk(tiles, min_nk, r, dev.sm_count, pl);
    std::memset(&t, 0, sizeof(t));
    int nj = 0, tb = 0;
    for (size_t k = g; k < end; ++k) {
      const lora_fwd_desc_t& d = descs[group[k]];
      if (!splitk_job(t.job[nj], d.X, d.W, d.A, d.B, d.Y, d.M, d.d_in, d.d_out, r, pl, tb)) return LORA_ERR_CUDA;
      tb += int(((d.M + 127) / 128) * ((d.d_out + 127) / 128));
      ++nj;
    }
    splitk_table_common(t, nj, pl, alpha / float(r));
    if ((s = launch_splitk(t, tb, pl, st)) != LORA_OK) return s;
    g = end;
  }
  return LORA_OK;
}

size_t lora_bwd_workspace_size(int64_t M, int64_t d_in, int64_t d_out, int32_t r) {
  if (check_sizes(M, d_in, d_out, r) != LORA_OK || M == 0) return 0;
  BwdPlan p;
  plan_bwd(M, d_in, d_out, r, p);
  return p.total;
}

// Launches 1 and 2 of the backward: T and dT into the workspace, then dA and
// dB.  Arguments already validated, M > 0.
static lora_status_t launch_bwd_grads(const void* X, const void* A, const void* B, const void* dY, void* dA,
                                      void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                                      void* workspace, bool f32, cudaStream_t st) {
  BwdPlan p;
  plan_bwd(M, d_in, d_out, r, p);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* Tws = reinterpret_cast<__nv_bfloat16*>(ws + p.off_t);
  __nv_bfloat16* dTws = reinterpret_cast<__nv_bfloat16*>(ws + p.off_dt);
  const float scale = alpha / float(r);
  const int r_pad = r_pad_of(r);
  const int rcw = rcw_of(r_pad);
  lora_status_t s = LORA_OK;

  // 1. One launch, two jobs: dT = s dY B and T = X A^T (recomputed), each
  //    bf16 [M, r_pad] with zero columns past r.  The longer contraction's
  //    job takes the first row tiles of the grid, so it starts first.
  {
    CUtensorMap mp_dt, mr_dt, mp_t, mr_t;
    if (!make_map(&mp_dt, dY, d_out, M, d_out, 64, 128, 128) ||
        !make_map(&mr_dt, B, r, d_out, r, rcw, 64, rcw * 2) ||
        !make_map(&mp_t, X, d_in, M, d_in, 64, 128, 128) || !make_map(&mr_t, A, d_in, r, d_in, 64, r_pad, 128))
      return LORA_ERR_CUDA;
    SkinnyCfg cdt = p.dt_cfg;
    cdt.args.out = dTws;
    cdt.args.scale = scale;
    SkinnyCfg ct = p.t_cfg;
    ct.args.out = Tws;
    s = d_out >= d_in ? launch_skinny<false>(mp_dt, mr_dt, cdt, st, &mp_t, &mr_t, &ct)
                      : launch_skinny<false>(mp_t, mr_t, ct, st, &mp_dt, &mr_dt, &cdt);
    if (s != LORA_OK) return s;
  }
  // 2. One launch:  dB = s * sum_m dY[m, i] T[m, j]  and
  //                     dA^T[i, j] = sum_m X[m, i] dT[m, j], written transposed into dA
  {
    CUtensorMap mp_b, mr_b, mp_a, mr_a;
    if (!make_map(&mp_b, dY, d_out, M, d_out, 64, 64, 128) ||
        !make_map(&mr_b, Tws, r_pad, M, r_pad, rcw, 64, rcw * 2) ||
        !make_map(&mp_a, X, d_in, M, d_in, 64, 64, 128) ||
        !make_map(&mr_a, dTws, r_pad, M, r_pad, rcw, 64, rcw * 2))
      return LORA_ERR_CUDA;
    SkinnyCfg cb = p.db_cfg;
    cb.args.out = reinterpret_cast<__nv_bfloat16*>(dB);
    cb.args.scale = scale;
    cb.args.out_f32 = f32 ? 1 : 0;
    SkinnyCfg ca = p.da_cfg;
    ca.args.out = reinterpret_cast<__nv_bfloat16*>(dA);
    ca.args.out_f32 = f32 ? 1 : 0;
    if ((s = launch_skinny<true>(mp_b, mr_b, cb, st, &mp_a, &mr_a, &ca)) != LORA_OK) return s;
  }
  return LORA_OK;
}

// Launch 3 of the backward: dX from dY, W, A and the workspace's dT.
// Arguments already validated, M > 0.
static lora_status_t launch_bwd_dx(const void* W, const void* A, const void* dY, void* dX, int64_t M, int64_t d_in,
                                   int64_t d_out, int32_t r, const void* workspace, int sm_count, cudaStream_t st) {
  BwdPlan p;
  plan_bwd(M, d_in, d_out, r, p);
  const __nv_bfloat16* dTws =
      reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const uint8_t*>(workspace) + p.off_dt);
  const int r_pad = r_pad_of(r);
  lora_status_t s = LORA_OK;
  // 3. dX = dY W + dT A: one GEMM over the contraction [d_out | r_pad]
  {
    FusedCfg c;
    if (!pick_fused(M, d_in, d_out, r, true, sm_count, c)) return LORA_ERR_RANK;
    c.args.scale = 1.0f;
    c.args.out = reinterpret_cast<__nv_bfloat16*>(dX);
    CUtensorMap maps[5];
    if (!make_map(&maps[0], dY, d_out, M, d_out, 64, 128, 128) ||
        !make_map(&maps[1], W, d_in, d_out, d_in, 64, 64, 128) ||
        !make_map(&maps[2], dTws, r_pad, M, r_pad, 64, 128, 128) ||
        !make_map(&maps[3], A, d_in, r, d_in, 64, 64, 128) ||
        !make_map(&maps[4], dX, d_in, M, d_in, kEpCols, 32, kEpCols * 2))
      return LORA_ERR_CUDA;
    if ((s = launch_fused<true>(maps, c, sm_count, st)) != LORA_OK) return s;
  }
  return LORA_OK;
}

// The backward, with `need` bytes of workspace required; `flags` as in
// lora_bwd_ex.
static lora_status_t bwd_run(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                             void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                             void* workspace, size_t workspace_bytes, size_t need, uint32_t flags, void* stream) {
  if ((flags & ~LORA_BWD_FP32_GRADS) != 0u) return LORA_ERR_FLAGS;
  const bool f32 = (flags & LORA_BWD_FP32_GRADS) != 0u;
  const int gb = f32 ? 4 : 2;  // bytes per dA / dB element
  const void* ptrs[9] = {X, W, A, B, dY, dX, dA, dB, workspace};
  lora_status_t s = check_bwd_args(ptrs, 9, M, d_in, d_out, r, workspace_bytes, need, gb);
  if (s != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0) {
    if ((s = zero_bytes(dA, size_t(r) * d_in * gb, st)) != LORA_OK) return s;
    return zero_bytes(dB, size_t(d_out) * r * gb, st);
  }
  if ((s = launch_bwd_grads(X, A, B, dY, dA, dB, M, d_in, d_out, r, alpha, workspace, f32, st)) != LORA_OK) return s;
  return launch_bwd_dx(W, A, dY, dX, M, d_in, d_out, r, workspace, dev.sm_count, st);
}

lora_status_t lora_bwd(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                       void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                 lora_bwd_workspace_size(M, d_in, d_out, r), 0u, stream);
}

// Pointer rules of the two-call backward: `required` buffers are non-null,
// every non-null buffer is 16-byte aligned, no output overlaps an input or
// another output.
struct BufSpec {
  const void* p;
  uint64_t bytes;
  bool required;
};

static lora_status_t check_bufs(const BufSpec* in, int n_in, const BufSpec* out, int n_out) {
  for (int pass = 0; pass < 2; ++pass) {
    const BufSpec* b = pass == 0 ? in : out;
    const int n = pass == 0 ? n_in : n_out;
    for (int i = 0; i < n; ++i) {
      if (b[i].required && b[i].p == nullptr) return LORA_ERR_NULL;
      if (b[i].p != nullptr && !aligned16(b[i].p)) return LORA_ERR_ALIGN;
    }
  }
  for (int o = 0; o < n_out; ++o) {
    if (out[o].p == nullptr) continue;
    const Range ro = range_of(out[o].p, out[o].bytes);
    for (int i = 0; i < n_in; ++i)
      if (in[i].p != nullptr && overlaps(ro, range_of(in[i].p, in[i].bytes))) return LORA_ERR_ALIAS;
    for (int o2 = o + 1; o2 < n_out; ++o2)
      if (out[o2].p != nullptr && overlaps(ro, range_of(out[o2].p, out[o2].bytes))) return LORA_ERR_ALIAS;
  }
  return LORA_OK;
}

// The workspace rule of lora_bwd for the two-call form.
static lora_status_t check_workspace(const void* workspace, size_t workspace_bytes, size_t need) {
  if (need == 0) return LORA_OK;
  if (workspace == nullptr || workspace_bytes < need) return LORA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LORA_ERR_ALIGN;
  return LORA_OK;
}

lora_status_t lora_bwd_grads(const void* X, const void* A, const void* B, const void* dY, void* dA, void* dB,
                             int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha, void* workspace,
                             size_t workspace_bytes, uint32_t flags, void* stream) {
  if ((flags & ~LORA_BWD_FP32_GRADS) != 0u) return LORA_ERR_FLAGS;
  lora_status_t s = check_sizes(M, d_in, d_out, r);
  if (s != LORA_OK) return s;
  const bool f32 = (flags & LORA_BWD_FP32_GRADS) != 0u;
  const uint64_t gb = f32 ? 4 : 2;
  const size_t need = lora_bwd_workspace_size(M, d_in, d_out, r);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != LORA_OK) return s;
  const bool rows = M > 0;
  const BufSpec in[4] = {{X, uint64_t(M) * d_in * 2, rows}, {A, uint64_t(r) * d_in * 2, true},
                         {B, uint64_t(d_out) * r * 2, true}, {dY, uint64_t(M) * d_out * 2, rows}};
  const BufSpec out[3] = {{dA, uint64_t(r) * d_in * gb, true}, {dB, uint64_t(d_out) * r * gb, true},
                          {rows ? workspace : nullptr, need, rows}};
  if ((s = check_bufs(in, 4, out, 3)) != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!rows) {
    if ((s = zero_bytes(dA, size_t(r) * d_in * gb, st)) != LORA_OK) return s;
    return zero_bytes(dB, size_t(d_out) * r * gb, st);
  }
  return launch_bwd_grads(X, A, B, dY, dA, dB, M, d_in, d_out, r, alpha, workspace, f32, st);
}

lora_status_t lora_bwd_dx(const void* W, const void* A, const void* dY, void* dX, int64_t M, int64_t d_in,
                          int64_t d_out, int32_t r, const void* workspace, size_t workspace_bytes, void* stream) {
  lora_status_t s = check_sizes(M, d_in, d_out, r);
  if (s != LORA_OK) return s;
  const size_t need = lora_bwd_workspace_size(M, d_in, d_out, r);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != LORA_OK) return s;
  const bool rows = M > 0;
  const BufSpec in[4] = {{W, uint64_t(d_out) * d_in * 2, true}, {A, uint64_t(r) * d_in * 2, true},
                         {dY, uint64_t(M) * d_out * 2, rows}, {rows ? workspace : nullptr, need, rows}};
  const BufSpec out[1] = {{dX, uint64_t(M) * d_in * 2, rows}};
  if ((s = check_bufs(in, 4, out, 1)) != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  if (!rows) return LORA_OK;
  return launch_bwd_dx(W, A, dY, dX, M, d_in, d_out, r, workspace, dev.sm_count,
                       reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_bwd_ex(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                          void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                          void* workspace, size_t workspace_bytes, uint32_t flags, void* stream) {
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha, workspace, workspace_bytes,
                 lora_bwd_workspace_size(M, d_in, d_out, r), flags, stream);
}

lora_status_t lora_merge(const void* W_src, const void* A, const void* B, void* W_dst, int64_t d_out,
                         int64_t d_in, int32_t r, float alpha, void* stream) {
  MergeItem it{W_src, A, B, W_dst, d_out, d_in};
  lora_status_t s = check_merge_item(it, r);
  if (s != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  return run_merge(&it, 1, r, alpha, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_merge_batched(const lora_merge_desc_t* descs, int32_t n, int32_t r, float alpha, void* stream) {
  if (n < 0) return LORA_ERR_SHAPE;
  if (n == 0) return LORA_OK;
  if (descs == nullptr) return LORA_ERR_NULL;
  std::vector<MergeItem> items(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    items[i] = MergeItem{descs[i].W_src, descs[i].A, descs[i].B, descs[i].W_dst, descs[i].d_out, descs[i].d_in};
    lora_status_t s = check_merge_item(items[i], r);
    if (s != LORA_OK) return s;
  }
  DeviceInfo dev;
  lora_status_t s = device_info(dev);
  if (s != LORA_OK) return s;
  return run_merge(items.data(), n, r, alpha, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_restore(const void* W_src, void* W_dst, int64_t n_elems, void* stream) {
  if (n_elems < 0) return LORA_ERR_SHAPE;
  if (n_elems == 0) return LORA_OK;
  if (!W_src || !W_dst) return LORA_ERR_NULL;
  if (!aligned16(W_src) || !aligned16(W_dst)) return LORA_ERR_ALIGN;
  if (W_src != W_dst && overlaps(range_of(W_src, uint64_t(n_elems) * 2), range_of(W_dst, uint64_t(n_elems) * 2)))
    return LORA_ERR_ALIAS;
  DeviceInfo dev;
  lora_status_t s = device_info(dev);
  if (s != LORA_OK) return s;
  if (W_src == W_dst) return LORA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t n16 = size_t(n_elems) * 2 / 16;
  if (n16 > 0) {
    const int blocks = int(std::min<size_t>((n16 + 255) / 256, size_t(dev.sm_count) * 8));
    s = launch_ex("copy", copy16_kernel, dim3(unsigned(blocks)), dim3(256), 0, st, nullptr,
                  reinterpret_cast<const uint4*>(W_src), reinterpret_cast<uint4*>(W_dst), n16);
    if (s != LORA_OK) return s;
  }
  const size_t done = n16 * 8;
  const size_t rest = size_t(n_elems) - done;
  if (rest > 0) {
    s = launch_ex("copy", copy2_kernel, dim3(1), dim3(256), 0, st, nullptr,
                  reinterpret_cast<const uint16_t*>(W_src) + done, reinterpret_cast<uint16_t*>(W_dst) + done, rest);
    if (s != LORA_OK) return s;
  }
  return LORA_OK;
}

lora_status_t lora_get_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return LORA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, lora::g_status, sizeof(v)) != cudaSuccess) return LORA_ERR_CUDA;
  if (v != 0u) {
    unsigned int info[4] = {0, 0, 0, 0};
    cudaMemcpyFromSymbol(info, lora::g_status_info, sizeof(info));
    std::fprintf(stderr, "lora_b200: bounded wait gave up (block %u, thread %u, site %u, parity %u)\n", info[0],
                 info[1], info[2], info[3]);
    const unsigned int zero[5] = {0, 0, 0, 0, 0};
    cudaMemcpyToSymbol(lora::g_status, zero, sizeof(unsigned int));
    cudaMemcpyToSymbol(lora::g_status_info, zero, sizeof(info));
    return LORA_ERR_TIMEOUT;
  }
  return LORA_OK;
}

lora_status_t lora_selftest_wait_timeout(int64_t limit_ns) {
  DeviceInfo dev;
  lora_status_t s = device_info(dev);
  if (s != LORA_OK) return s;
  const uint64_t lim = uint64_t(std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 1000000000));
  lora::selftest_wait_kernel<<<1, 32>>>(lim);
  if ((s = launch_status()) != LORA_OK) return s;
  return lora_get_device_status();
}

}  // extern "C"

// ====================================================== no-alloc backward ====
//
// lora_bwd_noalloc: the backward for callers that cannot call cudaMalloc.
//
// lora_bwd needs device scratch (T, dT and the split-M partial sums) and
// asks the caller for it.  Some callers have no way to provide it: a plugin
// running inside a host program that owns every device allocation through
// its own pool, or a service loop that must not allocate once it has
// started (cudaMalloc can block until the device is idle, and can fail
// when memory is tight, at a point where the caller cannot recover).  This
// entry point serves them with scratch that the library reserves itself:
// a fixed-size array in device global memory, part of the library's GPU
// module.  It is reserved on every GPU that loads the library and stays
// there until the process exits.
//
// The array is a file-scope __device__ symbol, so host code cannot use its
// name as a device address (on the host the name refers to a host-side
// stand-in).  The first call on each device, with that device current,
// looks the real address up with cudaGetSymbolAddress, checks the result,
// and keeps it for later calls on that device; that first call should be
// made before any stream capture begins.  The kernels then receive that
// address exactly as they would receive a caller's workspace.
//
// All calls share the one array, and it keeps whatever the previous call
// left in it.  Nothing in it needs to start at zero: each call writes every
// scratch byte before reading it.  Two calls whose work can overlap on the
// GPU (for example on two different streams) use the same bytes at the same
// time and corrupt each other's results; order them on one stream.

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
}  // namespace

static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_bwd_noalloc_scratch on the current device (looked up
// once per device).
lora_status_t noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      std::fprintf(stderr, "lora_bwd_noalloc: cudaGetSymbolAddress failed on device %d: %s\n", dev,
                   cudaGetErrorString(e));
      return LORA_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return LORA_OK;
}
}  // namespace

extern "C" lora_status_t lora_bwd_noalloc(const void* X, const void* W, const void* A, const void* B,
                                          const void* dY, void* dX, void* dA, void* dB, int64_t M,
                                          int64_t d_in, int64_t d_out, int32_t r, float alpha, void* stream) {
  lora_status_t s = check_sizes(M, d_in, d_out, r);
  if (s != LORA_OK) return s;
  const size_t need = lora_bwd_workspace_size(M, d_in, d_out, r);
  if (need > kNoAllocScratchBytes) {
    std::fprintf(stderr,
                 "lora_bwd_noalloc: M=%lld d_in=%lld d_out=%lld r=%d needs %zu bytes of scratch, more than the "
                 "fixed %zu bytes this entry point has; call lora_bwd with a workspace instead\n",
                 (long long)M, (long long)d_in, (long long)d_out, int(r), need, kNoAllocScratchBytes);
    return LORA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    DeviceInfo dev;
    if ((s = device_info(dev)) != LORA_OK) return s;
    if ((s = noalloc_scratch_address(&scratch)) != LORA_OK) return s;
  }
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                 need, 0u, stream);
}
