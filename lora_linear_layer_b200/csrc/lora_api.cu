// lora_api.cu - the extern "C" entry points declared in include/lora.h.
//
// Host side of the library, one translation unit: host_common.cuh holds the
// validation helpers, device state, tensor maps and the launch helper;
// host_plan.cuh the configuration and launch of each kernel; this file the
// entry points themselves (argument rules, then launches on the caller's
// stream).  All arithmetic of the layer runs in the kernels of fused.cuh,
// splitk.cuh, skinny.cuh and merge.cuh.
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
#include "host_common.cuh"
#include "host_plan.cuh"

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

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if unknown).  A
// device reset ends the context and reloads the library's module in the
// next one at another address; the id tells the two apart, where the
// context handle itself may be reused.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_cur == nullptr || get_id == nullptr) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return 0;
    get_cur = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// The forward's T exchange slots (texchange.cuh) of each device.  Each slot
// is bound to one stream, by the stream's unique id, the first time a
// launch on that stream asks for one, and stays bound to it.  Launches on
// one stream run one after the other (every kernel of this library waits
// for the previous kernel of its stream to complete before it touches
// global memory), so a slot is never used by two launches at once and each
// launch finds it as the previous one left it: clean.  A stream that finds
// every slot bound to other streams runs without the exchange, and so does
// a launch being captured into a graph (a replay could run at any time,
// beside the slot's stream).
struct TxPool {
  unsigned long long ctx_id = 0;
  TxSlot* base = nullptr;
  unsigned long long stream_id[kTxSlots] = {};  // bound stream's id + 1; 0 = unbound
};
std::mutex g_txpool_mu;
TxPool g_txpool[64];

// The exchange slot of stream `st` on the current device, or NULL.
TxSlot* tx_slot_for(cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (cs != cudaStreamCaptureStatusNone) return nullptr;
  unsigned long long sid = 0;
  if (cudaStreamGetId(st, &sid) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const unsigned long long ctx = current_ctx_id();
  if (ctx == 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_txpool_mu);
  TxPool& p = g_txpool[dev];
  if (p.base == nullptr || p.ctx_id != ctx) {
    // first use in this context (again after a device reset): the slots' address
    void* b = nullptr;
    if (cudaGetSymbolAddress(&b, g_tx) != cudaSuccess || b == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    p.base = reinterpret_cast<TxSlot*>(b);
    p.ctx_id = ctx;
    for (int i = 0; i < kTxSlots; ++i) p.stream_id[i] = 0;
  }
  for (int i = 0; i < kTxSlots; ++i)
    if (p.stream_id[i] == sid + 1) return p.base + i;
  for (int i = 0; i < kTxSlots; ++i)
    if (p.stream_id[i] == 0) {
      p.stream_id[i] = sid + 1;
      return p.base + i;
    }
  return nullptr;
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

// T = X A^T as bf16 [M, r_pad] (zero columns past r) into `Tws`: one
// skinny launch.  Arguments already validated, M > 0.
static lora_status_t launch_t(const void* X, const void* A, int64_t M, int64_t d_in, int32_t r,
                              __nv_bfloat16* Tws, int sm_count, cudaStream_t st) {
  SkinnyCfg ct;
  pick_skinny(M, d_in, r, false, OUT_ROWS_RPAD, (M + 127) / 128, sm_count, ct);
  ct.args.out = Tws;
  CUtensorMap mp, mr;
  if (!make_map(&mp, X, d_in, M, d_in, 64, 128, 128) || !make_map(&mr, A, d_in, r, d_in, 64, ct.r_pad, 128))
    return LORA_ERR_CUDA;
  return launch_skinny<false>(mp, mr, ct, st);
}

// The forward; when `Tws` is not NULL it also receives T = X A^T (bf16
// [M, r_pad], zero columns past r).  Arguments already validated, M > 0.
static lora_status_t fwd_run(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                             int64_t d_in, int64_t d_out, int32_t r, float scale, __nv_bfloat16* Tws,
                             int sm_count, cudaStream_t st) {
  {
    SplitkPlan pl;
    if (use_splitk(M, d_out, d_in, r, sm_count, pl)) {
      // split-K tiles each form their own partial T; the saved T is one
      // more (skinny) launch
      SplitkTable<1> t;
      std::memset(&t, 0, sizeof(t));
      splitk_table_common(t, 1, pl, scale);
      if (!splitk_job(t.job[0], X, W, A, B, Y, M, d_in, d_out, r, pl, 0)) return LORA_ERR_CUDA;
      const int tiles = int(((M + 127) / 128) * ((d_out + 127) / 128));
      const lora_status_t s = launch_splitk(t, tiles, pl, st);
      if (s != LORA_OK || Tws == nullptr) return s;
      return launch_t(X, A, M, d_in, r, Tws, sm_count, st);
    }
  }
  FusedCfg c;
  if (!pick_fused(M, d_out, d_in, r, false, sm_count, c)) return LORA_ERR_RANK;
  c.args.scale = scale;
  c.args.out = reinterpret_cast<__nv_bfloat16*>(Y);
  c.args.t_out = Tws;
  // with an exchange slot, the seeded schedule that shares T between
  // clusters (other schedules would gain nothing from the exchange: the
  // runs of an M block start together)
  TxSlot* const tx = c.tx_fits && c.seeded_l > 0 ? tx_slot_for(st) : nullptr;
  c.args.tx = tx;
  const bool seeded = tx != nullptr && c.seeded_l > 0;
  c.args.run_l = seeded ? c.seeded_l : c.run_l_plain;
  c.args.seeded = seeded ? 1 : 0;
  CUtensorMap maps[6];
  // Q and V rows per CTA, and U's rows per CTA; the pair fold's odd CTA
  // loads 96 rows of W (maps[5]) and 32 of A
  const bool pf = c.BN == kPairFoldBN;
  const uint32_t bnc = pf ? 128u : uint32_t(c.BN / c.CG);
  const uint32_t u_box = pf ? uint32_t(kPairFoldT) : uint32_t(c.r_pad / c.CG);
  if (!make_map(&maps[0], X, d_in, M, d_in, 64, 128, 128) ||
      !make_map(&maps[1], W, d_in, d_out, d_in, 64, bnc, 128) ||
      !make_map(&maps[2], A, d_in, r, d_in, 64, u_box, 128) ||
      !make_map(&maps[3], B, r, d_out, r, c.RCW, bnc, c.RCW * 2) ||
      !make_map(&maps[4], Y, d_out, M, d_out, kEpCols, 32, kEpCols * 2) ||
      !make_map(&maps[5], W, d_in, d_out, d_in, 64, pf ? uint32_t(128 - kPairFoldT) : bnc, 128))
    return LORA_ERR_CUDA;
  return launch_fused<false>(maps, c, sm_count, st);
}

// The forward with the scale given (alpha / r for lora_fwd).
static lora_status_t fwd_entry(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                               int64_t d_in, int64_t d_out, int32_t r, float scale, void* stream) {
  const void* ptrs[5] = {X, W, A, B, Y};
  lora_status_t s = lora_check_args(0, ptrs, 5, M, d_in, d_out, r, 0);
  if (s != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  if (M == 0) return LORA_OK;
  return fwd_run(X, W, A, B, Y, M, d_in, d_out, r, scale, nullptr, dev.sm_count,
                 reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_fwd(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                       int64_t d_in, int64_t d_out, int32_t r, float alpha, void* stream) {
  return fwd_entry(X, W, A, B, Y, M, d_in, d_out, r, alpha / float(r), stream);
}

lora_status_t lora_fwd_scaled(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                              int64_t d_in, int64_t d_out, int32_t r, float scale, void* stream) {
  return fwd_entry(X, W, A, B, Y, M, d_in, d_out, r, scale, stream);
}

// The grouped forward with the scale given (alpha / r for lora_fwd_batched).
static lora_status_t fwd_batched_entry(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float scale,
                                       void* stream) {
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
      if ((s = fwd_entry(d.X, d.W, d.A, d.B, d.Y, d.M, d.d_in, d.d_out, r, scale, stream)) != LORA_OK) return s;
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
    splitk_table_common(t, nj, pl, scale);
    if ((s = launch_splitk(t, tb, pl, st)) != LORA_OK) return s;
    g = end;
  }
  return LORA_OK;
}

lora_status_t lora_fwd_batched(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float alpha, void* stream) {
  return fwd_batched_entry(descs, n, r, alpha / float(r), stream);
}

lora_status_t lora_fwd_batched_scaled(const lora_fwd_desc_t* descs, int32_t n, int32_t r, float scale,
                                      void* stream) {
  return fwd_batched_entry(descs, n, r, scale, stream);
}

size_t lora_bwd_workspace_size(int64_t M, int64_t d_in, int64_t d_out, int32_t r) {
  if (check_sizes(M, d_in, d_out, r) != LORA_OK || M == 0) return 0;
  return bwd_workspace(M, r).total;
}

// Launches 1 and 2 of the backward: T (unless `t_saved`: the forward left
// it in the workspace) and dT into the workspace, then dA and dB.
// Arguments already validated, M > 0.
static lora_status_t launch_bwd_grads(const void* X, const void* A, const void* B, const void* dY, void* dA,
                                      void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                                      void* workspace, bool f32, bool t_saved, int sm_count, cudaStream_t st) {
  BwdPlan p;
  plan_bwd(M, d_in, d_out, r, sm_count, p);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* Tws = reinterpret_cast<__nv_bfloat16*>(ws + p.off_t);
  __nv_bfloat16* dTws = reinterpret_cast<__nv_bfloat16*>(ws + p.off_dt);
  const int r_pad = r_pad_of(r);
  const int rcw = rcw_of(r_pad);
  lora_status_t s = LORA_OK;

  // 1. One launch, two jobs: dT = s dY B and T = X A^T (recomputed), each
  //    bf16 [M, r_pad] with zero columns past r.  The longer contraction's
  //    job takes the first row tiles of the grid, so it starts first.
  //    With T saved by the forward: dT alone.
  if (t_saved) {
    CUtensorMap mp_dt, mr_dt;
    if (!make_map(&mp_dt, dY, d_out, M, d_out, 64, 128, 128) || !make_map(&mr_dt, B, r, d_out, r, rcw, 64, rcw * 2))
      return LORA_ERR_CUDA;
    SkinnyCfg cdt = p.dto_cfg;
    cdt.args.out = dTws;
    cdt.args.scale = scale;
    if ((s = launch_skinny<false>(mp_dt, mr_dt, cdt, st)) != LORA_OK) return s;
  } else {
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
  const __nv_bfloat16* dTws = reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const uint8_t*>(workspace) +
                                                                     bwd_workspace(M, r).off_dt);
  const int r_pad = r_pad_of(r);
  lora_status_t s = LORA_OK;
  // 3. dX = dY W + dT A: one GEMM over the contraction [d_out | r_pad]
  {
    FusedCfg c;
    if (!pick_fused(M, d_in, d_out, r, true, sm_count, c)) return LORA_ERR_RANK;
    c.args.scale = 1.0f;
    c.args.out = reinterpret_cast<__nv_bfloat16*>(dX);
    CUtensorMap maps[6];
    if (!make_map(&maps[0], dY, d_out, M, d_out, 64, 128, 128) ||
        !make_map(&maps[1], W, d_in, d_out, d_in, 64, 64, 128) ||
        !make_map(&maps[2], dTws, r_pad, M, r_pad, 64, 128, 128) ||
        !make_map(&maps[3], A, d_in, r, d_in, 64, 64, 128) ||
        !make_map(&maps[4], dX, d_in, M, d_in, kEpCols, 32, kEpCols * 2))
      return LORA_ERR_CUDA;
    maps[5] = maps[1];  // (unused by the dX form)
    if ((s = launch_fused<true>(maps, c, sm_count, st)) != LORA_OK) return s;
  }
  return LORA_OK;
}

// The backward, with `need` bytes of workspace required; `flags` as in
// lora_bwd_ex.
static lora_status_t bwd_run(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                             void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                             void* workspace, size_t workspace_bytes, size_t need, uint32_t flags, void* stream) {
  if ((flags & ~kBwdFlags) != 0u) return LORA_ERR_FLAGS;
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
  if ((s = launch_bwd_grads(X, A, B, dY, dA, dB, M, d_in, d_out, r, scale, workspace, f32,
                            (flags & LORA_BWD_T_SAVED) != 0u, dev.sm_count, st)) != LORA_OK)
    return s;
  return launch_bwd_dx(W, A, dY, dX, M, d_in, d_out, r, workspace, dev.sm_count, st);
}

lora_status_t lora_bwd(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                       void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha / float(r), workspace, workspace_bytes,
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

// lora_fwd_save with the scale given.
static lora_status_t fwd_save_entry(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                                    int64_t d_in, int64_t d_out, int32_t r, float scale, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  const void* ptrs[5] = {X, W, A, B, Y};
  lora_status_t s = lora_check_args(0, ptrs, 5, M, d_in, d_out, r, 0);
  if (s != LORA_OK) return s;
  const size_t need = lora_bwd_workspace_size(M, d_in, d_out, r);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != LORA_OK) return s;
  if (M > 0) {
    const Range ws = range_of(workspace, need);
    const uint64_t bytes[5] = {uint64_t(M) * d_in * 2, uint64_t(d_out) * d_in * 2, uint64_t(r) * d_in * 2,
                               uint64_t(d_out) * r * 2, uint64_t(M) * d_out * 2};
    for (int i = 0; i < 5; ++i)
      if (overlaps(ws, range_of(ptrs[i], bytes[i]))) return LORA_ERR_ALIAS;
  }
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  if (M == 0) return LORA_OK;
  __nv_bfloat16* Tws =
      reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(workspace) + bwd_workspace(M, r).off_t);
  return fwd_run(X, W, A, B, Y, M, d_in, d_out, r, scale, Tws, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_fwd_save(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                            int64_t d_in, int64_t d_out, int32_t r, float alpha, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return fwd_save_entry(X, W, A, B, Y, M, d_in, d_out, r, alpha / float(r), workspace, workspace_bytes, stream);
}

lora_status_t lora_fwd_save_scaled(const void* X, const void* W, const void* A, const void* B, void* Y, int64_t M,
                                   int64_t d_in, int64_t d_out, int32_t r, float scale, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return fwd_save_entry(X, W, A, B, Y, M, d_in, d_out, r, scale, workspace, workspace_bytes, stream);
}

// lora_bwd_grads with the scale given.
static lora_status_t bwd_grads_entry(const void* X, const void* A, const void* B, const void* dY, void* dA, void* dB,
                                     int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale, void* workspace,
                                     size_t workspace_bytes, uint32_t flags, void* stream) {
  if ((flags & ~kBwdFlags) != 0u) return LORA_ERR_FLAGS;
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
  return launch_bwd_grads(X, A, B, dY, dA, dB, M, d_in, d_out, r, scale, workspace, f32,
                          (flags & LORA_BWD_T_SAVED) != 0u, dev.sm_count, st);
}

lora_status_t lora_bwd_grads(const void* X, const void* A, const void* B, const void* dY, void* dA, void* dB,
                             int64_t M, int64_t d_in, int64_t d_out, int32_t r, float alpha, void* workspace,
                             size_t workspace_bytes, uint32_t flags, void* stream) {
  return bwd_grads_entry(X, A, B, dY, dA, dB, M, d_in, d_out, r, alpha / float(r), workspace, workspace_bytes, flags,
                         stream);
}

lora_status_t lora_bwd_grads_scaled(const void* X, const void* A, const void* B, const void* dY, void* dA, void* dB,
                                    int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale, void* workspace,
                                    size_t workspace_bytes, uint32_t flags, void* stream) {
  return bwd_grads_entry(X, A, B, dY, dA, dB, M, d_in, d_out, r, scale, workspace, workspace_bytes, flags, stream);
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
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha / float(r), workspace, workspace_bytes,
                 lora_bwd_workspace_size(M, d_in, d_out, r), flags, stream);
}

lora_status_t lora_bwd_scaled(const void* X, const void* W, const void* A, const void* B, const void* dY, void* dX,
                              void* dA, void* dB, int64_t M, int64_t d_in, int64_t d_out, int32_t r, float scale,
                              void* workspace, size_t workspace_bytes, uint32_t flags, void* stream) {
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, scale, workspace, workspace_bytes,
                 lora_bwd_workspace_size(M, d_in, d_out, r), flags, stream);
}

// lora_merge with the scale given.
static lora_status_t merge_entry(const void* W_src, const void* A, const void* B, void* W_dst, int64_t d_out,
                                 int64_t d_in, int32_t r, float scale, void* stream) {
  MergeItem it{W_src, A, B, W_dst, d_out, d_in};
  lora_status_t s = check_merge_item(it, r);
  if (s != LORA_OK) return s;
  DeviceInfo dev;
  if ((s = device_info(dev)) != LORA_OK) return s;
  return run_merge(&it, 1, r, scale, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_merge(const void* W_src, const void* A, const void* B, void* W_dst, int64_t d_out,
                         int64_t d_in, int32_t r, float alpha, void* stream) {
  return merge_entry(W_src, A, B, W_dst, d_out, d_in, r, alpha / float(r), stream);
}

lora_status_t lora_merge_scaled(const void* W_src, const void* A, const void* B, void* W_dst, int64_t d_out,
                                int64_t d_in, int32_t r, float scale, void* stream) {
  return merge_entry(W_src, A, B, W_dst, d_out, d_in, r, scale, stream);
}

// lora_merge_batched with the scale given.
static lora_status_t merge_batched_entry(const lora_merge_desc_t* descs, int32_t n, int32_t r, float scale,
                                         void* stream) {
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
  return run_merge(items.data(), n, r, scale, dev.sm_count, reinterpret_cast<cudaStream_t>(stream));
}

lora_status_t lora_merge_batched(const lora_merge_desc_t* descs, int32_t n, int32_t r, float alpha, void* stream) {
  return merge_batched_entry(descs, n, r, alpha / float(r), stream);
}

lora_status_t lora_merge_batched_scaled(const lora_merge_desc_t* descs, int32_t n, int32_t r, float scale,
                                        void* stream) {
  return merge_batched_entry(descs, n, r, scale, stream);
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
// lora_bwd needs device scratch (the bf16 T and dT of every row, which
// pass from its first launch to the later ones) and asks the caller for it.  Some callers have no way to provide it: a plugin
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
// and keeps it, with the id of the context it belongs to, for later calls
// on that device; that first call should be made before any stream capture
// begins.  After a device reset the next call finds a new context and looks
// the address up again (it should then also come before any capture).  The kernels then receive that
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
struct NoallocAddr {
  unsigned long long ctx_id;  // the context the address belongs to
  void* addr;
};
NoallocAddr g_noalloc_addr[64] = {};

// Device address of g_bwd_noalloc_scratch in the current device's context,
// looked up once per context (again after a device reset).
lora_status_t noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LORA_ERR_CUDA;
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocAddr& e = g_noalloc_addr[dev];
  if (e.addr == nullptr || ctx == 0 || e.ctx_id != ctx) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch);
    if (err != cudaSuccess || p == nullptr) {
      std::fprintf(stderr, "lora_bwd_noalloc: cudaGetSymbolAddress failed on device %d: %s\n", dev,
                   cudaGetErrorString(err));
      e.addr = nullptr;
      return LORA_ERR_CUDA;
    }
    e.addr = p;
    e.ctx_id = ctx;
  }
  *out = e.addr;
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
  return bwd_run(X, W, A, B, dY, dX, dA, dB, M, d_in, d_out, r, alpha / float(r), scratch,
                 need > 0 ? kNoAllocScratchBytes : 0,
                 need, 0u, stream);
}
