// host_plan.cuh - launch configuration and launches of every kernel: the
// fused kernel's tile shape, pipeline depth and run schedule; the split-K
// forward (one problem or a grouped table); the skinny split-M launches and
// the backward's workspace plan; the merge job tables.  Each plan is a pure
// function of the problem sizes and the device's SM count.
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
#include "fused.cuh"
#include "merge.cuh"
#include "skinny.cuh"
#include "splitk.cuh"
#include "host_common.cuh"

namespace {

using namespace lora;

// ------------------------------------------------------------ fused GEMM ----

struct FusedCfg {
  int BN, CG, RCW, r_pad, n_rchunks, stages, ep_bufs;
  uint32_t smem;
  bool tx_fits;              // forward whose T fits an exchange slot (and the exchange is enabled)
  int seeded_l;              // seeded schedule's run length when the launch gets a slot (0: runs) ...
  double seeded_cost;
  int run_l_plain;           // ... and the run length without one (runs cover every N tile)
  double model_cost;         // modelled makespan in 256 x 256 pair-tile times (CTA-pair tiles only; else 0)
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
  if (std::sscanf(e, "%d,%d", &b, &g) == 2 &&
      (((b == 128 || b == 256) && (g == 1 || g == 2)) || (b == kPairFoldBN && g == 2))) {
    BN = b;
    CG = g;
  }
}

// LORA_B200_TX=0 turns the forward's T exchange between clusters off (every
// tile that starts an M block then computes T itself); for tests.
bool tx_enabled() {
  const char* e = std::getenv("LORA_B200_TX");
  return !(e != nullptr && e[0] == '0');
}

// Optional schedule override from LORA_B200_FUSED_RUN (-1 = choose).
int run_override() {
  const char* e = std::getenv("LORA_B200_FUSED_RUN");
  if (e == nullptr) return -1;
  const int v = std::atoi(e);
  return v >= 0 && v <= 4096 ? v : -1;
}

// The plan for one tile choice: (fBN, fCG) forced, or 0, 0 to choose.
bool pick_fused_tile(int64_t M, int64_t N, int64_t K, int r, bool mn, int sm_count, int fBN, int fCG,
                     FusedCfg& c) {
  c.r_pad = r_pad_of(r);
  c.RCW = rcw_of(c.r_pad);
  c.n_rchunks = (c.r_pad + c.RCW - 1) / c.RCW;
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
  const int cands[5][2] = {
      {256, short_k ? 1 : 2}, {256, short_k ? 2 : 1}, {128, 1}, {128, 2}, {kPairFoldBN, 2}};
  c.BN = 0;
  for (int pass = 0; pass < 2 && c.BN == 0; ++pass) {  // pass 1 ignores an infeasible override
    for (int i = 0; i < 5; ++i) {
      const int BN = cands[i][0], CG = cands[i][1];
      const bool forced = pass == 0 && fBN != 0;
      if (forced && (BN != fBN || CG != fCG)) continue;
      if (!forced && i >= 3) break;  // the 128-wide pair and the pair fold only when forced (or chosen below)
      if (BN == kPairFoldBN && (mn || c.r_pad > kPairFoldT)) continue;  // forward only, T in 32 columns
      const int S = fused_stages(BN, CG, mn, c.RCW, c.r_pad, c.n_rchunks, 1);
      if (S < (BN >= 224 ? 3 : 2)) continue;
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
  a.t_out = nullptr;
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
  a.seeded = 0;
  a.tx = nullptr;             // the launch assigns a slot
  // The T exchange (texchange.cuh): a cluster starting on an M block whose
  // T another cluster has published copies it instead of computing it.
  // That allows the seeded schedule (TileSched): every cluster first runs
  // L tiles of one M block, which computes and publishes every block's T;
  // the rest is dealt round-robin like the dX form's single tiles, whose
  // operands stay in L2 (8192 x 4096 x 4096: dX read 114 MB from DRAM, the
  // forward's runs of 8 on 64 of 74 clusters 312 MB) and which keeps every
  // cluster busy.  Used when every M block gets a seeding run inside the
  // first column band and the model (L + 0.5 tile times for the seeding
  // run, 3% per copying tile after it) beats the runs.
  c.tx_fits = !mn && num_m <= int(kTxMaxBlocks) &&
              double(num_m) * double(kBM * c.CG) * double(c.r_pad) <= double(kTxElems) && tx_enabled();
  c.seeded_l = 0;
  c.seeded_cost = 0.0;
  if (c.tx_fits && best_l > 0 && clusters >= num_m) {
    for (int l = 2; l <= 4; ++l) {
      const int64_t a_lo = clusters / num_m, r0 = clusters % num_m;
      const int64_t w0 = std::min(a.band_w, num_n);
      if ((a_lo + (r0 > 0 ? 1 : 0)) * l > w0) continue;  // the seeding stays inside the first band
      const int64_t seeded = r0 * std::min<int64_t>(w0, (a_lo + 1) * l) +
                             (num_m - r0) * std::min<int64_t>(w0, a_lo * l);
      const int64_t rest = int64_t(num_m) * num_n - seeded;
      const double cost = l + 0.5 + double((rest + clusters - 1) / clusters) * 1.03;
      // shorter seeding runs keep more tiles in the L2-friendly order: a
      // longer one must be clearly cheaper in the model
      if (cost < best_cost - 0.25 && (c.seeded_l == 0 || cost < c.seeded_cost - 0.15)) {
        c.seeded_l = l;
        c.seeded_cost = cost;
      }
    }
  }
  // LORA_B200_SEEDED_L=L forces the seeded schedule's run length (when the
  // schedule applies at all); for tests and measurements
  if (const char* e = std::getenv("LORA_B200_SEEDED_L")) {
    const int l = std::atoi(e);
    if (c.seeded_l > 0 && l >= 1 && l <= num_n) c.seeded_l = l;
  }
  const int ro = run_override();
  if (ro >= 0) c.seeded_l = 0;
  c.run_l_plain = ro >= 0 ? ro : best_l;
  if (c.BN == kPairFoldBN) {
    // T comes with the base product: no exchange, and single-tile runs
    // dealt round-robin (as the dX form) keep the tiles in flight on a few
    // M blocks
    c.tx_fits = false;
    c.seeded_l = 0;
    c.run_l_plain = ro >= 0 ? ro : 1;
  }
  a.run_l = c.seeded_l > 0 ? c.seeded_l : c.run_l_plain;
  a.seeded = c.seeded_l > 0 ? 1 : 0;
  a.wait_limit_ns = kWaitLimitNs;
  // modelled makespan in 256 x 256 pair-tile times, for the choice below
  c.model_cost = 0.0;
  if (c.CG == 2 && c.BN == kPairFoldBN) {
    // a fold tile computes 256 columns for 224 of output: 1.15 tile times
    // fits the same-box measurements (512 x 8192^2: fold 0.84 of the
    // 256-wide pair's time, 1024 x 8192^2 0.93, 2048 x 8192^2 1.04,
    // 512 x 4096 x 14336 1.03-1.14)
    c.model_cost = 1.15 * double((int64_t(num_m) * num_n + clusters - 1) / clusters);
  } else if (c.CG == 2 && c.BN == 256 && !mn) {
    if (c.seeded_l > 0) {
      c.model_cost = c.seeded_cost;
    } else if (c.run_l_plain > 0) {
      const int64_t runs = int64_t(num_m) * ((num_n + c.run_l_plain - 1) / c.run_l_plain);
      c.model_cost = double((runs + clusters - 1) / clusters) * (c.run_l_plain + 0.5);
    } else {
      c.model_cost = double((int64_t(num_m) * num_n + clusters - 1) / clusters) + 0.5;
    }
  }
  return true;
}

// The forward's tile: as pick_fused_tile chooses, or, where that is the
// 256-wide pair, the 224-wide pair fold when its grid fills the pairs and its
// modelled makespan is at least 10% shorter.  The fold pays no separate T
// products (a T tile of the 256-wide pair costs about 1.5 tile times: the
// N = r products take as long as N = 128 ones), but every fold tile spends
// 32 of its 256 columns on T, and its 224-wide grid quantises differently:
// it wins where few tiles per pair each compute T (512 x 8192 x 8192: 64
// pair tiles with T against 74 fold tiles), and loses where the exchange or
// longer runs leave one T per pair (8192 x 4096 x 4096: 7.5 against 10.4).
bool pick_fused(int64_t M, int64_t N, int64_t K, int r, bool mn, int sm_count, FusedCfg& c) {
  int fBN, fCG;
  tile_override(fBN, fCG);
  if (!pick_fused_tile(M, N, K, r, mn, sm_count, fBN, fCG, c)) return false;
  if (fBN != 0 || mn || c.BN != 256 || c.CG != 2 || r_pad_of(r) > kPairFoldT) return true;
  FusedCfg pf;
  if (!pick_fused_tile(M, N, K, r, mn, sm_count, kPairFoldBN, 2, pf) || pf.BN != kPairFoldBN) return true;
  const int64_t pf_tiles = int64_t(pf.args.num_m) * pf.args.num_n;
  if (double(pf_tiles) >= 0.8 * double(sm_count / 2) && pf.model_cost <= 0.9 * c.model_cost) c = pf;
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

// maps: P, Q, U, V, OUT and the pair fold's second Q map (any valid map otherwise)
template <int BN, bool MN, int RCW, int CG, bool TX>
lora_status_t launch_fused_t(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  auto kern = fused_lora_kernel<BN, MN, RCW, CG, TX>;
  if (!ensure_smem_attr(kern, c.smem)) return LORA_ERR_CUDA;
  const int64_t tiles = int64_t(c.args.num_m) * c.args.num_n;
  const int clusters = int(std::min<int64_t>(tiles, max_clusters(kern, CG, c.smem, sm_count)));
  const dim3 cl(unsigned(CG), 1, 1);
  return launch_ex("fused", kern, dim3(unsigned(clusters * CG)), dim3(kFusedThreads), c.smem, st, &cl, maps[0],
                   maps[1], maps[2], maps[3], maps[4], maps[5], c.args);
}

// The forward instances with (TX) and without an exchange slot.
template <int BN, int RCW, int CG>
lora_status_t launch_fused_fwd(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  return c.args.tx != nullptr ? launch_fused_t<BN, false, RCW, CG, true>(maps, c, sm_count, st)
                              : launch_fused_t<BN, false, RCW, CG, false>(maps, c, sm_count, st);
}

template <bool MN, int CG>
lora_status_t launch_fused_cg(const CUtensorMap* maps, const FusedCfg& c, int sm_count, cudaStream_t st) {
  if constexpr (MN) {  // the dX form has no rank chunks in shared memory
    return c.BN == 256 ? launch_fused_t<256, true, 64, CG, false>(maps, c, sm_count, st)
                       : launch_fused_t<128, true, 64, CG, false>(maps, c, sm_count, st);
  } else {
    if constexpr (CG == 2) {
      if (c.BN == kPairFoldBN)  // r_pad <= 32, no exchange
        return c.RCW == 16 ? launch_fused_t<kPairFoldBN, false, 16, 2, false>(maps, c, sm_count, st)
                           : launch_fused_t<kPairFoldBN, false, 32, 2, false>(maps, c, sm_count, st);
    }
    if (c.BN == 256) {
      if (c.RCW == 16) return launch_fused_fwd<256, 16, CG>(maps, c, sm_count, st);
      if (c.RCW == 32) return launch_fused_fwd<256, 32, CG>(maps, c, sm_count, st);
      return launch_fused_fwd<256, 64, CG>(maps, c, sm_count, st);
    }
    if (c.RCW == 16) return launch_fused_fwd<128, 16, CG>(maps, c, sm_count, st);
    if (c.RCW == 32) return launch_fused_fwd<128, 32, CG>(maps, c, sm_count, st);
    return launch_fused_fwd<128, 64, CG>(maps, c, sm_count, st);
  }
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
// splits as keep every resident CTA slot of the device's `sm_count` SMs
// busy, at most 8 (the portable cluster size) and at least 4 K blocks per
// split.
void pick_skinny(int64_t rows, int64_t K, int r, bool r_mn, int out_mode, int64_t launch_tiles, int sm_count,
                 SkinnyCfg& c) {
  c.r_pad = r_pad_of(r);
  c.RCW = rcw_of(c.r_pad);
  c.n_rchunks = (c.r_pad + c.RCW - 1) / c.RCW;
  c.stages = 4;
  const SkinnyLayout L(r_mn, c.RCW, c.r_pad, c.n_rchunks, c.stages);
  c.smem = L.total + 1024;
  const int per_sm = std::max(1, std::min<int>(int(kSmemPerSM / (c.smem + 1024)),
                                               int(512 / tmem_cols_for(c.r_pad))));
  const int slots = per_sm * sm_count;
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
  SkinnyCfg dto_cfg;  // dT alone, when the forward saved T
  size_t off_t, off_dt, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The backward's workspace: T and dT as bf16 [M, r_pad] each, at 256-byte
// aligned offsets (independent of the launch plan and of the device).
struct BwdWorkspace {
  size_t off_t, off_dt, total;
};

BwdWorkspace bwd_workspace(int64_t M, int32_t r) {
  const size_t tb = align256(size_t(M) * size_t(r_pad_of(r)) * 2);
  return BwdWorkspace{0, tb, 2 * tb};
}

void plan_bwd(int64_t M, int64_t d_in, int64_t d_out, int32_t r, int sm_count, BwdPlan& p) {
  // dT (contraction d_out) and T (contraction d_in) share the first launch
  // and its split count, which the longer contraction sets for the row
  // tiles of both jobs; the longer job goes first in the grid
  const int64_t both_tiles = 2 * ((M + 127) / 128);
  pick_skinny(M, d_out, r, true, OUT_ROWS_RPAD, both_tiles, sm_count, p.dt_cfg);
  pick_skinny(M, d_in, r, false, OUT_ROWS_RPAD, both_tiles, sm_count, p.t_cfg);
  const int s1 = d_out >= d_in ? p.dt_cfg.splits : p.t_cfg.splits;
  resplit_skinny(p.dt_cfg, s1);
  resplit_skinny(p.t_cfg, s1);
  pick_skinny(M, d_out, r, true, OUT_ROWS_RPAD, (M + 127) / 128, sm_count, p.dto_cfg);
  // dB and dA share one launch, so they share its split count
  const int64_t dbda_tiles = (d_out + 127) / 128 + (d_in + 127) / 128;
  pick_skinny(d_out, M, r, true, OUT_ROWS_R, dbda_tiles, sm_count, p.db_cfg);
  pick_skinny(d_in, M, r, true, OUT_COLS_R, dbda_tiles, sm_count, p.da_cfg);
  const BwdWorkspace w = bwd_workspace(M, r);
  p.off_t = w.off_t;                                   // T   bf16 [M, r_pad]
  p.off_dt = w.off_dt;                                 // dT  bf16 [M, r_pad]
  p.total = w.total;
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

lora_status_t run_merge(const MergeItem* items, int n, int32_t r, float scale, int sm_count, cudaStream_t st) {
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
    tab.scale = scale;
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
