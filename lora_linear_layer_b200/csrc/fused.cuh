// fused.cuh - the fused LoRA GEMMs on tcgen05.
//
// One kernel serves two steps of the layer:
//   forward  (MN = false): OUT = P Q^T + (s P U^T) V^T with P = X[M,d_in],
//                          Q = W[d_out,d_in], U = A[r,d_in], V = B[d_out,r],
//                          all operands K-major:
//                          OUT = Y = X W^T + s (X A^T) B^T
//   dX       (MN = true):  OUT = [P | U] [Q ; V] with P = dY[M,d_out],
//                          Q = W[d_out,d_in], U = dT[M,r_pad] (the bf16
//                          s dY B of the backward's first pass, K-major) and
//                          V = A[r,d_in], read MN-major:
//                          OUT = dX = dY W + dT A, one accumulator, one
//                          rounding.  The rank-side product is just 1 or 2
//                          more K blocks of the same K loop.
// (fastaf 0.1.0, "FWD kernel speedup": base product plus the down- and
// up-projections, scale and add; "BWD kernel speedup": the dX kernel.)
//
// Forward, per output tile of (128 * CG) x BN:
//   * the K loop streams P, Q (and, on the first tile a cluster takes from an
//     M block, U) through a TMA -> shared-memory ring; one thread issues
//     tcgen05.mma for the base product into a TMEM accumulator and, on that
//     first tile, the N = r product T = P U^T into a second TMEM region;
//   * four epilogue warps drain T, scale it by s in fp32, round to bf16 and
//     write it into shared memory in the UMMA K-major swizzled layout; when
//     the caller asks for T (t_out), the tile of N index 0 of each M block
//     also writes the unscaled T, rounded to bf16, to global memory for the
//     backward (every M block's tile 0 is the first tile of a run, so T is
//     in the epilogue's registers there);
//   * the tile's V rows arrive through the same ring, as one more stage
//     after its K blocks; one more MMA pass (K = r) accumulates (sT) V^T
//     onto the base accumulator; the epilogue rounds once to bf16 and
//     writes OUT with TMA stores of 32 x 32 boxes staged in shared memory.
// T is kept in shared memory and reused for every following tile of the
// same M block (the schedule gives a cluster runs of consecutive N tiles of
// one M block).  dX tiles have none of the T, U, V steps and take single-tile
// runs.  Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer and TMEM
// owner, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4)...).
//
// BN = 224 (forward, CTA pairs, r_pad <= 32): the pair fold.  The odd CTA's
// Q slot holds the tile's W rows [128, 224) and 32 rows of U, so the
// tile's one N = 256 MMA per K step yields the base product in accumulator
// columns [0, 224) and T in [224, 256): no separate N = r products, at the
// price of 32 of every 256 columns.  Used where few tiles per pair would
// each compute T.
//
// CG = 2 runs each tile on a CTA pair (a cluster of two, cta_group::2):
// each CTA holds its own 128 rows of P and half of the Q/U/V rows, the even
// CTA issues every MMA (M = 256) for both, and each CTA keeps its 128 rows
// of every accumulator in its own TMEM.  The pair's TMA loads count their
// bytes on the even CTA's barriers; tcgen05.commit arrives on both CTAs'
// barriers; the odd CTA's epilogue arrives on the even CTA's barriers
// through shared::cluster addresses.  No load is multicast.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "texchange.cuh"

namespace lora {

constexpr int kBM = 128;          // rows per CTA (UMMA M per CTA)
constexpr int kBK = 64;           // K per pipeline stage (128 bytes of bf16)
constexpr int kFusedThreads = 192;
// Pair tile with T folded into the base product: 224 output columns and the
// 32 columns of T in one N = 256 MMA (forward, CTA pairs, r_pad <= 32).
constexpr int kPairFoldBN = 224;
constexpr int kPairFoldT = 32;
constexpr int kEpCols = 32;                    // output columns per epilogue store
constexpr uint32_t kEpBufBytes = 32u * kEpCols * 2u;  // one warp's 32 rows, 64-byte swizzle

struct FusedArgs {
  int32_t M, N, K;          // OUT is [M, N]; contraction length K
  int32_t r_pad;            // rank rounded up to 16 (UMMA N of the T product)
  int32_t n_rchunks;        // r_pad / RCW rounded up
  int32_t stages;           // pipeline depth
  int32_t ep_bufs;          // output staging buffers per epilogue warp (1 or 2)
  float scale;              // s = alpha / r (forward)
  __nv_bfloat16* out;       // [M, N] row-major, ld = N
  __nv_bfloat16* t_out;     // forward: NULL, or T = P U^T as bf16 [M, r_pad], ld = r_pad
  int32_t num_m, num_n;     // tile counts (M tiles of 128 * CG rows)
  int32_t band_w, n_bands;  // column bands of the schedule
  int32_t run_l;            // 0: contiguous ranges; L > 0: runs of L N-tiles dealt round-robin
  int32_t seeded;           // with run_l: 0 = runs cover every N tile; 1 = one seeding run of run_l
                            // tiles per cluster, then every other tile round-robin (see TileSched)
  TxSlot* tx;               // forward: exchange slot the clusters share T through (texchange.cuh), or NULL
  uint64_t wait_limit_ns;
};

// Byte sizes / offsets of one CTA's shared-memory carve-up (host and device).
struct FusedLayout {
  uint32_t p_bytes, q_bytes, u_bytes, stage_bytes, v_bytes, st_bytes, ep_bytes;
  uint32_t off_st, off_ep, off_bar, total;
  __host__ __device__ FusedLayout(int BN, int CG, bool mn, int rcw, int r_pad, int n_rchunks, int stages,
                                  int ep_bufs) {
    // Q / V rows held by this CTA (the 224-wide pair tile: 128 in each CTA,
    // of which the odd CTA's last 32 are rows of U)
    const int bnc = BN == kPairFoldBN ? 128 : BN / CG;
    p_bytes = kBM * kBK * 2;
    q_bytes = uint32_t(bnc * kBK * 2);
    // the dX form streams its rank-side operands through the ring; the
    // 224-wide pair tile holds U in its Q slot
    u_bytes = (mn || BN == kPairFoldBN) ? 0u : uint32_t((r_pad / CG) * 128);
    stage_bytes = p_bytes + q_bytes + u_bytes;
    // V (the up-projection's rank-side operand of one N tile) travels
    // through the ring as one more stage per tile: all its chunks fit in a
    // stage's P and Q slots (v_bytes <= p_bytes + q_bytes for r_pad <= 128)
    v_bytes = mn ? 0u : uint32_t(n_rchunks * bnc * rcw * 2);
    st_bytes = mn ? 0u : uint32_t(n_rchunks * kBM * rcw * 2);
    ep_bytes = 4u * uint32_t(ep_bufs) * kEpBufBytes;
    off_st = stage_bytes * stages;
    off_ep = off_st + st_bytes;
    off_bar = off_ep + ep_bytes;
    total = off_bar + 256;
  }
};

// Tile schedule over clusters (one cluster = CG CTAs = one tile at a time).
//  run_l == 0: the N tiles are grouped into column bands; the tiles of a band
//    are ordered M-major (N fastest) and split into G contiguous ranges, so a
//    cluster sweeps N inside one or two M blocks per band.
//  run_l > 0: "runs" of run_l consecutive N tiles of one M block, ordered
//    M-major, are dealt round-robin to the clusters: the tiles in flight at
//    any time cover only ~G*run_l/num_n M blocks (compact L2 footprint),
//    and T is computed once per run.
//  run_l > 0, seeded: two phases, for launches whose clusters share T
//    through the exchange (texchange.cuh).  Seeding: cluster c runs
//    run_l N tiles of M block c % num_m from N tile run_l * (c / num_m),
//    so every M block's T is computed (and published) at the start, by at
//    least one cluster when there are at least num_m clusters (the seeding
//    stays inside the first column band).  Then every tile the seeding left
//    over is dealt round-robin, band by band and M-major inside a band, as
//    in the dX form: the tiles in flight cover only a few M blocks and the
//    W tiles of one band, the operands stay in L2, and each of these tiles
//    copies its M block's s T instead of computing it.
struct TileSched {
  int num_m, num_n, band_w, n_bands, run_l, G, c;
  int band, t, t_end, band_n0, w;
  int runs_per_m, run, run_end, run_pos, run_len, run_m, run_n0;
  // seeded schedule: first-class blocks (m < r0) and their leftover tiles
  // per block in the first band (w0 wide), the other blocks' count, the
  // first band's leftover total, the next round-robin index, the total
  int seeded, r0, c_hi, c_lo, w0, p0, rr_i, rr_end;
  bool main_done;
  __device__ TileSched(const FusedArgs& a, int G_, int c_)
      : num_m(a.num_m), num_n(a.num_n), band_w(a.band_w), n_bands(a.n_bands), run_l(a.run_l), G(G_), c(c_),
        band(-1), t(0), t_end(0), band_n0(0), w(1), runs_per_m(1), run(0), run_end(0), run_pos(0), run_len(0),
        run_m(0), run_n0(0), seeded(a.seeded), r0(0), c_hi(0), c_lo(0), w0(0), p0(0), rr_i(0), rr_end(0),
        main_done(false) {
    if (run_l > 0 && seeded) {
      // clusters with c % num_m == m seed M block m: a(m) runs of run_l
      // (the host keeps every seeding run inside the first band; the kernel
      // clips a run at the last N tile in any case)
      const int a_lo = G / num_m;
      r0 = G % num_m;  // blocks m < r0 have a_lo + 1 seeding runs
      w0 = imin(band_w, num_n);
      c_hi = w0 - imin(w0, (a_lo + 1) * run_l);
      c_lo = w0 - imin(w0, a_lo * run_l);
      rr_i = c;
      p0 = r0 * c_hi + (num_m - r0) * c_lo;
      rr_end = p0 + num_m * (num_n - w0);
    } else if (run_l > 0) {
      runs_per_m = (num_n + run_l - 1) / run_l;
      run = c - G;
      run_end = num_m * runs_per_m;
    }
  }
  __device__ bool next(int& m, int& n) {
    if (run_l > 0 && seeded) {
      if (!main_done) {
        // the seeding run (empty when it would start past the last N tile)
        const int n0 = run_l * (c / num_m);
        if (run_pos < imin(run_l, num_n - n0)) {
          m = c % num_m;
          n = n0 + run_pos++;
          return true;
        }
        main_done = true;
      }
      if (rr_i >= rr_end) return false;
      const int i = rr_i;
      rr_i += G;
      if (i < r0 * c_hi) {  // first band, blocks with one more seeding run
        m = i / c_hi;
        n = w0 - c_hi + i % c_hi;
      } else if (i < p0) {  // first band, the other blocks
        const int j = i - r0 * c_hi;
        m = r0 + j / c_lo;
        n = w0 - c_lo + j % c_lo;
      } else {              // later bands, whole, M-major (only the last may be narrower)
        const int j = i - p0;
        const int b = 1 + j / (num_m * band_w);
        const int jb = j - (b - 1) * num_m * band_w;
        const int wb = imin(band_w, num_n - b * band_w);
        m = jb / wb;
        n = b * band_w + jb % wb;
      }
      return true;
    }
    if (run_l > 0) {
      if (run_pos >= run_len) {
        run += G;
        if (run >= run_end) return false;
        run_m = run / runs_per_m;
        run_n0 = (run % runs_per_m) * run_l;
        run_len = imin(run_l, num_n - run_n0);
        run_pos = 0;
      }
      m = run_m;
      n = run_n0 + run_pos++;
      return true;
    }
    while (t >= t_end) {
      if (++band >= n_bands) return false;
      band_n0 = band * band_w;
      w = imin(band_w, num_n - band_n0);
      const long long T = (long long)num_m * w;
      const int cc = (c + band * 37) % G;  // rotate who gets the longer ranges
      t = int(T * cc / G);
      t_end = int(T * (cc + 1) / G);
    }
    m = t / w;
    n = band_n0 + t % w;
    ++t;
    return true;
  }
};

// PTX forms by CTA-group size.
template <int CG>
struct Group;

template <>
struct Group<1> {
  static __device__ __forceinline__ void alloc(uint32_t slot, uint32_t n) {
    tmem_alloc(slot, n);
    tmem_relinquish();
  }
  static __device__ __forceinline__ void dealloc(uint32_t t, uint32_t n) { tmem_dealloc(t, n); }
  static __device__ __forceinline__ void load(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int c0, int c1) {
    tma_load_2d(dst, tm, bar, c0, c1);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_bf16(d, a, b, id, acc);
  }
  static __device__ __forceinline__ void commit_all(uint32_t bar) { umma_commit(bar); }
  static __device__ __forceinline__ void commit_local(uint32_t bar) { umma_commit(bar); }
  static __device__ __forceinline__ uint32_t leader_addr(uint32_t bar) { return bar; }
  static __device__ __forceinline__ void arrive_leader(uint32_t bar) { mbar_arrive(bar); }
  static __device__ __forceinline__ void cluster_sync() {}
};

template <>
struct Group<2> {
  static __device__ __forceinline__ void alloc(uint32_t slot, uint32_t n) {
    tmem_alloc_pair(slot, n);
    tmem_relinquish_pair();
  }
  static __device__ __forceinline__ void dealloc(uint32_t t, uint32_t n) { tmem_dealloc_pair(t, n); }
  static __device__ __forceinline__ void load(uint32_t dst, const CUtensorMap* tm, uint32_t bar_leader, int c0,
                                              int c1) {
    tma_load_2d_pair(dst, tm, bar_leader, c0, c1);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_bf16_pair(d, a, b, id, acc);
  }
  static __device__ __forceinline__ void commit_all(uint32_t bar) { umma_commit_pair_mc(bar, uint16_t(3)); }
  static __device__ __forceinline__ void commit_local(uint32_t bar) { umma_commit_pair(bar); }
  static __device__ __forceinline__ uint32_t leader_addr(uint32_t bar) { return mapa_shared(bar, 0); }
  static __device__ __forceinline__ void arrive_leader(uint32_t bar) { mbar_arrive_cluster(mapa_shared(bar, 0)); }
  static __device__ __forceinline__ void cluster_sync() { cluster_barrier_sync(); }
};

// TX: the forward with an exchange slot (texchange.cuh); its steps are
// compiled only into these instances, so a launch without a slot runs a
// kernel with none of them (a smaller kernel: the tiny forward measured
// 1-2 us slower with the exchange code compiled in but not taken).
template <int BN, bool MN, int RCW, int CG, bool TX>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_lora_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmQ2,
                      const FusedArgs a) {
  static_assert(BN == 128 || BN == 256 || (BN == kPairFoldBN && CG == 2 && !MN), "BN");
  static_assert(CG == 1 || CG == 2, "CG");
  static_assert(RCW == 16 || RCW == 32 || RCW == 64, "RCW");
  static_assert(!(TX && MN), "the exchange is a forward feature");
  constexpr bool kQmn = MN;             // Q read MN-major
  using G = Group<CG>;
  // 224-wide pair tile (kPairFoldBN): the even CTA holds Q rows [0, 128) of
  // the tile, the odd one Q rows [128, 224) and U's rows, so one N = 256
  // MMA puts the base product in accumulator columns [0, 224) and T in
  // [224, 256) (the single-CTA fold's idea on the pair; tmQ2 is Q with a
  // 96-row box)
  constexpr bool kPF = BN == kPairFoldBN;
  constexpr int BNC = kPF ? 128 : BN / CG;  // Q / V rows held by this CTA
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;  // bytes per swizzled rank row
  constexpr bool kClusterScope = CG > 1;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);

  const FusedLayout L(BN, CG, MN, RCW, a.r_pad, a.n_rchunks, a.stages, a.ep_bufs);
  const int S = a.stages;
  const uint32_t bar0 = sbase + L.off_bar;
  // barrier map (8 bytes each); full / accempty / stfull / drain are used
  // on the even CTA only
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t accfull0 = bar0 + 8u * (2 * S + 0);   // +8*b
  const uint32_t accempty0 = bar0 + 8u * (2 * S + 2);  // +8*b
  const uint32_t tfull = bar0 + 8u * (2 * S + 4);
  const uint32_t stfull = bar0 + 8u * (2 * S + 5);
  const uint32_t drain = bar0 + 8u * (2 * S + 6);
  const uint32_t txbar = bar0 + 8u * (2 * S + 7);      // a T tile's mode message is in tx_msg
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 8 * (2 * S + 8));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // T tile mode message from the MMA thread to the epilogues of both CTAs:
  // 1 = copy s T from the exchange, 0 = compute it
  volatile uint32_t* const tx_msg = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
  // from the (leader's) producer to the MMA thread, published by its arrive
  // on a T tile's first stage: each T tile's mode, in a ring (the producer
  // runs at most `stages` stages, so fewer than 8 T tiles, ahead)
  volatile uint8_t* const tx_mode = reinterpret_cast<volatile uint8_t*>(tmem_slot + 3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG > 1 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accfull0, 1);
    mbar_init(accfull0 + 8, 1);
    mbar_init(accempty0, 4 * CG);
    mbar_init(accempty0 + 8, 4 * CG);
    mbar_init(tfull, 1);
    mbar_init(stfull, 4 * CG);
    mbar_init(drain, 1);
    mbar_init(txbar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmV);
    if constexpr (kPF) tma_prefetch_desc(&tmQ2);
  }
  if (warp == 2 && lane == 0) tma_prefetch_desc(&tmO);
  if (warp == 1) G::alloc(smem_addr(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  G::cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above touches no global memory, so it may overlap the
  // previous kernel on the stream; every global access comes after the wait.
  griddep_launch_dependents();
  griddep_wait();

  // T placement.  128-wide single-CTA forward tiles fold T into the base
  // product: U's rows follow Q's rows in the stage, so one MMA with
  // N = BN + r_pad covers both, and each accumulator buffer is BN + r_pad
  // columns wide with T in its last r_pad.  The 224-wide pair tile does the
  // same on the pair: its accumulators are 256 columns wide, T in the last
  // 32 (every MMA of its K loop has N = 256).  Otherwise T gets its own
  // columns if two BN-wide accumulators and r_pad columns fit in 512, else
  // it borrows the other accumulator.
  constexpr bool kFold = CG == 1 && BN == 128 && !MN;
  const uint32_t acc_stride = kFold ? uint32_t(BN + a.r_pad) : kPF ? uint32_t(BN + kPairFoldT) : uint32_t(BN);
  const bool borrow = !MN && !kFold && !kPF && (2 * BN + a.r_pad) > 512;
  const int nk = (a.K + kBK - 1) / kBK;
  // dX: K blocks [nk, nk_all) hold the rank-side product dT A
  const int nk_all = MN ? nk + (a.r_pad + kBK - 1) / kBK : nk;
  const uint64_t lim = a.wait_limit_ns;
  const int n_clusters = int(gridDim.x) / CG;
  const int cluster_id = int(blockIdx.x) / CG;
  const int u_rows = a.r_pad / CG;        // U rows held by this CTA
  const uint32_t tx_full = (1u << (4 * CG)) - 1u;  // every epilogue warp of the cluster has published
  TxSlot* const tx = TX ? a.tx : nullptr;  // a compile-time NULL without TX

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      TileSched sch(a, n_clusters, cluster_id);
      int m, n, prev_m = -1, stage = 0;
      uint32_t phase = 0, ntp = 0;
      bool ok = true;
      while (ok && sch.next(m, n)) {
        const bool ttile = !MN && (m != prev_m);
        prev_m = m;
        if (ttile && leader && tx != nullptr) {
          // copy s T when another cluster has published this M block's
          // (checked here, a few stages ahead of the MMA thread)
          tx_mode[ntp & 7u] = ld_acquire_gpu(&tx->flags[m]) == tx_full ? 1 : 0;
          ++ntp;
        }
        const uint32_t bytes = L.p_bytes + L.q_bytes + (ttile ? L.u_bytes : 0u);
        const int row0 = m * (kBM * CG) + int(rank) * kBM;
        const int qrow0 = n * BN + int(rank) * BNC;  // (the pair fold's odd CTA: its first W row)
        for (int kb = 0; kb < nk_all; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY, kClusterScope)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
          const uint32_t fb = G::leader_addr(full_bar(stage));
          if (leader) mbar_arrive_expect_tx(full_bar(stage), bytes * CG);
          // Each branch names its tensor maps directly: selecting between
          // two kernel-parameter maps through a pointer makes every load take
          // its descriptor from a runtime address, which measured ~10% slower
          // (8192 x 4096 x 4096 dX: 181 vs 162 us without the tail block).
          if (!MN || kb < nk) {
            const int k0 = kb * kBK;
            G::load(st, &tmP, fb, k0, row0);
            if (kPF) {
              if (rank == 0) {
                G::load(st + L.p_bytes, &tmQ, fb, k0, qrow0);
              } else {
                G::load(st + L.p_bytes, &tmQ2, fb, k0, qrow0);
                G::load(st + L.p_bytes + uint32_t((128 - kPairFoldT) * 128), &tmU, fb, k0, 0);
              }
            } else if (!kQmn) {
              G::load(st + L.p_bytes, &tmQ, fb, k0, qrow0);
            } else {
#pragma unroll
              for (int i = 0; i < BNC / 64; ++i)
                G::load(st + L.p_bytes + uint32_t(i) * 8192u, &tmQ, fb, qrow0 + 64 * i, k0);
            }
            if (!kPF && ttile) G::load(st + L.p_bytes + L.q_bytes, &tmU, fb, k0, int(rank) * u_rows);
          } else {
            // dX tail: dT and A in place of dY and W (columns of dT and rows
            // of A past r_pad come from the tensor maps' zero fill)
            const int k0 = (kb - nk) * kBK;
            G::load(st, &tmU, fb, k0, row0);
#pragma unroll
            for (int i = 0; i < BNC / 64; ++i)
              G::load(st + L.p_bytes + uint32_t(i) * 8192u, &tmV, fb, qrow0 + 64 * i, k0);
          }
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (MN) continue;
        // rank-side operand of the up-projection for this N tile: one more
        // ring stage, its RCW-wide chunks side by side from the stage base
        if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY, kClusterScope)) break;
        const uint32_t sv = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t vb = G::leader_addr(full_bar(stage));
        if (leader) mbar_arrive_expect_tx(full_bar(stage), L.v_bytes * CG);
        for (int c = 0; c < a.n_rchunks; ++c)
          G::load(sv + uint32_t(c) * uint32_t(BNC * kRSpan), &tmV, vb, c * RCW, qrow0);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (*abort_flag) settle_ns(200000);  // let copies in flight land
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0 && leader) {
      const uint32_t id_base = idesc_bf16(kBM * CG, kPF ? BN + kPairFoldT : BN, false, kQmn);
      const uint32_t id_tail = idesc_bf16(kBM * CG, BN, false, true);  // dX: V = A is MN-major
      const uint32_t id_t = idesc_bf16(kBM * CG, a.r_pad, false, false);
      const uint32_t id_up = idesc_bf16(kBM * CG, kPF ? BN + kPairFoldT : BN, false, MN);
      const uint32_t id_fold = idesc_bf16(kBM * CG, BN + a.r_pad, false, false);
      TileSched sch(a, n_clusters, cluster_id);
      int m, n, prev_m = -1, stage = 0;
      uint32_t phase = 0, ntt = 0, tcount = 0;
      uint32_t acc_waits0 = 0u, acc_waits1 = 0u;  // completed waits per accumulator
      auto next_acc_parity = [&](uint32_t buf) {
        const uint32_t k = buf ? acc_waits1++ : acc_waits0++;
        return (k & 1u) ^ 1u;
      };
      bool ok = true;
      while (ok && sch.next(m, n)) {
        const bool ttile = !MN && (m != prev_m);
        prev_m = m;
        // A T tile copies s T from the exchange when the producer found this
        // M block's published, else computes T; both CTAs' epilogues are
        // told which (the previous T tile's message has been read: its
        // stfull wait came after).  The producer's choice is visible once
        // the tile's first stage is full.
        // (launches without an exchange slot take none of these steps)
        bool tload = false;
        if (ttile && tx != nullptr) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL, kClusterScope)) break;
          tload = tx_mode[ntt & 7u] != 0;
          const uint32_t msg = tload ? 1u : 0u;
          *tx_msg = msg;
          if constexpr (CG > 1) {
            st_shared_cluster_u32(mapa_shared(smem_addr(const_cast<uint32_t*>(tx_msg)), 1u), msg);
            mbar_arrive_cluster(mapa_shared(txbar, 1u));
          }
          mbar_arrive(txbar);
        }
        const bool tcomp = ttile && !tload;
        const uint32_t b = tcount & 1u;
        if (!wait_bounded(accempty0 + 8u * b, next_acc_parity(b), abort_flag, lim, SITE_ACCEMPTY, kClusterScope))
          break;
        uint32_t t_col = (kFold || kPF) ? b * acc_stride + BN : 2u * BN;
        if (tcomp && borrow) {
          const uint32_t ob = b ^ 1u;
          if (!wait_bounded(accempty0 + 8u * ob, next_acc_parity(ob), abort_flag, lim, SITE_ACCEMPTY,
                            kClusterScope))
            break;
          t_col = ob * BN;
        }
        tc_fence_after();
        const uint32_t d_acc = tmem + b * acc_stride;
        // The K loop, instantiated twice: with the N = r products of T (first
        // tile of an M block) and without.  Keeping the plain loop free of
        // the second MMA stream, and issuing the T products after the base
        // products of each stage rather than interleaved with them, keeps
        // the tensor pipe fed (measured: 242 -> 216 us on 8192x4096x4096).
        auto k_loop = [&](auto with_t) -> bool {
          constexpr bool kWithT = decltype(with_t)::value;
          for (int kb = 0; kb < nk_all; ++kb) {
            if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL, kClusterScope)) return false;
            tc_fence_after();
            const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
            const uint32_t sq = st + L.p_bytes;
            if (!MN || kb < nk) {
              // fully unrolled (a data-dependent trip count here measured
              // 206 vs 185 us on the 8192 x 4096 x 4096 dX)
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint64_t ad = smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B);
                const uint64_t bd = kQmn ? smem_desc(sq + kk * 2048u, 8192u, 1024u, SWZ_128B)
                                         : smem_desc(sq + kk * 32u, 16u, 1024u, SWZ_128B);
                G::mma(d_acc, ad, bd, (kFold && kWithT) ? id_fold : id_base, (kb | kk) != 0);
              }
            } else {
              // dX tail block: A is MN-major; stop at r_pad (the rest is zero fill)
              const int kk_n = imin(kBK / 16, (a.r_pad - (kb - nk) * kBK) / 16);
              for (int kk = 0; kk < kk_n; ++kk)
                G::mma(d_acc, smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B),
                       smem_desc(sq + kk * 2048u, 8192u, 1024u, SWZ_128B), id_tail, 1u);
            }
            if constexpr (kWithT && !kFold && !kPF) {
              const uint32_t su = sq + L.q_bytes;
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                G::mma(tmem + t_col, smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B),
                       smem_desc(su + kk * 32u, 16u, 1024u, SWZ_128B), id_t, (kb | kk) != 0);
            }
            G::commit_all(empty_bar(stage));
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
          return true;
        };
        ok = tcomp ? k_loop(std::true_type{}) : k_loop(std::false_type{});
        if (!ok) break;
        if (MN) {
          G::commit_all(accfull0 + 8u * b);
          ++tcount;
          continue;
        }
        if (ttile) {
          if (tcomp) G::commit_all(tfull);
          if (!wait_bounded(stfull, ntt & 1u, abort_flag, lim, SITE_STFULL, kClusterScope)) break;
          ++ntt;
        }
        if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL, kClusterScope)) break;
        tc_fence_after();
        const uint32_t s_t = sbase + L.off_st;
        const uint32_t s_v = sbase + uint32_t(stage) * L.stage_bytes;  // this tile's V stage
        for (int kk = 0; kk < a.r_pad / 16; ++kk) {
          const uint32_t c = uint32_t(kk * 16) / RCW;
          const uint32_t off = uint32_t((kk * 16) % RCW) * 2u;
          const uint64_t ad = smem_desc(s_t + c * uint32_t(kBM * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          const uint64_t bd = smem_desc(s_v + c * uint32_t(BNC * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          G::mma(d_acc, ad, bd, id_up, 1u);
        }
        G::commit_all(empty_bar(stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
        G::commit_all(accfull0 + 8u * b);
        ++tcount;
      }
      // make sure no tcgen05 op is still running before TMEM is released
      G::commit_local(drain);
      wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN, false);
    }
  } else {
    // ---------------------------------------------------- epilogue ----
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int row = q * 32 + lane;     // tile row owned by this thread
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    TileSched sch(a, n_clusters, cluster_id);
    int m, n, prev_m = -1;
    uint32_t ntt = 0, ntc = 0, tcount = 0;  // T tiles; T tiles that computed T
    uint32_t full_waits0 = 0u, full_waits1 = 0u;  // completed accfull waits per buffer
    uint8_t* const st_ptr = gbase + L.off_st;
    // this warp's output staging buffers (used in turn when there are two)
    const uint32_t ep_off = L.off_ep + uint32_t(q * a.ep_bufs) * kEpBufBytes;
    uint32_t epc = 0;  // output blocks staged so far
    while (sch.next(m, n)) {
      const bool ttile = !MN && (m != prev_m);
      prev_m = m;
      const uint32_t b = tcount & 1u;
      if (ttile) {
        // the MMA thread's message: compute T (and publish it) or copy it
        // (without an exchange slot, always compute)
        bool tload = false;
        if (tx != nullptr) {
          if (!warp_wait_bounded(txbar, ntt & 1u, abort_flag, lim, SITE_TXMSG, kClusterScope)) break;
          ++ntt;
          tload = (*tx_msg & 1u) != 0u;
        }
        const int t_row = m * (kBM * CG) + int(rank) * kBM + row;
        if (!tload) {
          if (!warp_wait_bounded(tfull, ntc & 1u, abort_flag, lim, SITE_TFULL, kClusterScope)) break;
          ++ntc;
          tc_fence_after();
          const uint32_t t_col = (kFold || kPF) ? b * acc_stride + BN : borrow ? (b ^ 1u) * BN : 2u * BN;
          // every tile that computes T stores it for the backward when asked
          // (the same values whichever tile of the M block does)
          __nv_bfloat16* const t_dst =
              a.t_out != nullptr && t_row < a.M ? a.t_out + size_t(t_row) * size_t(a.r_pad) : nullptr;
          __nv_bfloat16* const x_dst = tx != nullptr ? tx->t + size_t(t_row) * size_t(a.r_pad) : nullptr;
#pragma unroll 1
          for (int col = 0; col < a.r_pad; col += 16) {
            uint32_t v[16];
            tmem_ld_x16(tmem + lane_base + t_col + uint32_t(col), v);
            tmem_ld_wait();
            if (t_dst != nullptr) {
              uint32_t tu[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                tu[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              uint4* d = reinterpret_cast<uint4*>(t_dst + col);
              d[0] = make_uint4(tu[0], tu[1], tu[2], tu[3]);
              d[1] = make_uint4(tu[4], tu[5], tu[6], tu[7]);
            }
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * a.scale, __uint_as_float(v[2 * i + 1]) * a.scale);
            const uint4 lo = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            const uint4 hi = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            const int c = col / RCW;
            const int cin = (col % RCW) / 8;  // 16-byte chunk inside the rank row
            uint8_t* chunk = st_ptr + c * (kBM * kRSpan);
            *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin, kRSpan)) = lo;
            *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin + 1, kRSpan)) = hi;
            if (x_dst != nullptr) {
              uint4* d = reinterpret_cast<uint4*>(x_dst + col);
              d[0] = lo;
              d[1] = hi;
            }
          }
          if (tx != nullptr) {
            // publish: this warp's 32 rows of s T are in the exchange
            __threadfence();
            __syncwarp();
            if (lane == 0) atom_or_release_gpu(&tx->flags[m], 1u << (int(rank) * 4 + q));
          }
        } else {
          // another cluster published this M block's s T (the MMA thread saw
          // its flag complete): copy this thread's row into shared memory
          if (!wait_word_bounded(&tx->flags[m], tx_full, abort_flag, lim, SITE_TXFLAG)) break;
          const __nv_bfloat16* const src = tx->t + size_t(t_row) * size_t(a.r_pad);
          // kept rolled: unrolled, this loop took the kernel from about 100 to
          // 210 registers and the tiny forward 1-2 us slower
#pragma unroll 1
          for (int col = 0; col < a.r_pad; col += 16) {
            const uint4 lo = ld_global_cg_v4(src + col);
            const uint4 hi = ld_global_cg_v4(src + col + 8);
            const int c = col / RCW;
            const int cin = (col % RCW) / 8;
            uint8_t* chunk = st_ptr + c * (kBM * kRSpan);
            *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin, kRSpan)) = lo;
            *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin + 1, kRSpan)) = hi;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          G::arrive_leader(stfull);
          if (borrow && !tload) G::arrive_leader(accempty0 + 8u * (b ^ 1u));
        }
      }
      const uint32_t fpar = (b ? full_waits1++ : full_waits0++) & 1u;
      if (!warp_wait_bounded(accfull0 + 8u * b, fpar, abort_flag, lim, SITE_ACCFULL, kClusterScope)) break;
      tc_fence_after();
      const uint32_t acc_col = b * acc_stride;
      // Each 32-column chunk: TMEM -> registers -> bf16 -> this warp's
      // swizzled staging buffer -> one TMA store of 32 rows x 64 bytes
      // (rows past M and columns past N are clipped by the tensor map).
      const int wrow0 = m * (kBM * CG) + int(rank) * kBM + q * 32;
#pragma unroll 1
      for (int ch = 0; ch < BN / kEpCols; ++ch) {
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_base + acc_col + uint32_t(ch * kEpCols), v);
        tmem_ld_wait();
        const int col0 = n * BN + ch * kEpCols;
        if (col0 >= a.N || wrow0 >= a.M) continue;
        uint4 pk[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          pk[g].x = pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1]));
          pk[g].y = pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3]));
          pk[g].z = pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5]));
          pk[g].w = pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7]));
        }
        // the store that last used this buffer has read it
        if (lane == 0) {
          if (a.ep_bufs == 2) bulk_wait_group_read1();
          else bulk_wait_group_read0();
        }
        __syncwarp();
        const uint32_t bo = ep_off + (a.ep_bufs == 2 ? (epc & 1u) * kEpBufBytes : 0u);
        ++epc;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4*>(gbase + bo + swz_offset(uint32_t(lane), uint32_t(g), kEpCols * 2)) = pk[g];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmO, sbase + bo, col0, wrow0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) G::arrive_leader(accempty0 + 8u * b);
      ++tcount;
    }
    if (lane == 0) bulk_wait_group0();  // every output store has completed
  }

  tc_fence_before();
  __syncthreads();
  G::cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    G::dealloc(tmem, 512);
  }
  if (warp == 0 && leader && tx != nullptr) {
    // every role of both CTAs is done with the exchange slot
    __syncwarp();
    tx_finish(tx, n_clusters, a.num_m, lane);
  }
}

}  // namespace lora
