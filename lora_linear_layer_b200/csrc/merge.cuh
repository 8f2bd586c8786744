// merge.cuh - W_dst = bf16_rne(W_src + s * B A) for a table of matrices.
//
// unsloth fork commit log (scripts/benchmarks/qwen3_flex_inference.py): the
// refresh merges each LoRA target from its pristine base in one pass,
// addmm(pristine, B, A, alpha=scaling, out=W_inf), with the rank-r product
// accumulated in fp32 and rounded once; restoring from pristine keeps the
// base bit-identical across refreshes.
//
// A persistent kernel: CTA c processes the 128 x 128 tiles c, c + G, ... of
// the table (G CTAs, one per SM) through a ring of shared-memory stages.
// Per tile, TMA brings the W_src tile (two 64-column SW128 boxes), the B rows
// [128, r] (K-major, K = r) and the A columns [r, 128] (MN-major) into one
// stage; one thread issues the r/16 tcgen05.mma steps of the K = r product
// into one of two TMEM accumulators; eight epilogue warps read the fp32
// product row by row, add s * product to the W_src value in fp32, round once
// to bf16, write the result over the W_src tile in the same stage (same
// swizzled place) and TMA-store it to W_dst.  Loads of later tiles, the MMA
// of the next tile and the stores of this one overlap.  A tile is read
// completely before it is written and tiles are disjoint, so W_dst == W_src
// works.  The kernel is bound by HBM traffic (read W_src, write W_dst).
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kMergeBN = 128;
constexpr int kMergeMaxJobs = 48;
constexpr int kMergeMaxStages = 6;

struct MergeJob {
  CUtensorMap w_src;  // [d_out, d_in], box {64, 128}, SW128
  CUtensorMap w_dst;  // [d_out, d_in], box {64, 32}, SW128 (per-warp stores)
  CUtensorMap a;      // A [r, d_in] read MN-major, box {64, r_pad}, SW128
  CUtensorMap b;      // B [d_out, r] read K-major, box {RCW, 128}
  int32_t tiles_n;    // column tiles of this matrix
  int32_t tile_begin; // first global tile index of this matrix
  int32_t rows, cols; // d_out, d_in
};

struct MergeTable {
  MergeJob job[kMergeMaxJobs];
  int32_t n_jobs;
  int32_t n_tiles;    // tiles of all jobs
  int32_t r_pad;
  int32_t n_rchunks;
  int32_t stages;
  float scale;
  uint64_t wait_limit_ns;
};

struct MergeLayout {
  uint32_t w_bytes, b_bytes, a_bytes, off_b, off_a, stage_bytes, off_bar, total;
  __host__ __device__ MergeLayout(int rcw, int r_pad, int n_rchunks, int stages) {
    w_bytes = 128 * kMergeBN * 2;                      // 32 KB
    b_bytes = uint32_t(n_rchunks * 128 * rcw * 2);
    a_bytes = uint32_t((kMergeBN / 64) * r_pad * 128);
    off_b = w_bytes;
    off_a = off_b + b_bytes;
    stage_bytes = (off_a + a_bytes + 1023u) & ~1023u;
    off_bar = stage_bytes * uint32_t(stages);
    total = off_bar + 256;
  }
};

// Where global tile t lies: its job (searching forward from job j), row and
// column offsets.
struct MergeTile {
  int j, m0, n0;
};
__device__ __forceinline__ MergeTile merge_tile(const MergeTable& tab, int j, int t) {
  while (j + 1 < tab.n_jobs && t >= tab.job[j + 1].tile_begin) ++j;
  const int lt = t - tab.job[j].tile_begin;
  return MergeTile{j, (lt / tab.job[j].tiles_n) * 128, (lt % tab.job[j].tiles_n) * kMergeBN};
}

constexpr int kMergeThreads = 320;  // producer, MMA, 8 epilogue warps

template <int RCW>
__global__ void __launch_bounds__(kMergeThreads, 1) merge_kernel(const __grid_constant__ MergeTable tab) {
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);
  const int S = tab.stages;
  const MergeLayout L(RCW, tab.r_pad, tab.n_rchunks, S);
  const uint32_t bar0 = sbase + L.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t accfull0 = bar0 + 8u * (2 * S);      // +8*b
  const uint32_t accempty0 = bar0 + 8u * (2 * S + 2);  // +8*b
  const uint32_t drain = bar0 + 8u * (2 * S + 4);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 8 * (2 * S + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = tab.wait_limit_ns;
  const int G = int(gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8u * b, 1);
      mbar_init(accempty0 + 8u * b, 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 2 * kMergeBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above touches no global memory, so it may overlap the
  // previous kernel on the stream; every global access comes after the wait.
  griddep_launch_dependents();
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      int stage = 0, j = 0;
      uint32_t phase = 0;
      for (int t = int(blockIdx.x); t < tab.n_tiles; t += G) {
        if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY)) break;
        const MergeTile mt = merge_tile(tab, j, t);
        j = mt.j;
        const MergeJob& job = tab.job[j];
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t fb = full_bar(stage);
        mbar_arrive_expect_tx(fb, L.w_bytes + L.b_bytes + L.a_bytes);
        tma_load_2d(st, &job.w_src, fb, mt.n0, mt.m0);
        tma_load_2d(st + 16384u, &job.w_src, fb, mt.n0 + 64, mt.m0);
        for (int c = 0; c < tab.n_rchunks; ++c)
          tma_load_2d(st + L.off_b + uint32_t(c) * (128u * kRSpan), &job.b, fb, c * RCW, mt.m0);
        tma_load_2d(st + L.off_a, &job.a, fb, mt.n0, 0);
        tma_load_2d(st + L.off_a + uint32_t(tab.r_pad) * 128u, &job.a, fb, mt.n0 + 64, 0);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (*abort_flag) settle_ns(200000);  // let copies in flight land
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, kMergeBN, false, true);
      int stage = 0;
      uint32_t phase = 0, k = 0;
      for (int t = int(blockIdx.x); t < tab.n_tiles; t += G, ++k) {
        const uint32_t b = k & 1u;
        if (!wait_bounded(accempty0 + 8u * b, ((k >> 1) & 1u) ^ 1u, abort_flag, lim, SITE_ACCEMPTY)) break;
        if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL)) break;
        tc_fence_after();
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t sb = st + L.off_b;
        const uint32_t sa = st + L.off_a;
        for (int kk = 0; kk < tab.r_pad / 16; ++kk) {
          const uint32_t c = uint32_t(kk * 16) / RCW;
          const uint32_t off = uint32_t((kk * 16) % RCW) * 2u;
          const uint64_t ad = smem_desc(sb + c * (128u * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          const uint64_t bd = smem_desc(sa + uint32_t(kk) * 2048u, uint32_t(tab.r_pad) * 128u, 1024u, SWZ_128B);
          umma_bf16(tmem + b * uint32_t(kMergeBN), ad, bd, idesc, kk != 0);
        }
        umma_commit(accfull0 + 8u * b);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      // make sure no tcgen05 op is still running before TMEM is released
      umma_commit(drain);
      wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN);
    }
  } else {
    // ---------------------------------------------------- epilogue ----
    // Eight warps: warp 2 + 4h + i handles TMEM lane quarter (warp % 4) of
    // the 64-column box h.
    const int h = (warp - 2) >> 2;
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    int stage = 0, j = 0, prev_stage = -1;
    uint32_t phase = 0, k = 0;
    for (int t = int(blockIdx.x); t < tab.n_tiles; t += G, ++k) {
      const uint32_t b = k & 1u;
      if (!warp_wait_bounded(accfull0 + 8u * b, (k >> 1) & 1u, abort_flag, lim, SITE_ACCFULL)) break;
      // the W_src tile of this stage has landed (and is visible to this warp)
      if (!warp_wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL)) break;
      tc_fence_after();
      const MergeTile mt = merge_tile(tab, j, t);
      j = mt.j;
      uint8_t* const box = gbase + stage * L.stage_bytes + h * 16384;
      for (int half = 0; half < 2; ++half) {     // 32 columns at a time
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_base + b * uint32_t(kMergeBN) + uint32_t(h * 64 + half * 32), v);
        tmem_ld_wait();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {         // 16-byte chunks of 8 values
          const int chunk = half * 4 + c4;
          uint4* p = reinterpret_cast<uint4*>(box + swz_offset(row, chunk, 128));
          uint4 w = *p;
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = fmaf(tab.scale, __uint_as_float(v[c4 * 8 + 2 * e]), bf16lo_to_f32(wv[e]));
            const float hi = fmaf(tab.scale, __uint_as_float(v[c4 * 8 + 2 * e + 1]), bf16hi_to_f32(wv[e]));
            o[e] = pack_bf16x2(lo, hi);
          }
          *p = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(accempty0 + 8u * b);  // this warp is done with the accumulator
        const MergeJob& job = tab.job[j];
        const int r0 = mt.m0 + q * 32;
        const int c0 = mt.n0 + h * 64;
        if (r0 < job.rows && c0 < job.cols)  // this warp's 32 rows of its box
          tma_store_2d(&job.w_dst, sbase + uint32_t(stage) * L.stage_bytes + uint32_t(h * 16384 + q * 32 * 128), c0,
                       r0);
        bulk_commit_group();
        // the previous tile's store has read its rows: give that stage back
        bulk_wait_group_read1();
        if (prev_stage >= 0) mbar_arrive(empty_bar(prev_stage));
      }
      __syncwarp();
      prev_stage = stage;
      if (++stage == S) { stage = 0; phase ^= 1u; }
    }
    if (lane == 0) {
      bulk_wait_group0();  // every store has completed
      if (prev_stage >= 0) mbar_arrive(empty_bar(prev_stage));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kMergeBN);
  }
}


// The plain copy and fill kernels have internal linkage: this header is
// included by more than one translation unit of the library.

// W_dst <- W_src, 16 bytes per thread per step (restore from pristine).
static __global__ void copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// Tail of a copy that is not a multiple of 16 bytes (2-byte elements).
static __global__ void copy2_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, size_t n) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i];
}

static __global__ void zero16_kernel(uint4* __restrict__ dst, size_t n16) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace lora
