// merge.cuh - W_dst = bf16_rne(W_src + s * B A) for a table of matrices.
//
// unsloth fork commit log (scripts/benchmarks/qwen3_flex_inference.py): the
// refresh merges each LoRA target from its pristine base in one pass,
// addmm(pristine, B, A, alpha=scaling, out=W_inf), with the rank-r product
// accumulated in fp32 and rounded once; restoring from pristine keeps the
// base bit-identical across refreshes.
//
// One CTA per 128 x 128 tile of one matrix.  TMA brings the W_src tile
// (two 64-column SW128 boxes), the B rows [128, r] (K-major, K = r) and the
// A columns [r, 128] (MN-major) into shared memory; one thread issues the
// r/16 tcgen05.mma steps of the K = r product into TMEM; the four epilogue
// warps read the fp32 product row by row, add s * product to the W_src
// value in fp32, round once to bf16, write the result over the W_src tile
// in shared memory (same swizzled place) and TMA-store it to W_dst.  The
// tile is read completely before it is written, so W_dst == W_src works.
// The kernel is bound by HBM traffic (read W_src, write W_dst).
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kMergeBN = 128;
constexpr int kMergeMaxJobs = 48;

struct MergeJob {
  CUtensorMap w_src;  // [d_out, d_in], box {64, 128}, SW128
  CUtensorMap w_dst;  // [d_out, d_in], box {64, 32}, SW128 (per-warp stores)
  CUtensorMap a;      // A [r, d_in] read MN-major, box {64, r_pad}, SW128
  CUtensorMap b;      // B [d_out, r] read K-major, box {RCW, 128}
  int32_t tiles_n;    // column tiles of this matrix
  int32_t tile_begin; // first global tile index of this matrix
  int32_t pad0, pad1;
};

struct MergeTable {
  MergeJob job[kMergeMaxJobs];
  int32_t n_jobs;
  int32_t r_pad;
  int32_t n_rchunks;
  float scale;
  uint64_t wait_limit_ns;
};

struct MergeLayout {
  uint32_t w_bytes, b_bytes, a_bytes, off_b, off_a, off_bar, total;
  __host__ __device__ MergeLayout(int rcw, int r_pad, int n_rchunks) {
    w_bytes = 128 * kMergeBN * 2;                      // 32 KB
    b_bytes = uint32_t(n_rchunks * 128 * rcw * 2);
    a_bytes = uint32_t((kMergeBN / 64) * r_pad * 128);
    off_b = w_bytes;
    off_a = off_b + b_bytes;
    off_bar = off_a + a_bytes;
    total = off_bar + 64;
  }
};

template <int RCW>
__global__ void __launch_bounds__(192) merge_kernel(const __grid_constant__ MergeTable tab) {
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);
  const MergeLayout L(RCW, tab.r_pad, tab.n_rchunks);
  const uint32_t full = sbase + L.off_bar;
  const uint32_t accfull = full + 8;
  const uint32_t drain = full + 16;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 24);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // locate this block's matrix and tile
  int j = 0;
  while (j + 1 < tab.n_jobs && int(blockIdx.x) >= tab.job[j + 1].tile_begin) ++j;
  const MergeJob& job = tab.job[j];
  const int t = int(blockIdx.x) - job.tile_begin;
  const int m0 = (t / job.tiles_n) * 128;
  const int n0 = (t % job.tiles_n) * kMergeBN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = tab.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kMergeBN);
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
    if (lane == 0) {
      mbar_arrive_expect_tx(full, L.w_bytes + L.b_bytes + L.a_bytes);
      tma_load_2d(sbase, &job.w_src, full, n0, m0);
      tma_load_2d(sbase + 16384u, &job.w_src, full, n0 + 64, m0);
      for (int c = 0; c < tab.n_rchunks; ++c)
        tma_load_2d(sbase + L.off_b + uint32_t(c) * (128u * kRSpan), &job.b, full, c * RCW, m0);
      tma_load_2d(sbase + L.off_a, &job.a, full, n0, 0);
      tma_load_2d(sbase + L.off_a + uint32_t(tab.r_pad) * 128u, &job.a, full, n0 + 64, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (wait_bounded(full, 0u, abort_flag, lim, SITE_FULL)) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, kMergeBN, false, true);
        const uint32_t sb = sbase + L.off_b;
        const uint32_t sa = sbase + L.off_a;
        for (int kk = 0; kk < tab.r_pad / 16; ++kk) {
          const uint32_t c = uint32_t(kk * 16) / RCW;
          const uint32_t off = uint32_t((kk * 16) % RCW) * 2u;
          const uint64_t ad = smem_desc(sb + c * (128u * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          const uint64_t bd = smem_desc(sa + uint32_t(kk) * 2048u, uint32_t(tab.r_pad) * 128u, 1024u, SWZ_128B);
          umma_bf16(tmem, ad, bd, idesc, kk != 0);
        }
        umma_commit(accfull);
      }
      umma_commit(drain);
      wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    if (warp_wait_bounded(accfull, 0u, abort_flag, lim, SITE_ACCFULL)) {
      tc_fence_after();
      for (int h = 0; h < 2; ++h) {              // two 64-column boxes
        uint8_t* box = gbase + h * 16384;
        for (int half = 0; half < 2; ++half) {   // 32 columns at a time
          uint32_t v[32];
          tmem_ld_x32(tmem + lane_base + uint32_t(h * 64 + half * 32), v);
          tmem_ld_wait();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {       // 16-byte chunks of 8 values
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
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // this warp's 32 rows of both boxes
        tma_store_2d(&job.w_dst, sbase + uint32_t(q * 32) * 128u, n0, m0 + q * 32);
        tma_store_2d(&job.w_dst, sbase + 16384u + uint32_t(q * 32) * 128u, n0 + 64, m0 + q * 32);
        bulk_commit_group();
        bulk_wait_group0();
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kMergeBN);
  }
}

// W_dst <- W_src, 16 bytes per thread per step (restore from pristine).
__global__ void copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// Tail of a copy that is not a multiple of 16 bytes (2-byte elements).
__global__ void copy2_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, size_t n) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i];
}

__global__ void zero16_kernel(uint4* __restrict__ dst, size_t n16) {
  griddep_launch_dependents();
  griddep_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace lora
