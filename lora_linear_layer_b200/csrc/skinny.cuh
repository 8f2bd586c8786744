// skinny.cuh - OUT[i, j] = scale * sum_k P(i, k) R(j, k) with j < r_pad.
//
// The rank-sized products of the backward (fastaf 0.1.0, "BWD kernel
// speedup": the dA and dB kernels, with the M reduction made parallel):
//   T recompute:  P = X[M, d_in] (K-major),  R = A[r, d_in] (K-major)
//   dT = s dY B:  P = dY[M, d_out] (K-major), R(j,k) = B[k, j] (MN)
//   dB:           P(i,k) = dY[k, i] (MN),    R(j,k) = T[k, j] (MN)
//   dA:           P(i,k) = X[k, i] (MN),     R(j,k) = dT[k, j] (MN)
// i runs over 128-row tiles (UMMA M = 128) and the rank is the UMMA N.  The
// contraction K (d_in for T, tokens for dA/dB) is split into S fixed ranges
// (blockIdx.y).  The S CTAs of one row tile form a cluster: each leaves its
// fp32 partial in its own shared memory, then each reduces 1/S of the rows,
// reading the S partials over distributed shared memory and adding them in
// split order, before one rounding to bf16.
// Nothing goes through global memory and no atomics are used, so results
// are bitwise repeatable for a given shape.
// One launch can carry two independent jobs with the same P layout and
// split count (dT and T; dB and dA): row tiles [0, x_split) of the grid run
// job 0, the rest job 1.  R's layout is a per-job argument.
#pragma once

#include "common.cuh"

namespace lora {

enum SkinnyOut : int32_t {
  OUT_ROWS_RPAD = 0,   // out[i * r_pad + j], every j < r_pad       (T)
  OUT_ROWS_R = 1,      // out[i * r + j], j < r                     (dB)
  OUT_COLS_R = 2,      // out[j * rows + i], j < r (transposed)     (dA)
};

struct SkinnyArgs {
  int32_t rows;           // number of output rows (size of the i dimension)
  int32_t K;              // contraction length
  int32_t r_pad;          // rank rounded up to 16
  int32_t r;              // rank
  int32_t n_rchunks;      // r_pad / RCW rounded up
  int32_t stages;
  int32_t kb_per_split;   // K blocks (of 64) per split
  int32_t splits;         // gridDim.y; the cluster size when > 1
  int32_t out_mode;       // SkinnyOut
  int32_t r_mn;           // R is read MN-major (rank contiguous) rather than K-major
  int32_t out_f32;        // OUT_ROWS_R / OUT_COLS_R: write fp32 (no rounding) instead of bf16
  float scale;            // applied to the reduced fp32 sum before rounding
  __nv_bfloat16* out;     // (a float* when out_f32)
  uint64_t wait_limit_ns;
};

struct SkinnyLayout {
  uint32_t p_bytes, r_bytes, stage_bytes, ring_bytes, red_stride, red_bytes, off_bar, total;
  __host__ __device__ SkinnyLayout(bool r_mn, int rcw, int r_pad, int n_rchunks, int stages) {
    p_bytes = 128 * 64 * 2;
    r_bytes = r_mn ? uint32_t(n_rchunks * rcw * 128) : uint32_t(r_pad * 128);
    stage_bytes = p_bytes + r_bytes;
    ring_bytes = stage_bytes * stages;
    // fp32 partial rows, padded by 4 floats so the 16-byte accesses of 8
    // consecutive rows fall in distinct bank groups
    red_stride = uint32_t((r_pad + 4) * 4);
    red_bytes = 128u * red_stride;
    const uint32_t body = ring_bytes > red_bytes ? ring_bytes : red_bytes;  // the partial reuses the ring
    off_bar = (body + 1023u) & ~1023u;
    total = off_bar + 256;
  }
};

__host__ __device__ inline uint32_t tmem_cols_for(int r_pad) {
  uint32_t c = 32;
  while (c < uint32_t(r_pad)) c <<= 1;
  return c;
}

template <bool P_MN, int RCW>
__global__ void __launch_bounds__(192, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmP0, const __grid_constant__ CUtensorMap tmR0,
                  const __grid_constant__ CUtensorMap tmP1, const __grid_constant__ CUtensorMap tmR1,
                  const __grid_constant__ SkinnyArgs a0, const __grid_constant__ SkinnyArgs a1, const int32_t x_split) {
  const bool second = int(blockIdx.x) >= x_split;
  const SkinnyArgs& a = second ? a1 : a0;
  const int bx = second ? int(blockIdx.x) - x_split : int(blockIdx.x);   // row tile within the job
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);
  const bool r_mn = a.r_mn != 0;
  const SkinnyLayout L(r_mn, RCW, a.r_pad, a.n_rchunks, a.stages);
  const int S = a.stages;
  const uint32_t bar0 = sbase + L.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t accfull = bar0 + 8u * (2 * S);
  const uint32_t drain = bar0 + 8u * (2 * S + 1);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 8 * (2 * S + 2));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols_for(a.r_pad);
  const bool clustered = a.splits > 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), ncols);
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

  const int i0 = bx * 128;
  const int split = blockIdx.y;
  const int nk_total = (a.K + 63) / 64;
  const int kb0 = split * a.kb_per_split;
  const int kb1 = imin(nk_total, kb0 + a.kb_per_split);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 0) {
    // The loop is instantiated once per job with that job's tensor maps
    // named directly: a map chosen through a runtime pointer would make
    // every load take its descriptor from a runtime address (measured
    // ~10% slower on the fused kernel).
    auto produce = [&](const CUtensorMap& tmP, const CUtensorMap& tmR) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY)) break;
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t fb = full_bar(stage);
        mbar_arrive_expect_tx(fb, L.stage_bytes);
        const int k0 = kb * 64;
        if (!P_MN) {
          tma_load_2d(st, &tmP, fb, k0, i0);
        } else {
          tma_load_2d(st, &tmP, fb, i0, k0);
          tma_load_2d(st + 8192u, &tmP, fb, i0 + 64, k0);
        }
        const uint32_t sr = st + L.p_bytes;
        if (!r_mn) {
          tma_load_2d(sr, &tmR, fb, k0, 0);
        } else {
          for (int c = 0; c < a.n_rchunks; ++c)
            tma_load_2d(sr + uint32_t(c) * (64u * kRSpan), &tmR, fb, c * RCW, k0);
        }
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    };
    if (lane == 0) {
      if (second) produce(tmP1, tmR1);
      else produce(tmP0, tmR0);
      if (*abort_flag) settle_ns(200000);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, a.r_pad, P_MN, r_mn);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t sr = st + L.p_bytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = P_MN ? smem_desc(st + kk * 2048u, 8192u, 1024u, SWZ_128B)
                                   : smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B);
          const uint64_t bd = r_mn ? smem_desc(sr + kk * (16u * kRSpan), 64u * kRSpan, 8u * kRSpan, kRSwz)
                                   : smem_desc(sr + kk * 32u, 16u, 1024u, SWZ_128B);
          umma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        umma_commit(empty_bar(stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (ok) umma_commit(accfull);
      umma_commit(drain);
      wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN);
    }
  }

  // ---------------------------------------------- partial / output -----
  const int q = warp & 3;
  const int row = q * 32 + lane;
  const int gi = i0 + row;
  auto write_out = [&](const float* acc, int col0) {  // 16 reduced values of row gi
    if (gi >= a.rows) return;
    if (a.out_mode == OUT_ROWS_RPAD) {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(acc[2 * e] * a.scale, acc[2 * e + 1] * a.scale);
      uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)gi * a.r_pad + col0);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else if (a.out_mode == OUT_ROWS_R) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {               // 8 values, r % 8 == 0
        if (col0 + 8 * h >= a.r) break;
        if (a.out_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + (size_t)gi * a.r + col0 + 8 * h);
          dst[0] = make_float4(acc[8 * h] * a.scale, acc[8 * h + 1] * a.scale, acc[8 * h + 2] * a.scale,
                               acc[8 * h + 3] * a.scale);
          dst[1] = make_float4(acc[8 * h + 4] * a.scale, acc[8 * h + 5] * a.scale, acc[8 * h + 6] * a.scale,
                               acc[8 * h + 7] * a.scale);
          continue;
        }
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[e] = pack_bf16x2(acc[8 * h + 2 * e] * a.scale, acc[8 * h + 2 * e + 1] * a.scale);
        *reinterpret_cast<uint4*>(a.out + (size_t)gi * a.r + col0 + 8 * h) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (col0 + e >= a.r) continue;
        const size_t o = (size_t)(col0 + e) * a.rows + gi;
        if (a.out_f32) reinterpret_cast<float*>(a.out)[o] = acc[e] * a.scale;
        else a.out[o] = __float2bfloat16_rn(acc[e] * a.scale);
      }
    }
  };

  uint8_t* const red = gbase;  // fp32 partial rows (reuses the ring once the MMAs are done)
  if (warp >= 2) {
    bool have = true;
    if (nkb > 0) {
      have = warp_wait_bounded(accfull, 0u, abort_flag, lim, SITE_ACCFULL);
      tc_fence_after();
    }
    if (have) {
      const uint32_t lane_base = uint32_t(q * 32) << 16;
      for (int col = 0; col < a.r_pad; col += 16) {
        uint32_t v[16];
        if (nkb > 0) {
          tmem_ld_x16(tmem + lane_base + uint32_t(col), v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;  // empty split: contributes zero
        }
        if (!clustered) {
          float acc[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(v[e]);
          write_out(acc, col);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(red + row * L.red_stride + col * 4);
#pragma unroll
          for (int g = 0; g < 4; ++g) dst[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (clustered) {
    cluster_barrier_sync();  // every split's partial is in its shared memory
    // Every CTA of the cluster reduces its own slice of the 128 rows: one
    // float4 (4 consecutive columns) per task, the S partials loaded
    // together and added in split order.
    if (warp >= 2 && !*abort_flag) {
      const int S = a.splits;
      const int f4_per_row = a.r_pad / 4;
      const int rows_per = (128 + S - 1) / S;
      const int r0 = split * rows_per;
      const int r1 = imin(128, r0 + rows_per);
      for (int task = int(threadIdx.x) - 64; task < (r1 - r0) * f4_per_row; task += 128) {
        const int rr = r0 + task / f4_per_row;
        const int c4 = task % f4_per_row;
        const uint32_t off = smem_addr(red + rr * L.red_stride + c4 * 16);
        float4 p[8];
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S) p[s2] = ld_shared_cluster_f4(mapa_shared(off, uint32_t(s2)));
        float4 acc = p[0];
#pragma unroll
        for (int s2 = 1; s2 < 8; ++s2)
          if (s2 < S) {
            acc.x += p[s2].x;
            acc.y += p[s2].y;
            acc.z += p[s2].z;
            acc.w += p[s2].w;
          }
        const int g = i0 + rr;
        const int j0 = c4 * 4;
        if (g < a.rows) {
          const float v[4] = {acc.x * a.scale, acc.y * a.scale, acc.z * a.scale, acc.w * a.scale};
          if (a.out_mode == OUT_ROWS_RPAD) {
            *reinterpret_cast<uint2*>(a.out + (size_t)g * a.r_pad + j0) =
                make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
          } else if (a.out_mode == OUT_ROWS_R) {
            if (j0 < a.r) {  // r % 8 == 0, so the 4 columns are all in or all out
              if (a.out_f32)
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + (size_t)g * a.r + j0) =
                    make_float4(v[0], v[1], v[2], v[3]);
              else
                *reinterpret_cast<uint2*>(a.out + (size_t)g * a.r + j0) =
                    make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (j0 + e >= a.r) continue;
              const size_t o = (size_t)(j0 + e) * a.rows + g;
              if (a.out_f32) reinterpret_cast<float*>(a.out)[o] = v[e];
              else a.out[o] = __float2bfloat16_rn(v[e]);
            }
          }
        }
      }
    }
    cluster_barrier_sync();  // peers keep their shared memory until every slice is done
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace lora
