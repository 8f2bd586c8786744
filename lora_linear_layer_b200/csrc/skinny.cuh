// skinny.cuh - OUT[i, j] = scale * sum_k P(i, k) R(j, k) with j < r_pad.
//
// The rank-sized products of the backward (fastaf 0.1.0, "BWD kernel
// speedup": the dA and dB kernels; the M reduction made sequence-parallel):
//   T recompute:  P = X[M, d_in] (K-major),  R = A[r, d_in] (K-major)
//   dB partials:  P(i,k) = dY[k, i] (MN),    R(j,k) = T[k, j] (MN)
//   dA partials:  P(i,k) = X[k, i] (MN),     R(j,k) = dT[k, j] (MN)
// i runs over 128-row tiles (UMMA M = 128), the rank is the UMMA N, and the
// contraction K (tokens for dA/dB) is split across blockIdx.y into
// fixed ranges.  Each split writes its fp32 partial; reduce_partials sums
// them in split order, so the result does not depend on scheduling.
#pragma once

#include "common.cuh"

namespace lora {

struct SkinnyArgs {
  int32_t rows;           // number of output rows (size of the i dimension)
  int32_t K;              // contraction length
  int32_t r_pad;          // rank rounded up to 16
  int32_t n_rchunks;      // r_pad / RCW rounded up
  int32_t stages;
  int32_t kb_per_split;   // K blocks (of 64) per split
  float scale;            // applied in the bf16 mode
  __nv_bfloat16* out_bf16;  // mode bf16: [rows, r_pad]
  float* out_f32;           // mode partials: [splits, rows, r_pad]
  uint64_t wait_limit_ns;
};

struct SkinnyLayout {
  uint32_t p_bytes, r_bytes, stage_bytes, off_bar, total;
  __host__ __device__ SkinnyLayout(bool r_mn, int rcw, int r_pad, int n_rchunks, int stages) {
    p_bytes = 128 * 64 * 2;
    r_bytes = r_mn ? uint32_t(n_rchunks * rcw * 128) : uint32_t(r_pad * 128);
    stage_bytes = p_bytes + r_bytes;
    off_bar = stage_bytes * stages;
    total = off_bar + 256;
  }
};

__host__ __device__ inline uint32_t tmem_cols_for(int r_pad) {
  uint32_t c = 32;
  while (c < uint32_t(r_pad)) c <<= 1;
  return c;
}

template <bool P_MN, bool R_MN, int RCW, bool PARTIALS>
__global__ void __launch_bounds__(192, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmR,
                  const SkinnyArgs a) {
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);
  const SkinnyLayout L(R_MN, RCW, a.r_pad, a.n_rchunks, a.stages);
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

  const int i0 = blockIdx.x * 128;
  const int nk_total = (a.K + 63) / 64;
  const int kb0 = blockIdx.y * a.kb_per_split;
  const int kb1 = imin(nk_total, kb0 + a.kb_per_split);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 0) {
    if (lane == 0) {
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
        if (!R_MN) {
          tma_load_2d(sr, &tmR, fb, k0, 0);
        } else {
          for (int c = 0; c < a.n_rchunks; ++c)
            tma_load_2d(sr + uint32_t(c) * (64u * kRSpan), &tmR, fb, c * RCW, k0);
        }
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (*abort_flag) settle_ns(200000);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, a.r_pad, P_MN, R_MN);
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
          const uint64_t bd = R_MN ? smem_desc(sr + kk * (16u * kRSpan), 64u * kRSpan, 8u * kRSpan, kRSwz)
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
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int gi = i0 + row;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    bool have = true;
    if (nkb > 0) {
      have = warp_wait_bounded(accfull, 0u, abort_flag, lim, SITE_ACCFULL);
      tc_fence_after();
    }
    if (have) {
      for (int col = 0; col < a.r_pad; col += 16) {
        uint32_t v[16];
        if (nkb > 0) {
          tmem_ld_x16(tmem + lane_base + uint32_t(col), v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0u;  // empty split: contributes zero
        }
        if (gi < a.rows) {
          if (PARTIALS) {
            float* dst = a.out_f32 + ((size_t)blockIdx.y * a.rows + gi) * a.r_pad + col;
#pragma unroll
            for (int g = 0; g < 4; ++g)
              reinterpret_cast<uint4*>(dst)[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
          } else {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * a.scale, __uint_as_float(v[2 * i + 1]) * a.scale);
            uint4* dst = reinterpret_cast<uint4*>(a.out_bf16 + (size_t)gi * a.r_pad + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// dst = bf16(scale * sum_{s < splits} part[s]) in split order.
//   part: [splits, rows, r_pad] fp32.  Only j < r is written.
//   transpose = false: dst[i * r + j]       (dB: [d_out, r])
//   transpose = true:  dst[j * rows + i]    (dA: [r, d_in])
// One block covers 32 rows x r_pad; the transposed case goes through shared
// memory so both the reads and the writes are coalesced.
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ part, int splits,
                                                               int rows, int r_pad, int r, float scale,
                                                               __nv_bfloat16* __restrict__ dst, int transpose) {
  __shared__ float tile[32][257];
  const int i0 = blockIdx.x * 32;
  const int nelem = 32 * r_pad;
  const size_t plane = (size_t)rows * r_pad;
  for (int e = threadIdx.x; e < nelem; e += blockDim.x) {
    const int i = i0 + e / r_pad;
    const int j = e % r_pad;
    float acc = 0.f;
    if (i < rows) {
      const float* p = part + (size_t)i * r_pad + j;
      for (int s = 0; s < splits; ++s) acc += p[(size_t)s * plane];
    }
    acc *= scale;
    if (!transpose) {
      if (i < rows && j < r) dst[(size_t)i * r + j] = __float2bfloat16_rn(acc);
    } else {
      tile[e / r_pad][j] = acc;
    }
  }
  if (transpose) {
    __syncthreads();
    for (int e = threadIdx.x; e < nelem; e += blockDim.x) {
      const int j = e / 32;
      const int ii = e % 32;
      const int i = i0 + ii;
      if (j < r && i < rows) dst[(size_t)j * rows + i] = __float2bfloat16_rn(tile[ii][j]);
    }
  }
}

}  // namespace lora

namespace lora {

// Bt[j, n] = B[n, j] for j < r: the transposed copy of the LoRA B matrix
// that the dX step reads K-major (B is [d_out, r], Bt is [r, d_out]).
// Tiles of 32 rows of B through shared memory; r <= 128.
__global__ void __launch_bounds__(256) transpose_rank_kernel(const __nv_bfloat16* __restrict__ B, int d_out, int r,
                                                              __nv_bfloat16* __restrict__ Bt) {
  __shared__ __nv_bfloat16 tile[32][129];
  const int n0 = blockIdx.x * 32;
  for (int e = threadIdx.x; e < 32 * r; e += blockDim.x) {
    const int i = e / r, j = e % r;
    if (n0 + i < d_out) tile[i][j] = B[(size_t)(n0 + i) * r + j];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 32 * r; e += blockDim.x) {
    const int j = e / 32, i = e % 32;
    if (n0 + i < d_out) Bt[(size_t)j * d_out + n0 + i] = tile[i][j];
  }
}

}  // namespace lora
