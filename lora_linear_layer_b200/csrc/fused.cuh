// fused.cuh - the fused LoRA GEMM: OUT = P Q^T + (s P U^T) V^T on tcgen05.
//
// One kernel serves two steps of the layer:
//   forward  (MN = false): P = X[M,d_in], Q = W[d_out,d_in], U = A[r,d_in],
//                          V = B[d_out,r]; all operands K-major.
//                          OUT = Y = X W^T + s (X A^T) B^T
//   dX       (MN = true):  P = dY[M,d_out], Q(n,k) = W[k,n], U(j,k) = B[k,j],
//                          V(n,j) = A[j,n]; Q, U, V are read MN-major.
//                          OUT = dX = dY W + (s dY B) A, and the bf16 dT = s dY B
//                          is also written out (for dA).
// (fastaf 0.1.0, "FWD kernel speedup": base product plus the down- and
// up-projections, scale and add; "BWD kernel speedup": the dX kernel.)
//
// Per 128 x BN output tile:
//   * the K loop streams P, Q (and, on the first tile of an M block, U)
//     through a TMA -> shared-memory ring; one thread issues
//     tcgen05.mma for the base product into a TMEM accumulator and, on that
//     first tile, the N = r product T = P U^T into a second TMEM region;
//   * four epilogue warps drain T, scale it by s in fp32, round to bf16 and
//     write it into shared memory in the UMMA K-major swizzled layout (it
//     never goes to global memory in the forward);
//   * one more MMA pass (K = r) accumulates (sT) V^T onto the base
//     accumulator; the epilogue rounds once to bf16 and stores.
// T is kept in shared memory and reused for every further tile of the same
// M block the CTA processes (tiles are scheduled so a CTA sweeps N within
// an M block).  Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer and
// TMEM owner, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4)...).
#pragma once

#include "common.cuh"

namespace lora {

constexpr int kBM = 128;          // tile rows (UMMA M)
constexpr int kBK = 64;           // K per pipeline stage (128 bytes of bf16)
constexpr int kFusedThreads = 192;

struct FusedArgs {
  int32_t M, N, K;          // OUT is [M, N]; contraction length K
  int32_t r_pad;            // rank rounded up to 16 (UMMA N of the T product)
  int32_t n_rchunks;        // r_pad / RCW rounded up
  int32_t stages;           // pipeline depth
  float scale;              // s = alpha / r
  __nv_bfloat16* out;       // [M, N] row-major, ld = N
  __nv_bfloat16* t_out;     // optional [M, r_pad] bf16 copy of s*T (dT), or null
  int32_t num_m, num_n;     // tile counts
  int32_t band_w, n_bands;  // column bands of the schedule
  uint64_t wait_limit_ns;
};

// Byte sizes / offsets of the shared-memory carve-up (host and device).
struct FusedLayout {
  uint32_t p_bytes, q_bytes, u_bytes, stage_bytes, v_bytes, st_bytes;
  uint32_t off_v, off_st, off_bar, total;
  __host__ __device__ FusedLayout(int BN, bool mn, int rcw, int r_pad, int n_rchunks, int stages) {
    p_bytes = kBM * kBK * 2;
    q_bytes = BN * kBK * 2;
    u_bytes = mn ? uint32_t(n_rchunks * rcw * 128) : uint32_t(r_pad * 128);
    stage_bytes = p_bytes + q_bytes + u_bytes;
    v_bytes = mn ? uint32_t((BN / 64) * r_pad * 128) : uint32_t(n_rchunks * BN * rcw * 2);
    st_bytes = uint32_t(n_rchunks * kBM * rcw * 2);
    off_v = stage_bytes * stages;
    off_st = off_v + v_bytes;
    off_bar = off_st + st_bytes;
    total = off_bar + 256;
  }
};

// Tile schedule: the N tiles are grouped into column bands; the tiles of a
// band are ordered M-major (N fastest) and split into gridDim.x contiguous
// ranges.  A CTA therefore sweeps N inside one or two M blocks per band,
// which lets it keep T of an M block on chip, while all CTAs work in the
// same band (bounded L2 footprint).
struct TileSched {
  int num_m, num_n, band_w, n_bands, G, c;
  int band, t, t_end, band_n0, w;
  __device__ TileSched(const FusedArgs& a)
      : num_m(a.num_m), num_n(a.num_n), band_w(a.band_w), n_bands(a.n_bands), G(gridDim.x),
        c(blockIdx.x), band(-1), t(0), t_end(0), band_n0(0), w(1) {}
  __device__ bool next(int& m, int& n) {
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

template <int BN, bool MN, int RCW>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_lora_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmV,
                      const FusedArgs a) {
  static_assert(BN == 128 || BN == 256, "BN");
  static_assert(RCW == 16 || RCW == 32 || RCW == 64, "RCW");
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;  // bytes per swizzled rank row

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);

  const FusedLayout L(BN, MN, RCW, a.r_pad, a.n_rchunks, a.stages);
  const int S = a.stages;
  const uint32_t bar0 = sbase + L.off_bar;
  // barrier map (8 bytes each)
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t vfull = bar0 + 8u * (2 * S + 0);
  const uint32_t vempty = bar0 + 8u * (2 * S + 1);
  const uint32_t accfull0 = bar0 + 8u * (2 * S + 2);   // +8*b
  const uint32_t accempty0 = bar0 + 8u * (2 * S + 4);  // +8*b
  const uint32_t tfull = bar0 + 8u * (2 * S + 6);
  const uint32_t stfull = bar0 + 8u * (2 * S + 7);
  const uint32_t drain = bar0 + 8u * (2 * S + 8);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 8 * (2 * S + 9));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(vfull, 1);
    mbar_init(vempty, 1);
    mbar_init(accfull0, 1);
    mbar_init(accfull0 + 8, 1);
    mbar_init(accempty0, 4);
    mbar_init(accempty0 + 8, 4);
    mbar_init(tfull, 1);
    mbar_init(stfull, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // T accumulator placement: its own columns if two BN-wide accumulators
  // and r_pad columns fit in 512, else it borrows the other accumulator.
  const bool borrow = (2 * BN + a.r_pad) > 512;
  const int nk = (a.K + kBK - 1) / kBK;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      TileSched sch(a);
      int m, n, prev_m = -1, stage = 0;
      uint32_t phase = 0, vcount = 0;
      bool ok = true;
      while (ok && sch.next(m, n)) {
        const bool ttile = (m != prev_m);
        prev_m = m;
        const uint32_t bytes = L.p_bytes + L.q_bytes + (ttile ? L.u_bytes : 0u);
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY)) { ok = false; break; }
          const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, bytes);
          const int k0 = kb * kBK;
          tma_load_2d(st, &tmP, fb, k0, m * kBM);
          if (!MN) {
            tma_load_2d(st + L.p_bytes, &tmQ, fb, k0, n * BN);
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(st + L.p_bytes + uint32_t(i) * 8192u, &tmQ, fb, n * BN + 64 * i, k0);
          }
          if (ttile) {
            const uint32_t su = st + L.p_bytes + L.q_bytes;
            if (!MN) {
              tma_load_2d(su, &tmU, fb, k0, 0);
            } else {
              for (int c = 0; c < a.n_rchunks; ++c)
                tma_load_2d(su + uint32_t(c) * (64u * kRSpan), &tmU, fb, c * RCW, k0);
            }
          }
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        // rank-side operand of the up-projection for this N tile
        if (!wait_bounded(vempty, (vcount & 1u) ^ 1u, abort_flag, lim, SITE_VEMPTY)) break;
        ++vcount;
        const uint32_t sv = sbase + L.off_v;
        mbar_arrive_expect_tx(vfull, L.v_bytes);
        if (!MN) {
          for (int c = 0; c < a.n_rchunks; ++c)
            tma_load_2d(sv + uint32_t(c) * uint32_t(BN * kRSpan), &tmV, vfull, c * RCW, n * BN);
        } else {
#pragma unroll
          for (int i = 0; i < BN / 64; ++i)
            tma_load_2d(sv + uint32_t(i) * uint32_t(a.r_pad * 128), &tmV, vfull, n * BN + 64 * i, 0);
        }
      }
      if (*abort_flag) settle_ns(200000);  // let copies in flight land
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint32_t id_base = idesc_bf16(kBM, BN, false, MN);
      const uint32_t id_t = idesc_bf16(kBM, a.r_pad, false, MN);
      const uint32_t id_up = idesc_bf16(kBM, BN, false, MN);
      TileSched sch(a);
      int m, n, prev_m = -1, stage = 0;
      uint32_t phase = 0, vcount = 0, ntt = 0, tcount = 0;
      uint32_t acc_waits0 = 0u, acc_waits1 = 0u;  // completed waits per accumulator
      auto next_acc_parity = [&](uint32_t buf) {
        const uint32_t k = buf ? acc_waits1++ : acc_waits0++;
        return (k & 1u) ^ 1u;
      };
      bool ok = true;
      while (ok && sch.next(m, n)) {
        const bool ttile = (m != prev_m);
        prev_m = m;
        const uint32_t b = tcount & 1u;
        if (!wait_bounded(accempty0 + 8u * b, next_acc_parity(b), abort_flag, lim, SITE_ACCEMPTY)) break;
        uint32_t t_col = 2u * BN;
        if (ttile && borrow) {
          const uint32_t ob = b ^ 1u;
          if (!wait_bounded(accempty0 + 8u * ob, next_acc_parity(ob), abort_flag, lim, SITE_ACCEMPTY)) break;
          t_col = ob * BN;
        }
        tc_fence_after();
        const uint32_t d_acc = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
          const uint32_t sq = st + L.p_bytes;
          const uint32_t su = sq + L.q_bytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            const uint64_t ad = smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B);
            const uint64_t bd = MN ? smem_desc(sq + kk * 2048u, 8192u, 1024u, SWZ_128B)
                                   : smem_desc(sq + kk * 32u, 16u, 1024u, SWZ_128B);
            umma_bf16(d_acc, ad, bd, id_base, acc);
            if (ttile) {
              const uint64_t ud = MN ? smem_desc(su + kk * (16u * kRSpan), 64u * kRSpan, 8u * kRSpan, kRSwz)
                                     : smem_desc(su + kk * 32u, 16u, 1024u, SWZ_128B);
              umma_bf16(tmem + t_col, ad, ud, id_t, acc);
            }
          }
          umma_commit(empty_bar(stage));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (ttile) {
          umma_commit(tfull);
          if (!wait_bounded(stfull, ntt & 1u, abort_flag, lim, SITE_STFULL)) break;
          ++ntt;
        }
        if (!wait_bounded(vfull, vcount & 1u, abort_flag, lim, SITE_VFULL)) break;
        ++vcount;
        tc_fence_after();
        const uint32_t s_t = sbase + L.off_st;
        const uint32_t s_v = sbase + L.off_v;
        for (int kk = 0; kk < a.r_pad / 16; ++kk) {
          const uint32_t c = uint32_t(kk * 16) / RCW;
          const uint32_t off = uint32_t((kk * 16) % RCW) * 2u;
          const uint64_t ad = smem_desc(s_t + c * uint32_t(kBM * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          const uint64_t bd = MN ? smem_desc(s_v + uint32_t(kk) * 2048u, uint32_t(a.r_pad) * 128u, 1024u, SWZ_128B)
                                 : smem_desc(s_v + c * uint32_t(BN * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          umma_bf16(d_acc, ad, bd, id_up, 1u);
        }
        umma_commit(vempty);
        umma_commit(accfull0 + 8u * b);
        ++tcount;
      }
      // make sure no tcgen05 op is still running before TMEM is released
      umma_commit(drain);
      wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN);
    }
  } else {
    // ---------------------------------------------------- epilogue ----
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int row = q * 32 + lane;     // tile row owned by this thread
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    TileSched sch(a);
    int m, n, prev_m = -1;
    uint32_t ntt = 0, tcount = 0;
    uint32_t full_waits0 = 0u, full_waits1 = 0u;  // completed accfull waits per buffer
    uint8_t* const st_ptr = gbase + L.off_st;
    while (sch.next(m, n)) {
      const bool ttile = (m != prev_m);
      prev_m = m;
      const uint32_t b = tcount & 1u;
      const int grow = m * kBM + row;
      if (ttile) {
        if (!warp_wait_bounded(tfull, ntt & 1u, abort_flag, lim, SITE_TFULL)) break;
        ++ntt;
        tc_fence_after();
        const uint32_t t_col = borrow ? (b ^ 1u) * BN : 2u * BN;
        for (int col = 0; col < a.r_pad; col += 16) {
          uint32_t v[16];
          tmem_ld_x16(tmem + lane_base + t_col + uint32_t(col), v);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * a.scale, __uint_as_float(v[2 * i + 1]) * a.scale);
          const int c = col / RCW;
          const int cin = (col % RCW) / 8;  // 16-byte chunk inside the rank row
          uint8_t* chunk = st_ptr + c * (kBM * kRSpan);
          *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin, kRSpan)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(chunk + swz_offset(row, cin + 1, kRSpan)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          if (a.t_out != nullptr && n == 0 && grow < a.M) {
            uint4* dst = reinterpret_cast<uint4*>(a.t_out + (size_t)grow * a.r_pad + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(stfull);
          if (borrow) mbar_arrive(accempty0 + 8u * (b ^ 1u));
        }
      }
      const uint32_t fpar = (b ? full_waits1++ : full_waits0++) & 1u;
      if (!warp_wait_bounded(accfull0 + 8u * b, fpar, abort_flag, lim, SITE_ACCFULL)) break;
      tc_fence_after();
      const uint32_t acc_col = b * BN;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld_x32(tmem + lane_base + acc_col + uint32_t(ch * 32), v);
        tmem_ld_wait();
        if (grow < a.M) {
          const int col0 = n * BN + ch * 32;
          __nv_bfloat16* orow = a.out + (size_t)grow * a.N;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = col0 + 8 * g;
            if (col < a.N) {
              uint4 pk;
              pk.x = pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1]));
              pk.y = pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3]));
              pk.z = pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5]));
              pk.w = pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7]));
              *reinterpret_cast<uint4*>(orow + col) = pk;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty0 + 8u * b);
      ++tcount;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace lora
