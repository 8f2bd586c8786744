// splitk.cuh - the fused LoRA forward for grids with few output tiles:
// Y = X W^T + (s X A^T) B^T with the contraction split across a cluster.
//
// (fastaf 0.1.0, "FWD kernel speedup": base product, down-projection kept on
// chip, scale, up-projection and add in one kernel.)  With few 128 x 128
// output tiles (small M, or a small weight) one CTA per tile leaves most SMs
// idle and runs a long K loop.  Here the S CTAs of a cluster share one tile:
//   * CTA c runs K blocks [c * kb_per_split, (c + 1) * kb_per_split) and
//     accumulates, in ONE tcgen05.mma per 16-wide K step, the base product
//     X W^T and the down-projection X A^T: the A rows sit right after the W
//     rows in the stage, so B = [W tile; A] has N = 128 + r_pad rows and the
//     accumulator columns [0, 128) hold the base, [128, 128 + r_pad) hold T;
//   * every CTA moves its fp32 partials (T and base) from TMEM to its own
//     shared memory; after a cluster barrier, CTA 0 sums the S partials of T
//     (distributed shared memory, split order), scales by s, rounds to bf16
//     and accumulates (sT) B^T onto its base partial with one more MMA pass;
//   * after a second cluster barrier, CTA c sums rows [c*128/S, ...) of the S
//     base partials in split order, rounds once to bf16 and stores them.
// Nothing goes through global memory but Y, no atomics are used, and the
// result is bitwise repeatable for a given shape.
// A launch carries a table of problems with the same rank and scale
// (blockIdx.y runs over the tiles of all of them), so many small layers can
// share one launch.
#pragma once

#include "common.cuh"

namespace lora {

// One output problem of a launch (a grouped launch carries several, all with
// the same rank and scale).
struct SplitkJob {
  CUtensorMap p;            // X [M, d_in], box {64, 128}
  CUtensorMap q;            // W [d_out, d_in], box {64, 128}
  CUtensorMap u;            // A [r, d_in], box {64, r_pad}
  CUtensorMap v;            // B [d_out, r], box {RCW, 128}
  int32_t M, N, K;          // Y is [M, N]; contraction length K
  int32_t num_n;            // column tiles of 128
  int32_t tile_begin;       // first tile (blockIdx.y) of this problem
  int32_t kb_per_split;     // K blocks of 64 per split
  __nv_bfloat16* out;       // [M, N] row-major
};

template <int NJ>
struct SplitkTable {
  SplitkJob job[NJ];
  int32_t n_jobs;
  int32_t r_pad;            // rank rounded up to 16
  int32_t n_rchunks;        // r_pad / RCW rounded up
  int32_t stages;           // pipeline depth
  int32_t splits;           // cluster size S (gridDim.x)
  float scale;              // s = alpha / r
  uint64_t wait_limit_ns;
};

struct SplitkLayout {
  uint32_t p_bytes, q_bytes, u_bytes, stage_bytes, ring_bytes, rb_stride, rt_stride, off_rt, body;
  uint32_t v_bytes, st_bytes, off_v, off_st, off_bar, total;
  __host__ __device__ SplitkLayout(int rcw, int r_pad, int n_rchunks, int stages) {
    p_bytes = 128 * 64 * 2;
    q_bytes = 128 * 64 * 2;
    u_bytes = uint32_t(r_pad * 128);
    stage_bytes = (p_bytes + q_bytes + u_bytes + 1023u) & ~1023u;
    ring_bytes = stage_bytes * uint32_t(stages);
    // fp32 partials (reuse the ring once the K loop is done); rows padded by
    // 4 floats so the 16-byte accesses of 8 consecutive rows hit distinct banks
    rb_stride = (128 + 4) * 4;
    rt_stride = uint32_t((r_pad + 4) * 4);
    off_rt = 128u * rb_stride;
    const uint32_t red = off_rt + 128u * rt_stride;
    body = ((ring_bytes > red ? ring_bytes : red) + 1023u) & ~1023u;
    v_bytes = uint32_t(n_rchunks * 128 * rcw * 2);
    st_bytes = uint32_t(n_rchunks * 128 * rcw * 2);
    off_v = body;
    off_st = off_v + v_bytes;
    off_bar = off_st + st_bytes;
    total = off_bar + 256;
  }
};

template <int RCW, int NJ>
__global__ void __launch_bounds__(192, 1) fused_splitk_kernel(const __grid_constant__ SplitkTable<NJ> a) {
  static_assert(RCW == 16 || RCW == 32 || RCW == 64, "RCW");
  constexpr uint32_t kRSwz = RCW == 16 ? SWZ_32B : RCW == 32 ? SWZ_64B : SWZ_128B;
  constexpr uint32_t kRSpan = RCW * 2;  // bytes per swizzled rank row

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (sbase - raw);
  const SplitkLayout L(RCW, a.r_pad, a.n_rchunks, a.stages);
  const int S = a.stages;
  const uint32_t bar0 = sbase + L.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t accfull = bar0 + 8u * (2 * S + 0);
  const uint32_t vfull = bar0 + 8u * (2 * S + 1);
  const uint32_t stfull = bar0 + 8u * (2 * S + 2);
  const uint32_t upfull = bar0 + 8u * (2 * S + 3);
  const uint32_t drain = bar0 + 8u * (2 * S + 4);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.off_bar + 8 * (2 * S + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = int(cluster_ctarank());
  // this cluster's problem and tile
  const int tile = int(blockIdx.y);
  int jix = 0;
  if constexpr (NJ > 1)
    while (jix + 1 < a.n_jobs && tile >= a.job[jix + 1].tile_begin) ++jix;
  // with one job the index is a compile-time 0, so its tensor maps are
  // named directly rather than through a runtime address
  const SplitkJob& jb = a.job[NJ > 1 ? jix : 0];
  const int m = (tile - jb.tile_begin) / jb.num_n;
  const int n = (tile - jb.tile_begin) % jb.num_n;
  const int nk_total = (jb.K + 63) / 64;
  const int kb0 = split * jb.kb_per_split;
  const int kb1 = imin(nk_total, kb0 + jb.kb_per_split);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;
  const uint64_t lim = a.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accfull, 1);
    mbar_init(vfull, 1);
    mbar_init(stfull, 4);
    mbar_init(upfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&jb.p);
    tma_prefetch_desc(&jb.q);
    tma_prefetch_desc(&jb.u);
    tma_prefetch_desc(&jb.v);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_barrier_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above touches no global memory, so it may overlap the
  // previous kernel on the stream; every global access comes after the wait.
  griddep_launch_dependents();
  griddep_wait();

  const int q = warp & 3;            // TMEM lane quarter of an epilogue warp
  const int row = q * 32 + lane;     // tile row owned by an epilogue thread
  const uint32_t lane_base = uint32_t(q * 32) << 16;
  const uint32_t t_col = 128u;       // T columns follow the 128 base columns

  // --------------------------------------------- phase 1: K loop -----
  if (warp == 0) {
    if (lane == 0) {
      if (split == 0) {  // rank-side operand of the up-projection (B rows of this tile)
        mbar_arrive_expect_tx(vfull, L.v_bytes);
        for (int c = 0; c < a.n_rchunks; ++c)
          tma_load_2d(sbase + L.off_v + uint32_t(c) * (128u * kRSpan), &jb.v, vfull, c * RCW, n * 128);
      }
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, lim, SITE_EMPTY)) break;
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t fb = full_bar(stage);
        mbar_arrive_expect_tx(fb, L.p_bytes + L.q_bytes + L.u_bytes);
        const int k0 = kb * 64;
        tma_load_2d(st, &jb.p, fb, k0, m * 128);
        tma_load_2d(st + L.p_bytes, &jb.q, fb, k0, n * 128);
        tma_load_2d(st + L.p_bytes + L.q_bytes, &jb.u, fb, k0, 0);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (*abort_flag) settle_ns(200000);  // let copies in flight land
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // B = [W tile; A] (N = 128 + r_pad): base and T in one instruction
      const uint32_t idesc = idesc_bf16(128, 128 + a.r_pad, false, false);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(full_bar(stage), phase, abort_flag, lim, SITE_FULL)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + uint32_t(stage) * L.stage_bytes;
        const uint32_t sq = st + L.p_bytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, smem_desc(st + kk * 32u, 16u, 1024u, SWZ_128B), smem_desc(sq + kk * 32u, 16u, 1024u, SWZ_128B),
                    idesc, (kb | kk) != 0);
        umma_commit(empty_bar(stage));
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (ok && nkb > 0) umma_commit(accfull);
    }
  } else {
    // move this split's fp32 partials to shared memory (the ring is free:
    // every load has been consumed by the MMAs behind accfull)
    bool have = true;
    if (nkb > 0) {
      have = warp_wait_bounded(accfull, 0u, abort_flag, lim, SITE_ACCFULL);
      tc_fence_after();
    }
    if (have) {
      uint8_t* const rt = gbase + L.off_rt + row * L.rt_stride;
      for (int col = 0; col < a.r_pad; col += 16) {
        uint32_t v[16];
        if (nkb > 0) {
          tmem_ld_x16(tmem + lane_base + t_col + uint32_t(col), v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;  // empty split: contributes zero
        }
        uint4* dst = reinterpret_cast<uint4*>(rt + col * 4);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      }
      if (split != 0) {  // CTA 0 adds the up-projection first
        uint8_t* const rb = gbase + row * L.rb_stride;
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          if (nkb > 0) {
            tmem_ld_x32(tmem + lane_base + uint32_t(ch * 32), v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          uint4* dst = reinterpret_cast<uint4*>(rb + ch * 128);
#pragma unroll
          for (int g = 0; g < 8; ++g) dst[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_barrier_sync();  // every split's T partial (and base partial) is in its shared memory
  tc_fence_after();

  // ------------------------- phase 2 (CTA 0): T, up-projection ------
  if (split == 0) {
    if (warp >= 2) {
      if (!*abort_flag) {
        // one float4 of T per task: the S partials loaded together, added in
        // split order, scaled, rounded and written into the swizzled K-major
        // tile of the up-projection
        uint8_t* const st_ptr = gbase + L.off_st;
        const uint32_t rt0 = smem_addr(gbase + L.off_rt);
        const int f4_per_row = a.r_pad / 4;
        for (int task = int(threadIdx.x) - 64; task < 128 * f4_per_row; task += 128) {
          const int rr = task / f4_per_row;
          const int col = (task % f4_per_row) * 4;
          const uint32_t off = rt0 + uint32_t(rr) * L.rt_stride + uint32_t(col * 4);
          float4 p[8];
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            if (s2 < a.splits) p[s2] = ld_shared_cluster_f4(mapa_shared(off, uint32_t(s2)));
          float4 acc = p[0];
#pragma unroll
          for (int s2 = 1; s2 < 8; ++s2)
            if (s2 < a.splits) {
              acc.x += p[s2].x;
              acc.y += p[s2].y;
              acc.z += p[s2].z;
              acc.w += p[s2].w;
            }
          const int c = col / RCW;
          const int cin = (col % RCW) / 8;  // 16-byte chunk inside the rank row
          uint8_t* dst = st_ptr + c * (128 * kRSpan) + swz_offset(rr, cin, kRSpan) + (col % 8) * 2;
          *reinterpret_cast<uint2*>(dst) =
              make_uint2(pack_bf16x2(acc.x * a.scale, acc.y * a.scale), pack_bf16x2(acc.z * a.scale, acc.w * a.scale));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(stfull);
      // base partial of CTA 0 plus (sT) B^T, to shared memory
      const bool have = warp_wait_bounded(upfull, 0u, abort_flag, lim, SITE_ACCFULL);
      tc_fence_after();
      if (have) {
        uint8_t* const rb = gbase + row * L.rb_stride;
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          tmem_ld_x32(tmem + lane_base + uint32_t(ch * 32), v);
          tmem_ld_wait();
          uint4* dst = reinterpret_cast<uint4*>(rb + ch * 128);
#pragma unroll
          for (int g = 0; g < 8; ++g) dst[g] = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
      }
    } else if (warp == 1 && lane == 0) {
      if (wait_bounded(stfull, 0u, abort_flag, lim, SITE_STFULL) &&
          wait_bounded(vfull, 0u, abort_flag, lim, SITE_VFULL)) {
        tc_fence_after();
        const uint32_t id_up = idesc_bf16(128, 128, false, false);
        const uint32_t s_t = sbase + L.off_st;
        const uint32_t s_v = sbase + L.off_v;
        for (int kk = 0; kk < a.r_pad / 16; ++kk) {
          const uint32_t c = uint32_t(kk * 16) / RCW;
          const uint32_t off = uint32_t((kk * 16) % RCW) * 2u;
          const uint64_t ad = smem_desc(s_t + c * uint32_t(128 * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          const uint64_t bd = smem_desc(s_v + c * uint32_t(128 * kRSpan) + off, 16u, 8u * kRSpan, kRSwz);
          umma_bf16(tmem, ad, bd, id_up, (nkb > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(upfull);
      }
    }
  }
  if (warp == 1 && lane == 0) {
    // make sure no tcgen05 op is still running before TMEM is released
    umma_commit(drain);
    wait_bounded(drain, 0u, abort_flag, lim, SITE_DRAIN);
  }
  tc_fence_before();
  __syncthreads();
  cluster_barrier_sync();  // every split's final base partial is in its shared memory
  tc_fence_after();

  // ---------------- phase 3: rows [split*128/S, ...) summed, stored -----
  if (!*abort_flag) {
    const int rows_per = (128 + a.splits - 1) / a.splits;
    const int r0 = split * rows_per;
    const int r1 = imin(128, r0 + rows_per);
    const int ntasks = (r1 - r0) * 32;
    const int nthr = int(blockDim.x);
    // two float4 tasks per thread and step, the S partials of each loaded
    // together, added in split order
    for (int t0 = int(threadIdx.x); t0 < ntasks; t0 += 2 * nthr) {
      float4 p[2][8];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int task = t0 + u * nthr;
        if (task < ntasks) {
          const uint32_t off = smem_addr(gbase + (r0 + task / 32) * L.rb_stride + (task % 32) * 16);
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            if (s2 < a.splits) p[u][s2] = ld_shared_cluster_f4(mapa_shared(off, uint32_t(s2)));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int task = t0 + u * nthr;
        if (task >= ntasks) break;
        float4 acc = p[u][0];
#pragma unroll
        for (int s2 = 1; s2 < 8; ++s2)
          if (s2 < a.splits) {
            acc.x += p[u][s2].x;
            acc.y += p[u][s2].y;
            acc.z += p[u][s2].z;
            acc.w += p[u][s2].w;
          }
        const int grow = m * 128 + r0 + task / 32;
        const int gcol = n * 128 + (task % 32) * 4;
        if (grow < jb.M && gcol < jb.N)  // N % 8 == 0: the 4 columns are all in or all out
          *reinterpret_cast<uint2*>(jb.out + (size_t)grow * jb.N + gcol) =
              make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      }
    }
  }
  cluster_barrier_sync();  // peers keep their shared memory until every read is done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace lora
