// texchange.cuh - the down-projection exchange between the clusters of one
// forward launch.
//
// The forward keeps T = X A^T on chip (fastaf 0.1.0, "FWD kernel speedup":
// the [seq, rank] down-projection is never written out between the two
// matmuls).  A cluster computes T once per run of N tiles of an M block;
// when several clusters work on the same M block, each used to compute the
// same T again.  Here the first cluster to compute an M block's T also
// publishes its scaled, rounded form s T (bf16, the exact operand of the
// up-projection) in an exchange slot, and a cluster that starts on that M
// block later copies it instead of running the N = r products again.  The
// result is bit for bit the same either way: the published values are
// those the cluster would have computed itself.
//
// The slots are library-owned device memory (kTxSlots per device).  The
// host binds each slot to one stream, and launches on one stream run one
// after the other, so a slot is used by one launch at a time; a launch that
// gets none runs without the exchange.  A slot starts with every flag and
// the done count at zero, and the last cluster of the launch to finish
// puts them back to zero.  Nothing here waits on another cluster except a
// copying epilogue on a flag that its MMA thread has already seen complete.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace lora {

constexpr int kTxSlots = 8;
constexpr uint32_t kTxMaxBlocks = 4096;        // M blocks per launch
constexpr size_t kTxElems = size_t(2) << 20;   // bf16 values of s T per slot (4 MiB)

struct alignas(16) TxSlot {     // 16-byte vector loads and stores of t
  uint32_t done;                 // clusters of the current launch that have finished
  uint32_t pad[3];
  uint32_t flags[kTxMaxBlocks];  // per M block: one bit per epilogue warp that has published its rows
  __nv_bfloat16 t[kTxElems];     // s T, row-major [rows of the launch, r_pad]
};

static __device__ TxSlot g_tx[kTxSlots];

// Called once per cluster (one warp of the leader CTA, converged) after
// every role of the cluster is done with the slot.  The last cluster of
// the launch clears the first `num_m` flags and the done count.
__device__ __forceinline__ void tx_finish(TxSlot* tx, int n_clusters, int num_m, int lane) {
  int last = 0;
  if (lane == 0) last = atom_add_acq_rel_gpu(&tx->done, 1u) == uint32_t(n_clusters - 1) ? 1 : 0;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    for (int i = lane; i < num_m; i += 32) tx->flags[i] = 0u;
    if (lane == 0) tx->done = 0u;
    __threadfence();
  }
}

}  // namespace lora
