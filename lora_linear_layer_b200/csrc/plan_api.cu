// plan_api.cu - lora_plan: the launch configuration the entry points would
// choose for a shape, computed by the same host planning code (host only:
// no device state is read and nothing is launched).  A translation unit of
// its own, beside lora_api.cu.
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

extern "C" {

lora_status_t lora_plan(int64_t M, int64_t d_in, int64_t d_out, int32_t r, int32_t sm_count, lora_plan_t* out) {
  if (out == nullptr) return LORA_ERR_NULL;
  std::memset(out, 0, sizeof(*out));
  lora_status_t s = check_sizes(M, d_in, d_out, r);
  if (s != LORA_OK) return s;
  if (sm_count < 2 || sm_count > 4096) return LORA_ERR_SHAPE;
  if (M == 0) return LORA_OK;
  SplitkPlan pl;
  if (use_splitk(M, d_out, d_in, r, sm_count, pl)) {
    out->fwd_kind = 1;
    out->fwd_bn = 128;
    out->fwd_cg = 1;
    out->fwd_stages = pl.stages;
    out->fwd_num_m = int32_t((M + 127) / 128);
    out->fwd_num_n = int32_t((d_out + 127) / 128);
    out->fwd_splits = pl.splits;
    out->fwd_smem = pl.smem;
  } else {
    FusedCfg c;
    if (!pick_fused(M, d_out, d_in, r, false, sm_count, c)) return LORA_ERR_RANK;
    out->fwd_bn = c.BN;
    out->fwd_cg = c.CG;
    out->fwd_stages = c.stages;
    out->fwd_run_l = c.args.run_l;
    out->fwd_seeded = c.args.seeded;
    out->fwd_tx = c.tx_fits && c.seeded_l > 0 ? 1 : 0;
    out->fwd_num_m = c.args.num_m;
    out->fwd_num_n = c.args.num_n;
    out->fwd_splits = 1;
    out->fwd_smem = c.smem;
  }
  BwdPlan p;
  plan_bwd(M, d_in, d_out, r, sm_count, p);
  out->bwd1_splits_dt = p.dt_cfg.splits;
  out->bwd1_splits_t = p.t_cfg.splits;
  out->bwd1_saved_splits = p.dto_cfg.splits;
  out->bwd1_smem = std::max(p.dt_cfg.smem, p.t_cfg.smem);
  out->bwd2_splits_db = p.db_cfg.splits;
  out->bwd2_splits_da = p.da_cfg.splits;
  out->bwd2_smem = std::max(p.db_cfg.smem, p.da_cfg.smem);
  FusedCfg dx;
  if (!pick_fused(M, d_in, d_out, r, true, sm_count, dx)) return LORA_ERR_RANK;
  out->dx_bn = dx.BN;
  out->dx_cg = dx.CG;
  out->dx_stages = dx.stages;
  out->dx_smem = dx.smem;
  out->workspace_bytes = p.total;
  return LORA_OK;
}

}  // extern "C"
