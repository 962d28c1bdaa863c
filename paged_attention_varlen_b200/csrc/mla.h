// mla.h -- host plan for the MLA decode / speculative-decode path.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/ala.h"

namespace ala {

struct MlaPlan {
  int32_t dtype = 0, heads = 0, batch = 0, block_size = 0, max_blocks = 0;
  int32_t calc_type = 0, mask_type = 0;
  bool kv8 = false, qn_int8 = false;  // int8 latent cache (cacheMode 2); qNope holds int8 codes
  const float *qk_descale = nullptr, *pv_descale = nullptr;
  float qk_scale = 1.f;
  int64_t tokens = 0, num_blocks = 0;
  void *q_nope = nullptr, *q_rope = nullptr, *ct_kv = nullptr, *k_rope = nullptr, *out = nullptr;
  float* lse = nullptr;
  const int32_t* block_tables = nullptr;
  const uint16_t* mask = nullptr;      // explicit MASK_TYPE_SPEC mask [tokens, mask_cols], or null
  int64_t mask_cols = 0;
  bool mask_f16 = false;
  std::vector<int32_t> ctx, qs;
  // row blocks of tpc tokens x hpc heads; groups = heads / hpc
  int32_t tpc = 1, hpc = 64, groups = 1;
  // schedule and workspace: [status | pieces | lane offsets | combine list | partial lse | partial O]
  int32_t n_lanes = 0, n_work = 0, n_splits_total = 0, n_combine = 0;
  uint64_t ws_size = 0, off_work = 0, off_lanes = 0, off_rows = 0, off_part_o = 0, off_part_lse = 0,
           image_size = 0;
  std::vector<uint8_t> image;  // host copy of [status | pieces | lane offsets | combine list]
  void* pinned = nullptr;      // page-locked copy of `image`, made on first run
  bool maps_ready = false;
  CUtensorMap tmQr, tmKV, tmKV3, tmKR, tmO;
  CUtensorMap tmPO;                // partial-output map, bound to the workspace it was encoded for
  const void* tmPO_base = nullptr;
  const void* bound_ws = nullptr;  // a workspace that holds this plan's schedule (ala_op_bind_workspace)
  MlaPlan() = default;
  MlaPlan(const MlaPlan&) = delete;
  MlaPlan& operator=(const MlaPlan&) = delete;
  ~MlaPlan();
};

int mla_plan(MlaPlan* plan, const ala_tensor* qNope, const ala_tensor* qRope, const ala_tensor* ctKV,
             const ala_tensor* kRope, const ala_tensor* blockTables, const ala_tensor* contextLens,
             const ala_tensor* mask, const ala_tensor* qSeqLen, const ala_tensor* qkDescale,
             const ala_tensor* pvDescale, int32_t headNum, float qkScale, int32_t kvHeadNum, int maskType,
             int calcType, uint8_t cacheMode, ala_tensor* attenOut, ala_tensor* lse, char* err, size_t errlen);

int mla_run(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t errlen);
// Copies the plan's schedule image into `workspace` (stream-ordered).
int mla_upload(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t errlen);

}  // namespace ala
