// mla.cu -- MLA decode / speculative decode over a paged latent cache
// (ATB "MLA" page, definition and parameter table).
#include <cstdio>
#include <cstring>

#include "internal.h"
#include "mla.h"
#include "ptx.cuh"

namespace ala {

namespace {
int mfail(char* err, size_t n, int st, const char* msg) {
  snprintf(err, n, "%s", msg);
  return st;
}
}  // namespace

int mla_plan(MlaPlan* plan, const ala_tensor* qNope, const ala_tensor* qRope, const ala_tensor* ctKV,
             const ala_tensor* kRope, const ala_tensor* blockTables, const ala_tensor* contextLens,
             const ala_tensor* mask, const ala_tensor* qSeqLen, const ala_tensor* qkDescale,
             const ala_tensor* pvDescale, int32_t headNum, float qkScale, int32_t kvHeadNum, int maskType,
             int calcType, uint8_t cacheMode, ala_tensor* attenOut, ala_tensor* lse, char* err, size_t n) {
  if (!qNope || !qRope || !ctKV || !kRope || !blockTables || !contextLens || !attenOut)
    return mfail(err, n, ALA_NULL_REQUIRED, "qNope, qRope, ctKV, kRope, blockTables, contextLens, attenOut are required");
  if (!qNope->data || !qRope->data || !ctKV->data || !kRope->data || !blockTables->data || !contextLens->data ||
      !attenOut->data)
    return mfail(err, n, ALA_NULL_REQUIRED, "a required tensor has a NULL data pointer");
  if (cacheMode != ALA_MLA_CACHE_KROPE_CTKV)
    return mfail(err, n, ALA_UNSUPPORTED, "only cacheMode KROPE_CTKV (1) is built");
  if (calcType == ALA_MLA_CALC_RING || calcType == ALA_MLA_CALC_PREFILL)
    return mfail(err, n, ALA_UNSUPPORTED, "calcType RING and PREFILL are not built");
  if (calcType != ALA_MLA_CALC_UNDEFINED && calcType != ALA_MLA_CALC_SPEC)
    return mfail(err, n, ALA_INVALID_PARAM, "calcType must be 0..3");
  if (maskType == 3 || maskType == 4 || maskType == 5)
    return mfail(err, n, ALA_INVALID_PARAM, "ALiBi masks apply only to the encoder paths");
  if (maskType != ALA_MLA_MASK_UNDEFINED && maskType != ALA_MLA_MASK_SPEC)
    return mfail(err, n, maskType == ALA_MLA_MASK_FREE ? ALA_UNSUPPORTED : ALA_INVALID_PARAM,
                 "maskType must be UNDEFINED (0) or SPEC (1)");
  if (mask && mask->data) return mfail(err, n, ALA_INVALID_PARAM, "mask must be NULL: the spec mask is generated");
  if ((qkDescale && qkDescale->data) || (pvDescale && pvDescale->data))
    return mfail(err, n, ALA_INVALID_PARAM, "qkDescale/pvDescale must be NULL (int8 cache not built)");
  if (headNum <= 0) return mfail(err, n, ALA_INVALID_PARAM, "headNum must be > 0");
  if (headNum % 64 != 0) return mfail(err, n, ALA_UNSUPPORTED, "headNum must be a multiple of 64");
  if (kvHeadNum != 1) return mfail(err, n, ALA_UNSUPPORTED, "kvHeadNum must be 1");
  const int32_t dt = qNope->dtype;
  if (dt != ALA_BF16 && dt != ALA_F16) return mfail(err, n, ALA_INVALID_DTYPE, "qNope must be bf16 or f16");
  if (qRope->dtype != dt || ctKV->dtype != dt || kRope->dtype != dt || attenOut->dtype != dt)
    return mfail(err, n, ALA_INVALID_DTYPE, "qRope, ctKV, kRope and attenOut must have qNope's dtype");
  if (blockTables->dtype != ALA_I32 || contextLens->dtype != ALA_I32)
    return mfail(err, n, ALA_INVALID_DTYPE, "blockTables and contextLens must be int32");
  if (qNope->ndim != 3 || qNope->dims[1] != headNum || qNope->dims[2] != 512)
    return mfail(err, n, ALA_INVALID_SHAPE, "qNope must be [tokens, headNum, 512]");
  const int64_t tokens = qNope->dims[0];
  if (qRope->ndim != 3 || qRope->dims[0] != tokens || qRope->dims[1] != headNum || qRope->dims[2] != 64)
    return mfail(err, n, ALA_INVALID_SHAPE, "qRope must be [tokens, headNum, 64]");
  if (ctKV->ndim != 4 || ctKV->dims[2] != 1 || ctKV->dims[3] != 512)
    return mfail(err, n, ALA_INVALID_SHAPE, "ctKV must be [numBlocks, blockSize, 1, 512]");
  if (kRope->ndim != 4 || kRope->dims[0] != ctKV->dims[0] || kRope->dims[1] != ctKV->dims[1] || kRope->dims[2] != 1 ||
      kRope->dims[3] != 64)
    return mfail(err, n, ALA_INVALID_SHAPE, "kRope must be [numBlocks, blockSize, 1, 64]");
  const int64_t bs = ctKV->dims[1];
  if (!(bs > 0 && bs % 16 == 0 && (128 % bs == 0 || bs % 128 == 0)))
    return mfail(err, n, ALA_UNSUPPORTED, "blockSize must be a multiple of 16 dividing 128, or a multiple of 128");
  if (attenOut->ndim != 3 || attenOut->dims[0] != tokens || attenOut->dims[1] != headNum || attenOut->dims[2] != 512)
    return mfail(err, n, ALA_INVALID_SHAPE, "attenOut must be [tokens, headNum, 512]");
  if (contextLens->ndim != 1) return mfail(err, n, ALA_INVALID_SHAPE, "contextLens must be [batch]");
  const int32_t batch = (int32_t)contextLens->dims[0];
  if (blockTables->ndim != 2 || blockTables->dims[0] != batch)
    return mfail(err, n, ALA_INVALID_SHAPE, "blockTables must be [batch, maxBlocks]");
  if (calcType == ALA_MLA_CALC_SPEC) {
    if (!qSeqLen || !qSeqLen->data) return mfail(err, n, ALA_NULL_REQUIRED, "qseqlen is required with calcType SPEC");
    if (qSeqLen->dtype != ALA_I32 || qSeqLen->ndim != 1 || qSeqLen->dims[0] != batch)
      return mfail(err, n, ALA_INVALID_SHAPE, "qseqlen must be int32 [batch]");
  } else if (qSeqLen && qSeqLen->data) {
    return mfail(err, n, ALA_INVALID_PARAM, "qseqlen is only passed with calcType SPEC");
  }
  if (lse && lse->data) {
    if (lse->dtype != ALA_F32) return mfail(err, n, ALA_INVALID_DTYPE, "lse must be fp32");
    int64_t ne = 1;
    for (int i = 0; i < lse->ndim; ++i) ne *= lse->dims[i];
    if (lse->dims[0] != tokens || ne != tokens * headNum)
      return mfail(err, n, ALA_INVALID_SHAPE, "lse must be [tokens, headNum, 1]");
  }
  const int32_t* cl = static_cast<const int32_t*>(contextLens->data);
  const int32_t* qs = qSeqLen && qSeqLen->data ? static_cast<const int32_t*>(qSeqLen->data) : nullptr;
  int64_t sum_q = 0;
  const int64_t max_blocks = blockTables->dims[1];
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t q = qs ? qs[b] : 1;
    if (q < 1) return mfail(err, n, ALA_INVALID_PARAM, "qseqlen entries must be >= 1");
    if (cl[b] < q) return mfail(err, n, ALA_INVALID_PARAM, "contextLens must be >= qseqlen");
    if ((cl[b] + bs - 1) / bs > max_blocks)
      return mfail(err, n, ALA_INVALID_PARAM, "contextLens needs more blocks than blockTables holds");
    if (q > 1 && maskType != ALA_MLA_MASK_SPEC)
      return mfail(err, n, ALA_INVALID_PARAM, "qseqlen > 1 needs maskType SPEC");
    sum_q += q;
  }
  if (sum_q != tokens) return mfail(err, n, ALA_INVALID_SHAPE, "sum(qseqlen) != tokens");
  if (ctKV->dims[0] * bs >= ((int64_t)1 << 31)) return mfail(err, n, ALA_UNSUPPORTED, "cache has more than 2^31 rows");

  plan->dtype = dt;
  plan->heads = headNum;
  plan->batch = batch;
  plan->block_size = (int32_t)bs;
  plan->max_blocks = (int32_t)max_blocks;
  plan->calc_type = calcType;
  plan->mask_type = maskType;
  plan->qk_scale = qkScale;
  plan->tokens = tokens;
  plan->num_blocks = ctKV->dims[0];
  plan->q_nope = qNope->data;
  plan->q_rope = qRope->data;
  plan->ct_kv = ctKV->data;
  plan->k_rope = kRope->data;
  plan->out = attenOut->data;
  plan->lse = lse && lse->data ? static_cast<float*>(lse->data) : nullptr;
  plan->block_tables = static_cast<const int32_t*>(blockTables->data);
  plan->ctx.assign(cl, cl + batch);
  plan->qs.assign(batch, 1);
  if (qs) plan->qs.assign(qs, qs + batch);
  plan->ws_size = 256;
  plan->image.assign(plan->ws_size, 0);
  return ALA_OK;
}

int mla_run(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t n) {
  (void)plan;
  (void)workspace;
  (void)stream;
  return mfail(err, n, ALA_UNSUPPORTED, "MLA kernel not built yet");
}

}  // namespace ala
