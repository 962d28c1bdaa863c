// api.cpp -- host side of the C ABI declared in include/ala.h: argument
// validation, the per-call schedule (work units packed longest first onto
// the CTAs, each CTA's list in (sequence, kv head) order), the workspace
// layout, TMA descriptor encoding and the kernel launches.
//
// Validation never touches the GPU, so every error path is testable on a
// machine without one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <queue>
#include <string>
#include <utility>
#include <vector>

#include "../../include/ala.h"
#include "internal.h"
#include "mla.h"

using namespace ala;

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int ok() {
  g_last_error.clear();
  return ALA_OK;
}

constexpr uint64_t kAlign = 256;
// SMs of the B200 the persistent prefill grid is planned for (one CTA per SM).  On a
// part with another SM count the grid still runs correctly, with CTAs queued or SMs idle.
constexpr size_t kPlannedSms = 148;
uint64_t align_up(uint64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int elem_size(int32_t dtype) { return dtype == ALA_F32 || dtype == ALA_I32 ? 4 : 2; }

int64_t numel(const ala_tensor* t) {
  int64_t n = 1;
  for (int i = 0; i < t->ndim; ++i) n *= t->dims[i];
  return n;
}

bool valid_tensor_header(const ala_tensor* t) {
  if (t->ndim < 1 || t->ndim > 4) return false;
  for (int i = 0; i < t->ndim; ++i)
    if (t->dims[i] < 0) return false;
  return true;
}

// ------------------------------------------------------------------ TMA encode
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

CUtensorMapDataType tma_dtype(int32_t dtype) {
  return dtype == ALA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                          : dtype == ALA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

}  // namespace

namespace ala {
bool encode_rows_heads_d(CUtensorMap* map, void* base, int32_t dtype, int64_t rows, int64_t heads, int64_t d,
                         int box_rows, bool mn_major_operand) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  const int es = elem_size(dtype);
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)std::max<int64_t>(rows, 1)};
  cuuint64_t strides[2] = {(cuuint64_t)(d * es), (cuuint64_t)(heads * d * es)};
  cuuint32_t box[3] = {(cuuint32_t)(128 / es), 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw =
      (mn_major_operand && es == 4) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  return enc(map, tma_dtype(dtype), 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace ala

// ------------------------------------------------------------------ op
// Page-locked copy of a host image, made on first use so the per-call upload
// is a plain asynchronous DMA (host memory only; no device memory is allocated).
struct PinnedImage {
  void* ptr = nullptr;
  size_t size = 0;
  ~PinnedImage() {
    if (ptr) cudaFreeHost(ptr);
  }
  const void* get(const std::vector<uint8_t>& img) {
    if (!ptr && !img.empty()) {
      if (cudaHostAlloc(&ptr, img.size(), cudaHostAllocDefault) != cudaSuccess) {
        ptr = nullptr;
        cudaGetLastError();
        return img.data();  // fall back to a staged copy from pageable memory
      }
      std::memcpy(ptr, img.data(), img.size());
      size = img.size();
    }
    return ptr ? ptr : img.data();
  }
};

struct ala_op {
  enum Kind { kPrefill, kMla } kind = kPrefill;
  // prefill
  int32_t dtype = 0, heads = 0, kv_heads = 0, head_size = 0, mask_type = 0, batch = 0;
  float qk_scale = 1.f;
  bool paged = false;
  int32_t block_size = 0, max_blocks = 0;
  int64_t n_tokens = 0, kv_rows = 0;  // kv_rows: nKvTokens or numBlocks*blockSize
  void *q = nullptr, *k = nullptr, *v = nullptr, *out = nullptr;
  const int32_t* block_tables = nullptr;
  const float* slopes = nullptr;
  float* lse = nullptr;
  uint64_t off_seqs = 0, off_units = 0, off_ctas = 0, ws_size = 0;
  int32_t n_units = 0, n_ctas = 0;
  std::vector<uint8_t> image;  // host copy of the workspace header (status, seqs, units)
  PinnedImage pinned;
  bool maps_ready = false;
  CUtensorMap tmQ, tmK, tmV;
  const void* bound_ws = nullptr;  // a workspace that holds this op's schedule (ala_op_bind_workspace)
  // mla
  MlaPlan mla;
};

extern "C" const char* ala_last_error(void) { return g_last_error.c_str(); }

namespace ala {
// Lets other translation units of the library report through ala_last_error.
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace ala

extern "C" void ala_op_destroy(ala_op* op) { delete op; }

extern "C" int ala_op_bind_workspace(ala_op* op, void* workspace, uint64_t workspaceSize, ala_stream_t stream) {
  NvtxRange nvtx_range("ala_op_bind_workspace");
  const char* fn = "ala_op_bind_workspace";
  if (!op) return fail(ALA_NULL_REQUIRED, "%s: op is NULL", fn);
  if (!workspace) {  // unbind
    op->bound_ws = nullptr;
    op->mla.bound_ws = nullptr;
    return ok();
  }
  const bool mla = op->kind == ala_op::kMla;
  const uint64_t need = mla ? op->mla.ws_size : op->ws_size;
  if (workspaceSize < need)
    return fail(ALA_WORKSPACE_TOO_SMALL, "%s: workspace %llu < required %llu", fn, (unsigned long long)workspaceSize,
                (unsigned long long)need);
  if (reinterpret_cast<uintptr_t>(workspace) % (mla ? 256 : 16))
    return fail(ALA_INVALID_PARAM, "%s: workspace must be %d-byte aligned", fn, mla ? 256 : 16);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  op->bound_ws = nullptr;
  op->mla.bound_ws = nullptr;
  if (mla) {
    char err[512] = {0};
    const int s = mla_upload(&op->mla, workspace, st, err, sizeof err);
    if (s != ALA_OK) return fail(s, "%s: %s", fn, err);
  } else if (cudaMemcpyAsync(workspace, op->pinned.get(op->image), op->ws_size, cudaMemcpyHostToDevice, st) !=
             cudaSuccess) {
    return fail(ALA_CUDA_ERROR, "%s: schedule upload failed: %s", fn, cudaGetErrorString(cudaGetLastError()));
  }
  // complete before returning, so that executions on any stream find the schedule in place
  if (cudaStreamSynchronize(st) != cudaSuccess)
    return fail(ALA_CUDA_ERROR, "%s: stream sync failed: %s", fn, cudaGetErrorString(cudaGetLastError()));
  if (mla) op->mla.bound_ws = workspace;
  else op->bound_ws = workspace;
  return ok();
}

extern "C" int ala_workspace_status(const ala_op* op, const void* workspace, ala_stream_t stream, int32_t* code) {
  NvtxRange nvtx_range("ala_workspace_status");
  if (!op || !workspace || !code) return fail(ALA_NULL_REQUIRED, "ala_workspace_status: null argument");
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(ALA_CUDA_ERROR, "ala_workspace_status: stream sync failed: %s",
                cudaGetErrorString(cudaGetLastError()));
  // word 0: a bounded wait that ran out; word 1: a bad block-table entry seen by a range-checking build
  int32_t v[2] = {0, 0};
  if (cudaMemcpy(v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(ALA_CUDA_ERROR, "ala_workspace_status: copy failed");
  *code = v[0] != 0 ? v[0] : v[1];
  return ok();
}

namespace {

// Shared checks and schedule for the prefill-type ops.
int build_prefill(ala_op* op, const ala_tensor* query, const ala_tensor* key, const ala_tensor* value,
                  const ala_tensor* blockTables, const ala_tensor* seqLen, const ala_tensor* kvSeqLen,
                  const ala_tensor* slopes, int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale,
                  ala_tensor* attnOut, ala_tensor* lse, const char* fn) {
  if (!query || !key || !value || !seqLen || !kvSeqLen || !attnOut)
    return fail(ALA_NULL_REQUIRED, "%s: query, key, value, seqLen, kvSeqLen and attnOut are required", fn);
  if (!query->data || !key->data || !value->data || !attnOut->data || !seqLen->data || !kvSeqLen->data)
    return fail(ALA_NULL_REQUIRED, "%s: a required tensor has a NULL data pointer", fn);
  for (const ala_tensor* t : {query, key, value, seqLen, kvSeqLen, (const ala_tensor*)attnOut})
    if (!valid_tensor_header(t)) return fail(ALA_INVALID_SHAPE, "%s: tensor with bad ndim or negative dim", fn);
  if (headNum <= 0) return fail(ALA_INVALID_PARAM, "%s: headNum must be > 0 (got %d)", fn, headNum);
  if (kvHeadNum <= 0 || headNum % kvHeadNum != 0)
    return fail(ALA_INVALID_PARAM, "%s: kvHeadNum must be > 0 and divide headNum (%d, %d)", fn, headNum, kvHeadNum);
  if (!(maskType == 0 || maskType == 3 || maskType == 4 || maskType == 5 || maskType == 9))
    return fail(ALA_INVALID_PARAM, "%s: maskType %d not in {0,3,4,5,9}", fn, maskType);
  if (!std::isfinite(qkScale)) return fail(ALA_INVALID_PARAM, "%s: qkScale must be finite", fn);

  const int32_t dt = query->dtype;
  if (!(dt == ALA_F16 || dt == ALA_BF16 || dt == ALA_F32))
    return fail(ALA_INVALID_DTYPE, "%s: query dtype must be f16, bf16 or f32", fn);
  if (key->dtype != dt || value->dtype != dt || attnOut->dtype != dt)
    return fail(ALA_INVALID_DTYPE, "%s: key, value and attnOut must have the query's dtype", fn);
  if (reinterpret_cast<uintptr_t>(attnOut->data) % 32)
    return fail(ALA_INVALID_PARAM, "%s: attnOut must be 32-byte aligned (the kernel writes rows in 32-byte pieces)", fn);
  if (seqLen->dtype != ALA_I32 || kvSeqLen->dtype != ALA_I32)
    return fail(ALA_INVALID_DTYPE, "%s: seqLen and kvSeqLen must be int32 (host)", fn);

  // query: [nTokens, headNum*headSize] or [nTokens, headNum, headSize]
  int64_t n_tokens = query->dims[0], head_size = 0;
  if (query->ndim == 2) {
    if (query->dims[1] % headNum) return fail(ALA_INVALID_SHAPE, "%s: query hidden size not divisible by headNum", fn);
    head_size = query->dims[1] / headNum;
  } else if (query->ndim == 3) {
    if (query->dims[1] != headNum) return fail(ALA_INVALID_SHAPE, "%s: query dims[1] != headNum", fn);
    head_size = query->dims[2];
  } else {
    return fail(ALA_INVALID_SHAPE, "%s: query must be 2-D or 3-D", fn);
  }
  if (attnOut->ndim != query->ndim)
    return fail(ALA_INVALID_SHAPE, "%s: attnOut must have the query's shape", fn);
  for (int i = 0; i < query->ndim; ++i)
    if (attnOut->dims[i] != query->dims[i]) return fail(ALA_INVALID_SHAPE, "%s: attnOut must have the query's shape", fn);

  const bool alibi = maskType == 3 || maskType == 4 || maskType == 5;
  if (alibi && head_size > 128)
    return fail(ALA_INVALID_PARAM, "%s: headSize must be <= 128 with ALiBi masks (got %lld)", fn, (long long)head_size);
  if (alibi && (!slopes || !slopes->data))
    return fail(ALA_NULL_REQUIRED, "%s: slopes are required for maskType %d", fn, maskType);
  if (!alibi && slopes && slopes->data)
    return fail(ALA_INVALID_PARAM, "%s: slopes must be NULL for maskType %d", fn, maskType);
  if (alibi) {
    if (slopes->dtype != ALA_F32) return fail(ALA_INVALID_DTYPE, "%s: slopes must be fp32", fn);
    if (slopes->ndim != 1 || slopes->dims[0] != headNum)
      return fail(ALA_INVALID_SHAPE, "%s: slopes must be [headNum]", fn);
  }

  // key/value
  const bool paged = blockTables != nullptr;
  int64_t kv_rows = 0;
  int32_t block_size = 0, max_blocks = 0;
  for (const ala_tensor* t : {key, value}) {
    int64_t hd = 0, rows = 0, bsz = 0;
    if (paged) {
      if (t->ndim == 3) {
        rows = t->dims[0];
        bsz = t->dims[1];
        hd = t->dims[2];
        if (hd != (int64_t)kvHeadNum * head_size) return fail(ALA_INVALID_SHAPE, "%s: key/value hidden != kvHeadNum*headSize", fn);
      } else if (t->ndim == 4) {
        rows = t->dims[0];
        bsz = t->dims[1];
        if (t->dims[2] != kvHeadNum || t->dims[3] != head_size)
          return fail(ALA_INVALID_SHAPE, "%s: key/value must be [numBlocks, blockSize, kvHeadNum, headSize]", fn);
      } else {
        return fail(ALA_INVALID_SHAPE, "%s: paged key/value must be 3-D or 4-D", fn);
      }
      if (t == value && (rows != key->dims[0] || bsz != key->dims[1]))
        return fail(ALA_INVALID_SHAPE, "%s: key and value caches differ in shape", fn);
      block_size = (int32_t)bsz;
      kv_rows = rows * bsz;
    } else {
      if (t->ndim != 3 || t->dims[1] != kvHeadNum || t->dims[2] != head_size)
        return fail(ALA_INVALID_SHAPE, "%s: key/value must be [nKvTokens, kvHeadNum, headSize]", fn);
      if (t == value && t->dims[0] != key->dims[0]) return fail(ALA_INVALID_SHAPE, "%s: key and value differ in length", fn);
      kv_rows = t->dims[0];
    }
  }
  if (paged) {
    if (!blockTables->data) return fail(ALA_NULL_REQUIRED, "%s: blockTables data is NULL", fn);
    if (blockTables->dtype != ALA_I32) return fail(ALA_INVALID_DTYPE, "%s: blockTables must be int32", fn);
    if (blockTables->ndim != 2) return fail(ALA_INVALID_SHAPE, "%s: blockTables must be [batch, maxBlockNum]", fn);
    if (!(block_size > 0 && block_size % 16 == 0))
      return fail(ALA_UNSUPPORTED, "%s: blockSize %d must be a multiple of 16", fn, block_size);
    max_blocks = (int32_t)blockTables->dims[1];
  }
  if (kv_rows >= (int64_t)1 << 31 || n_tokens >= (int64_t)1 << 31)
    return fail(ALA_UNSUPPORTED, "%s: more than 2^31 rows", fn);

  // metadata (host)
  if (seqLen->ndim != 1 || kvSeqLen->ndim != 1 || seqLen->dims[0] != kvSeqLen->dims[0])
    return fail(ALA_INVALID_SHAPE, "%s: seqLen and kvSeqLen must both be [batch]", fn);
  const int32_t batch = (int32_t)seqLen->dims[0];
  if (paged && blockTables->dims[0] != batch) return fail(ALA_INVALID_SHAPE, "%s: blockTables rows != batch", fn);
  const int32_t* sl = static_cast<const int32_t*>(seqLen->data);
  const int32_t* kl = static_cast<const int32_t*>(kvSeqLen->data);
  int64_t sum_q = 0, sum_kv = 0;
  for (int32_t b = 0; b < batch; ++b) {
    if (sl[b] < 0) return fail(ALA_INVALID_PARAM, "%s: seqLen[%d] = %d < 0", fn, b, sl[b]);
    if (kl[b] < sl[b]) return fail(ALA_INVALID_PARAM, "%s: kvSeqLen[%d] = %d < seqLen[%d] = %d", fn, b, kl[b], b, sl[b]);
    if (paged && (kl[b] + block_size - 1) / block_size > max_blocks)
      return fail(ALA_INVALID_PARAM, "%s: kvSeqLen[%d] = %d needs more than maxBlockNum = %d blocks", fn, b, kl[b],
                  max_blocks);
    sum_q += sl[b];
    sum_kv += kl[b];
  }
  if (sum_q != n_tokens) return fail(ALA_INVALID_SHAPE, "%s: sum(seqLen) = %lld != nTokens = %lld", fn, (long long)sum_q, (long long)n_tokens);
  if (!paged && sum_kv != kv_rows)
    return fail(ALA_INVALID_SHAPE, "%s: sum(kvSeqLen) = %lld != nKvTokens = %lld", fn, (long long)sum_kv, (long long)kv_rows);
  if (lse) {
    if (!lse->data) return fail(ALA_NULL_REQUIRED, "%s: lse data is NULL", fn);
    if (lse->dtype != ALA_F32) return fail(ALA_INVALID_DTYPE, "%s: lse must be fp32", fn);
    if (numel(lse) != n_tokens * headNum || lse->dims[0] != n_tokens)
      return fail(ALA_INVALID_SHAPE, "%s: lse must be [nTokens, headNum]", fn);
  }
  if (prefill_kernel_d(dt, head_size) == 0)
    return fail(ALA_UNSUPPORTED,
                "%s: headSize %lld with this dtype is not built (bf16/f16: a multiple of 8 up to 256; f32: a "
                "multiple of 8 up to 64)",
                fn, (long long)head_size);

  op->kind = ala_op::kPrefill;
  op->dtype = dt;
  op->heads = headNum;
  op->kv_heads = kvHeadNum;
  op->head_size = (int32_t)head_size;
  op->mask_type = maskType;
  op->batch = batch;
  op->qk_scale = qkScale;
  op->paged = paged;
  op->block_size = block_size;
  op->max_blocks = max_blocks;
  op->n_tokens = n_tokens;
  op->kv_rows = kv_rows;
  op->q = query->data;
  op->k = key->data;
  op->v = value->data;
  op->out = attnOut->data;
  op->block_tables = paged ? static_cast<const int32_t*>(blockTables->data) : nullptr;
  op->slopes = alibi ? static_cast<const float*>(slopes->data) : nullptr;
  op->lse = lse ? static_cast<float*>(lse->data) : nullptr;

  // schedule: units of up to two 128-row blocks that share a kv head, each visiting key tiles up to
  // its last allowed key (prefill_units)
  std::vector<SeqInfo> seqs(batch);
  for (int32_t b = 0, cq = 0, ckv = 0; b < batch; cq += sl[b], ckv += kl[b], ++b) seqs[b] = SeqInfo{cq, sl[b], kl[b], ckv};
  const PrefillShape shape = prefill_shape(prefill_kernel_d(dt, head_size));
  std::vector<PrefillUnit> units;
  units.reserve(prefill_unit_count(batch, sl, headNum, kvHeadNum, shape));
  prefill_units(batch, sl, kl, maskType, headNum, kvHeadNum, shape, [&](const PrefillUnit& u) { units.push_back(u); });
  // Persistent grid: one CTA per SM, each running a list of units.  Units are
  // assigned longest first to the least loaded CTA (greedy LPT); a unit costs
  // its key tiles plus about one tile of fixed work (Q load, epilogue).
  auto cost = prefill_unit_cost;
  std::stable_sort(units.begin(), units.end(),
                   [&](const PrefillUnit& a, const PrefillUnit& b) { return cost(a) > cost(b); });
  const int32_t n_ctas = (int32_t)std::min<size_t>(units.size(), kPlannedSms);
  std::vector<std::vector<int32_t>> lists(std::max(n_ctas, 1));
  {
    std::priority_queue<std::pair<int64_t, int32_t>, std::vector<std::pair<int64_t, int32_t>>, std::greater<>> load;
    for (int32_t c = 0; c < n_ctas; ++c) load.push({0, c});
    for (size_t i = 0; i < units.size(); ++i) {
      auto [l, c] = load.top();
      load.pop();
      lists[c].push_back((int32_t)i);
      load.push({l + cost(units[i]), c});
    }
  }
  // Each CTA then runs its units in (sequence, kv head) order, longest first within one head: every CTA
  // walks the heads in the same order, so the units running at one time read the K/V of a few heads,
  // which stay in L2 (in longest-first order every head's K/V is read at once, and over long sequences
  // that overflows L2).  A CTA's load is its units' sum, so the order leaves the balance as it is.
  const int32_t group = headNum / kvHeadNum;
  for (auto& list : lists)
    std::stable_sort(list.begin(), list.end(), [&](int32_t x, int32_t y) {
      const PrefillUnit &a = units[x], &c = units[y];
      return a.b != c.b ? a.b < c.b : a.head[0] / group < c.head[0] / group;
    });
  std::vector<PrefillUnit> ordered;
  std::vector<int32_t> offsets(n_ctas + 1, 0);
  ordered.reserve(units.size());
  for (int32_t c = 0; c < n_ctas; ++c) {
    for (int32_t i : lists[c]) ordered.push_back(units[i]);
    offsets[c + 1] = (int32_t)ordered.size();
  }
  op->n_units = (int32_t)units.size();
  op->n_ctas = n_ctas;
  op->off_seqs = kAlign;
  op->off_units = align_up(op->off_seqs + sizeof(SeqInfo) * std::max(batch, 1));
  op->off_ctas = align_up(op->off_units + sizeof(PrefillUnit) * std::max<size_t>(units.size(), 1));
  op->ws_size = align_up(op->off_ctas + sizeof(int32_t) * (n_ctas + 1));
  op->image.assign(op->ws_size, 0);
  std::memcpy(op->image.data() + op->off_seqs, seqs.data(), sizeof(SeqInfo) * batch);
  std::memcpy(op->image.data() + op->off_units, ordered.data(), sizeof(PrefillUnit) * ordered.size());
  std::memcpy(op->image.data() + op->off_ctas, offsets.data(), sizeof(int32_t) * (n_ctas + 1));
  return ALA_OK;
}

int run_prefill(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream, const char* fn) {
  if (!op) return fail(ALA_NULL_REQUIRED, "%s: op is NULL", fn);
  if (op->kind != ala_op::kPrefill) return fail(ALA_INVALID_PARAM, "%s: op was not made for this entry point", fn);
  if (!workspace) return fail(ALA_NULL_REQUIRED, "%s: workspace is NULL", fn);
  if (workspaceSize < op->ws_size)
    return fail(ALA_WORKSPACE_TOO_SMALL, "%s: workspace %llu < required %llu", fn, (unsigned long long)workspaceSize,
                (unsigned long long)op->ws_size);
  if (reinterpret_cast<uintptr_t>(workspace) % 16) return fail(ALA_INVALID_PARAM, "%s: workspace must be 16-byte aligned", fn);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!op->maps_ready) {
    const int tk = prefill_shape(prefill_kernel_d(op->dtype, op->head_size)).tile_keys;
    const int kv_box = op->paged ? kv_box_rows(op->block_size, tk) : tk;
    const int64_t q_rows = op->n_tokens;
    if (!encode_rows_heads_d(&op->tmQ, op->q, op->dtype, q_rows, op->heads, op->head_size, 128, false) ||
        !encode_rows_heads_d(&op->tmK, op->k, op->dtype, op->kv_rows, op->kv_heads, op->head_size, kv_box, false) ||
        !encode_rows_heads_d(&op->tmV, op->v, op->dtype, op->kv_rows, op->kv_heads, op->head_size, kv_box, true))
      return fail(ALA_CUDA_ERROR, "%s: cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)", fn);
    op->maps_ready = true;
  }
  // a bound workspace already holds the schedule and status words that only a failed execution sets
  // (ala_op_bind_workspace); any other workspace gets both copied in
  if (workspace != op->bound_ws &&
      cudaMemcpyAsync(workspace, op->pinned.get(op->image), op->ws_size, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return fail(ALA_CUDA_ERROR, "%s: schedule upload failed: %s", fn, cudaGetErrorString(cudaGetLastError()));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PrefillParams p{};
  p.units = reinterpret_cast<const PrefillUnit*>(ws + op->off_units);
  p.seqs = reinterpret_cast<const SeqInfo*>(ws + op->off_seqs);
  p.block_tables = op->block_tables;
  p.slopes = op->slopes;
  p.out = op->out;
  p.lse = op->lse;
  p.status = reinterpret_cast<int*>(ws);
  p.n_units = op->n_units;
  p.cta_offsets = reinterpret_cast<const int32_t*>(ws + op->off_ctas);
  p.n_ctas = op->n_ctas;
  p.max_blocks = op->max_blocks;
  p.block_size = op->block_size;
  p.oob_row = (int32_t)op->kv_rows;
  p.mask_type = op->mask_type;
  p.heads = op->heads;
  p.group = op->heads / op->kv_heads;
  p.scale_log2 = op->qk_scale * 1.4426950408889634f;
  p.d_out = op->head_size;
  const int tile_keys = prefill_shape(prefill_kernel_d(op->dtype, op->head_size)).tile_keys;
  p.kv_box_rows = op->paged ? kv_box_rows(op->block_size, tile_keys) : tile_keys;
  cudaError_t e = launch_prefill(op->dtype, prefill_kernel_d(op->dtype, op->head_size), op->tmQ, op->tmK, op->tmV, p, st);
  if (e != cudaSuccess) return fail(ALA_CUDA_ERROR, "%s: kernel launch failed: %s", fn, cudaGetErrorString(e));
  return ok();
}

}  // namespace

namespace {
int plan_prefix_encoder(const ala_tensor* query, const ala_tensor* key, const ala_tensor* value,
                        const ala_tensor* blockTables, const ala_tensor* mask, const ala_tensor* seqLen,
                        const ala_tensor* kvSeqLen, const ala_tensor* slopes, int maskType, int32_t headNum,
                        int32_t kvHeadNum, float qkScale, ala_tensor* attnOut, ala_tensor* lse,
                        uint64_t* workspaceSize, ala_op** op, const char* fn) {
  if (!workspaceSize || !op) return fail(ALA_NULL_REQUIRED, "%s: workspaceSize and op are required", fn);
  *op = nullptr;
  if (!blockTables) return fail(ALA_NULL_REQUIRED, "%s: blockTables is required", fn);
  if (!(maskType == 3 || maskType == 4 || maskType == 5 || maskType == 9))
    return fail(ALA_INVALID_PARAM, "%s: maskType %d not in {3,4,5,9}", fn, maskType);
  if (query && query->dtype == ALA_F32) return fail(ALA_INVALID_DTYPE, "%s: query must be f16 or bf16", fn);
  if (mask && mask->data) {
    if (maskType != 3 && maskType != 4)
      return fail(ALA_INVALID_PARAM, "%s: mask must be NULL unless maskType is 3 or 4", fn);
    const bool sq = mask->ndim == 2 && mask->dims[0] == 256 && mask->dims[1] == 256;
    const bool per_head = mask->ndim == 3 && mask->dims[0] == headNum && mask->dims[2] == 128;
    if (!sq && !per_head) return fail(ALA_INVALID_SHAPE, "%s: mask must be [256,256] or [headNum,seqLen,128]", fn);
  }
  ala_op* o = new ala_op();
  int st = build_prefill(o, query, key, value, blockTables, seqLen, kvSeqLen, slopes, maskType, headNum, kvHeadNum,
                         qkScale, attnOut, lse, fn);
  if (st != ALA_OK) {
    delete o;
    return st;
  }
  *workspaceSize = o->ws_size;
  *op = o;
  return ok();
}
}  // namespace

extern "C" int atb_like_prefix_encoder_get_workspace_size(
    const ala_tensor* query, const ala_tensor* key, const ala_tensor* value, const ala_tensor* blockTables,
    const ala_tensor* mask, const ala_tensor* seqLen, const ala_tensor* kvSeqLen, const ala_tensor* slopes,
    int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale, ala_tensor* attnOut, uint64_t* workspaceSize,
    ala_op** op) {
  NvtxRange nvtx_range("atb_like_prefix_encoder_get_workspace_size");
  return plan_prefix_encoder(query, key, value, blockTables, mask, seqLen, kvSeqLen, slopes, maskType, headNum,
                             kvHeadNum, qkScale, attnOut, nullptr, workspaceSize, op,
                             "atb_like_prefix_encoder_get_workspace_size");
}

extern "C" int atb_like_prefix_encoder_lse_get_workspace_size(
    const ala_tensor* query, const ala_tensor* key, const ala_tensor* value, const ala_tensor* blockTables,
    const ala_tensor* mask, const ala_tensor* seqLen, const ala_tensor* kvSeqLen, const ala_tensor* slopes,
    int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale, ala_tensor* attnOut, ala_tensor* lse,
    uint64_t* workspaceSize, ala_op** op) {
  NvtxRange nvtx_range("atb_like_prefix_encoder_lse_get_workspace_size");
  const char* fn = "atb_like_prefix_encoder_lse_get_workspace_size";
  if (!lse || !lse->data) return fail(ALA_NULL_REQUIRED, "%s: lse is required", fn);
  return plan_prefix_encoder(query, key, value, blockTables, mask, seqLen, kvSeqLen, slopes, maskType, headNum,
                             kvHeadNum, qkScale, attnOut, lse, workspaceSize, op, fn);
}

extern "C" int atb_like_prefix_encoder(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream) {
  NvtxRange nvtx_range("atb_like_prefix_encoder");
  return run_prefill(workspace, workspaceSize, op, stream, "atb_like_prefix_encoder");
}

extern "C" int varlen_attention_get_workspace_size(const ala_tensor* query, const ala_tensor* key,
                                                   const ala_tensor* value, const ala_tensor* seqLen,
                                                   const ala_tensor* kvSeqLen, const ala_tensor* slopes, int maskType,
                                                   int32_t headNum, int32_t kvHeadNum, float qkScale,
                                                   ala_tensor* attnOut, ala_tensor* lse, uint64_t* workspaceSize,
                                                   ala_op** op) {
  NvtxRange nvtx_range("varlen_attention_get_workspace_size");
  const char* fn = "varlen_attention_get_workspace_size";
  if (!workspaceSize || !op) return fail(ALA_NULL_REQUIRED, "%s: workspaceSize and op are required", fn);
  *op = nullptr;
  ala_op* o = new ala_op();
  int st = build_prefill(o, query, key, value, nullptr, seqLen, kvSeqLen, slopes, maskType, headNum, kvHeadNum,
                         qkScale, attnOut, lse, fn);
  if (st != ALA_OK) {
    delete o;
    return st;
  }
  *workspaceSize = o->ws_size;
  *op = o;
  return ok();
}

extern "C" int varlen_attention(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream) {
  NvtxRange nvtx_range("varlen_attention");
  return run_prefill(workspace, workspaceSize, op, stream, "varlen_attention");
}

// ------------------------------------------------------------------ MLA
extern "C" int atb_like_mla_get_workspace_size(const ala_tensor* qNope, const ala_tensor* qRope,
                                               const ala_tensor* ctKV, const ala_tensor* kRope,
                                               const ala_tensor* blockTables, const ala_tensor* contextLens,
                                               const ala_tensor* mask, const ala_tensor* qSeqLen,
                                               const ala_tensor* qkDescale, const ala_tensor* pvDescale,
                                               int32_t headNum, float qkScale, int32_t kvHeadNum, int maskType,
                                               int calcType, uint8_t cacheMode, ala_tensor* attenOut, ala_tensor* lse,
                                               uint64_t* workspaceSize, ala_op** op) {
  NvtxRange nvtx_range("atb_like_mla_get_workspace_size");
  const char* fn = "atb_like_mla_get_workspace_size";
  if (!workspaceSize || !op) return fail(ALA_NULL_REQUIRED, "%s: workspaceSize and op are required", fn);
  *op = nullptr;
  if (calcType == ALA_MLA_CALC_PREFILL) {
    // full prefill: every query token of a batch attends causally to the keys up to its own position, i.e.
    // token t of the qseqlen new tokens allows keys j <= contextLens - qseqlen + t (the speculative rule)
    if (!qSeqLen || !qSeqLen->data) return fail(ALA_NULL_REQUIRED, "%s: qseqlen is required with calcType PREFILL", fn);
    if (maskType != ALA_MLA_MASK_UNDEFINED && maskType != ALA_MLA_MASK_SPEC)
      return fail(ALA_INVALID_PARAM, "%s: calcType PREFILL takes maskType UNDEFINED or SPEC (causal either way)", fn);
    if (mask && mask->data)
      return fail(ALA_INVALID_PARAM, "%s: calcType PREFILL generates its causal mask; mask must be NULL", fn);
    calcType = ALA_MLA_CALC_SPEC;
    maskType = ALA_MLA_MASK_SPEC;
  }
  if (calcType == ALA_MLA_CALC_RING) {
    // ring attention: the same attention over the keys this call is given, with the lse it needs to merge
    // the result with the other ranges' (ala_lse_merge); one token per batch, or qseqlen tokens with SPEC
    if (!lse || !lse->data) return fail(ALA_NULL_REQUIRED, "%s: lse is required with calcType RING", fn);
    calcType = (qSeqLen && qSeqLen->data) ? ALA_MLA_CALC_SPEC : ALA_MLA_CALC_UNDEFINED;
  }
  ala_op* o = new ala_op();
  o->kind = ala_op::kMla;
  char err[512] = {0};
  int st = mla_plan(&o->mla, qNope, qRope, ctKV, kRope, blockTables, contextLens, mask, qSeqLen, qkDescale,
                    pvDescale, headNum, qkScale, kvHeadNum, maskType, calcType, cacheMode, attenOut, lse, err,
                    sizeof err);
  if (st != ALA_OK) {
    delete o;
    return fail(st, "%s: %s", fn, err);
  }
  *workspaceSize = o->mla.ws_size;
  *op = o;
  return ok();
}

extern "C" int atb_like_mla(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream) {
  NvtxRange nvtx_range("atb_like_mla");
  const char* fn = "atb_like_mla";
  if (!op) return fail(ALA_NULL_REQUIRED, "%s: op is NULL", fn);
  if (op->kind != ala_op::kMla) return fail(ALA_INVALID_PARAM, "%s: op was not made by atb_like_mla_get_workspace_size", fn);
  if (!workspace) return fail(ALA_NULL_REQUIRED, "%s: workspace is NULL", fn);
  if (workspaceSize < op->mla.ws_size)
    return fail(ALA_WORKSPACE_TOO_SMALL, "%s: workspace %llu < required %llu", fn, (unsigned long long)workspaceSize,
                (unsigned long long)op->mla.ws_size);
  char err[512] = {0};
  int st = mla_run(&op->mla, workspace, reinterpret_cast<cudaStream_t>(stream), err, sizeof err);
  if (st != ALA_OK) return fail(st, "%s: %s", fn, err);
  return ok();
}

extern "C" int ala_lse_merge(const ala_tensor* outA, const ala_tensor* lseA, const ala_tensor* outB,
                             const ala_tensor* lseB, ala_tensor* out, ala_tensor* lse, ala_stream_t stream) {
  NvtxRange nvtx_range("ala_lse_merge");
  const char* fn = "ala_lse_merge";
  const ala_tensor* ts[6] = {outA, lseA, outB, lseB, out, lse};
  for (const ala_tensor* t : ts)
    if (!t || !t->data) return fail(ALA_NULL_REQUIRED, "%s: all six tensors are required", fn);
  const int32_t dt = outA->dtype;
  if (dt != ALA_BF16 && dt != ALA_F16 && dt != ALA_F32)
    return fail(ALA_INVALID_DTYPE, "%s: outputs must be bf16, f16 or f32", fn);
  if (outB->dtype != dt || out->dtype != dt) return fail(ALA_INVALID_DTYPE, "%s: outA, outB and out differ in dtype", fn);
  if (lseA->dtype != ALA_F32 || lseB->dtype != ALA_F32 || lse->dtype != ALA_F32)
    return fail(ALA_INVALID_DTYPE, "%s: lse tensors must be fp32", fn);
  if (outA->ndim < 1 || outA->ndim > 4) return fail(ALA_INVALID_SHAPE, "%s: outA must have 1 to 4 dims", fn);
  const ala_tensor* same[2] = {outB, out};
  for (const ala_tensor* t : same) {
    if (t->ndim != outA->ndim) return fail(ALA_INVALID_SHAPE, "%s: outA, outB and out differ in shape", fn);
    for (int i = 0; i < outA->ndim; ++i)
      if (t->dims[i] != outA->dims[i]) return fail(ALA_INVALID_SHAPE, "%s: outA, outB and out differ in shape", fn);
  }
  const int64_t d = outA->dims[outA->ndim - 1];
  if (d <= 0 || d > 1024) return fail(ALA_INVALID_SHAPE, "%s: the last dim must be in 1..1024", fn);
  int64_t rows = 1;
  for (int i = 0; i + 1 < outA->ndim; ++i) rows *= outA->dims[i];
  const ala_tensor* lses[3] = {lseA, lseB, lse};
  for (const ala_tensor* t : lses) {
    int64_t ne = 1;
    for (int i = 0; i < t->ndim; ++i) ne *= t->dims[i];
    if (t->ndim < 1 || t->ndim > 4 || ne != rows)
      return fail(ALA_INVALID_SHAPE, "%s: every lse must hold one value per output row", fn);
  }
  const cudaError_t e = ala::launch_lse_merge(dt, outA->data, static_cast<const float*>(lseA->data), outB->data,
                                              static_cast<const float*>(lseB->data), out->data,
                                              static_cast<float*>(lse->data), rows, (int)d,
                                              reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(ALA_CUDA_ERROR, "%s: %s", fn, cudaGetErrorString(e));
  return ok();
}
