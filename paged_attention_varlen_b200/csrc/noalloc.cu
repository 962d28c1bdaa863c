// noalloc.cu -- varlen_attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: runtimes that hand out only
// pre-sized arenas, or embedded hosts whose device allocator is owned by
// another component.  They can still pass their own inputs and outputs, but
// not a workspace.  This entry point runs the same prefill kernel as
// varlen_attention with its scratch (the status word, the per-sequence table
// and the work units) held in one fixed-size array in device global memory
// that belongs to this library.
//
// Costs and rules of that choice:
//   - the array is kNoAllocScratchBytes (1 MiB); every GPU that loads the
//     library keeps it until the process exits;
//   - a call whose schedule does not fit is rejected with ALA_UNSUPPORTED and
//     a message naming the limit;
//   - all calls share the one array, and each call rewrites it (status word
//     cleared to zero first): two calls whose work overlaps on the GPU race
//     on it, so callers must order them (one stream, or events);
//   - the schedule is uploaded from a static host buffer that the next call
//     rewrites, so a call made while its stream is being captured into a
//     graph is refused (a replay of that graph would read whatever schedule
//     the buffer holds by then);
//   - the first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (with that device current) and keeps it;
//   - varlen_attention_noalloc_status reads the array's status word, so a
//     bounded kernel wait that ran out is visible to the caller;
//   - nothing here calls cudaMalloc, cudaFree or any other allocating routine:
//     the schedule is built in a static host buffer and uploaded with one
//     cudaMemcpyAsync from it.  (A rejected call stores its message in the
//     thread's ala_last_error text, which is ordinary host memory.)
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/ala.h"
#include "internal.h"

namespace ala {
void set_last_error(const char* msg);
}

namespace {

using namespace ala;

constexpr size_t kNoAllocScratchBytes = 1u << 20;
constexpr size_t kStatusBytes = 256;
constexpr int kMaxBatch = 4096;
constexpr size_t kSeqBytes = sizeof(SeqInfo) * kMaxBatch;
constexpr size_t kMaxUnits = (kNoAllocScratchBytes - kStatusBytes - kSeqBytes) / sizeof(PrefillUnit);
constexpr int kMaxDevices = 64;

// the device-side scratch of this entry point: [status | SeqInfo[kMaxBatch] | PrefillUnit[kMaxUnits]]
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// host staging of the same layout; guarded by g_mutex together with the device address table
static uint8_t g_stage[kNoAllocScratchBytes];
static void* g_scratch_dev[kMaxDevices];
static std::mutex g_mutex;

int nfail(int status, const char* fmt, ...) {
  char buf[384];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_last_error(buf);
  return status;
}

bool dims_ok(const ala_tensor* t) {
  if (t->ndim < 1 || t->ndim > 4) return false;
  for (int i = 0; i < t->ndim; ++i)
    if (t->dims[i] < 0) return false;
  return true;
}

}  // namespace

extern "C" ALA_API int varlen_attention_noalloc(const ala_tensor* query, const ala_tensor* key,
                                                const ala_tensor* value, const ala_tensor* seqLen,
                                                const ala_tensor* kvSeqLen, const ala_tensor* slopes, int maskType,
                                                int32_t headNum, int32_t kvHeadNum, float qkScale,
                                                ala_tensor* attnOut, ala_tensor* lse, ala_stream_t stream) {
  NvtxRange nvtx_range("varlen_attention_noalloc");
  const char* fn = "varlen_attention_noalloc";
  // ---- the same argument rules as varlen_attention
  if (!query || !key || !value || !seqLen || !kvSeqLen || !attnOut || !query->data || !key->data || !value->data ||
      !seqLen->data || !kvSeqLen->data || !attnOut->data)
    return nfail(ALA_NULL_REQUIRED, "%s: query, key, value, seqLen, kvSeqLen and attnOut are required", fn);
  for (const ala_tensor* t : {query, key, value, seqLen, kvSeqLen, (const ala_tensor*)attnOut})
    if (!dims_ok(t)) return nfail(ALA_INVALID_SHAPE, "%s: tensor with bad ndim or negative dim", fn);
  if (headNum <= 0) return nfail(ALA_INVALID_PARAM, "%s: headNum must be > 0", fn);
  if (kvHeadNum <= 0 || headNum % kvHeadNum)
    return nfail(ALA_INVALID_PARAM, "%s: kvHeadNum must be > 0 and divide headNum", fn);
  if (!(maskType == 0 || maskType == 3 || maskType == 4 || maskType == 5 || maskType == 9))
    return nfail(ALA_INVALID_PARAM, "%s: maskType %d not in {0,3,4,5,9}", fn, maskType);
  if (!std::isfinite(qkScale)) return nfail(ALA_INVALID_PARAM, "%s: qkScale must be finite", fn);
  const int32_t dt = query->dtype;
  if (!(dt == ALA_F16 || dt == ALA_BF16 || dt == ALA_F32))
    return nfail(ALA_INVALID_DTYPE, "%s: query dtype must be f16, bf16 or f32", fn);
  if (key->dtype != dt || value->dtype != dt || attnOut->dtype != dt)
    return nfail(ALA_INVALID_DTYPE, "%s: key, value and attnOut must have the query's dtype", fn);
  if (reinterpret_cast<uintptr_t>(attnOut->data) % 32)
    return nfail(ALA_INVALID_PARAM, "%s: attnOut must be 32-byte aligned (the kernel writes rows in 32-byte pieces)", fn);
  if (seqLen->dtype != ALA_I32 || kvSeqLen->dtype != ALA_I32)
    return nfail(ALA_INVALID_DTYPE, "%s: seqLen and kvSeqLen must be int32 (host)", fn);
  if (query->ndim != 3 || query->dims[1] != headNum)
    return nfail(ALA_INVALID_SHAPE, "%s: query must be [nTokens, headNum, headSize]", fn);
  const int64_t n_tokens = query->dims[0], d = query->dims[2];
  if (attnOut->ndim != 3 || attnOut->dims[0] != n_tokens || attnOut->dims[1] != headNum || attnOut->dims[2] != d)
    return nfail(ALA_INVALID_SHAPE, "%s: attnOut must have the query's shape", fn);
  for (const ala_tensor* t : {key, value})
    if (t->ndim != 3 || t->dims[1] != kvHeadNum || t->dims[2] != d || t->dims[0] != key->dims[0])
      return nfail(ALA_INVALID_SHAPE, "%s: key/value must be [nKvTokens, kvHeadNum, headSize]", fn);
  const bool alibi = maskType == 3 || maskType == 4 || maskType == 5;
  if (alibi && d > 128) return nfail(ALA_INVALID_PARAM, "%s: headSize must be <= 128 with ALiBi masks", fn);
  if (alibi && (!slopes || !slopes->data)) return nfail(ALA_NULL_REQUIRED, "%s: slopes are required for ALiBi", fn);
  if (!alibi && slopes && slopes->data) return nfail(ALA_INVALID_PARAM, "%s: slopes must be NULL for maskType %d", fn, maskType);
  if (alibi && (slopes->dtype != ALA_F32 || slopes->ndim != 1 || slopes->dims[0] != headNum))
    return nfail(ALA_INVALID_SHAPE, "%s: slopes must be fp32 [headNum]", fn);
  if (prefill_kernel_d(dt, d) == 0)
    return nfail(ALA_UNSUPPORTED, "%s: headSize %lld with this dtype is not built", fn, (long long)d);
  if (seqLen->ndim != 1 || kvSeqLen->ndim != 1 || seqLen->dims[0] != kvSeqLen->dims[0])
    return nfail(ALA_INVALID_SHAPE, "%s: seqLen and kvSeqLen must both be [batch]", fn);
  if (lse && lse->data) {
    // [nTokens, headNum] or [nTokens, headNum, 1]: the kernel writes nTokens * headNum floats
    if (lse->dtype != ALA_F32) return nfail(ALA_INVALID_DTYPE, "%s: lse must be fp32", fn);
    const bool shape_ok = dims_ok(lse) && lse->dims[0] == n_tokens &&
                          ((lse->ndim == 2 && lse->dims[1] == headNum) ||
                           (lse->ndim == 3 && lse->dims[1] == headNum && lse->dims[2] == 1));
    if (!shape_ok) return nfail(ALA_INVALID_SHAPE, "%s: lse must be [nTokens, headNum] or [nTokens, headNum, 1]", fn);
  }
  const int32_t batch = (int32_t)seqLen->dims[0];
  if (batch > kMaxBatch)
    return nfail(ALA_UNSUPPORTED, "%s: batch %d exceeds the %d sequences the fixed scratch holds", fn, batch, kMaxBatch);
  const int32_t* sl = static_cast<const int32_t*>(seqLen->data);
  const int32_t* kl = static_cast<const int32_t*>(kvSeqLen->data);
  int64_t sum_q = 0, sum_kv = 0;
  for (int32_t b = 0; b < batch; ++b) {
    if (sl[b] < 0 || kl[b] < sl[b]) return nfail(ALA_INVALID_PARAM, "%s: need 0 <= seqLen[b] <= kvSeqLen[b]", fn);
    sum_q += sl[b];
    sum_kv += kl[b];
  }
  if (sum_q != n_tokens || sum_kv != key->dims[0])
    return nfail(ALA_INVALID_SHAPE, "%s: sum(seqLen) / sum(kvSeqLen) do not match the token counts", fn);
  if (n_tokens >= ((int64_t)1 << 31) || key->dims[0] >= ((int64_t)1 << 31))
    return nfail(ALA_UNSUPPORTED, "%s: more than 2^31 rows", fn);

  // ---- count the work units first, so an oversized call is rejected before anything is written
  const int32_t group = headNum / kvHeadNum;
  const PrefillShape shape = prefill_shape(prefill_kernel_d(dt, d));
  const int64_t n_units = prefill_unit_count(batch, sl, headNum, kvHeadNum, shape);
  if (n_units > (int64_t)kMaxUnits)
    return nfail(ALA_UNSUPPORTED, "%s: the call needs %lld work units; the fixed %zu-byte scratch holds at most %zu", fn,
                 (long long)n_units, kNoAllocScratchBytes, kMaxUnits);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &capture) != cudaSuccess)
    return nfail(ALA_CUDA_ERROR, "%s: cudaStreamIsCapturing failed: %s", fn, cudaGetErrorString(cudaGetLastError()));
  if (capture != cudaStreamCaptureStatusNone)
    return nfail(ALA_UNSUPPORTED,
                 "%s: the stream is being captured; the schedule upload reads a host buffer that later calls "
                 "rewrite, so a replayed capture would run another call's schedule",
                 fn);

  std::lock_guard<std::mutex> lock(g_mutex);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nfail(ALA_CUDA_ERROR, "%s: no usable current device", fn);
  if (!g_scratch_dev[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return nfail(ALA_CUDA_ERROR, "%s: cudaGetSymbolAddress failed: %s", fn, cudaGetErrorString(e));
    g_scratch_dev[dev] = ptr;
  }
  uint8_t* scratch = static_cast<uint8_t*>(g_scratch_dev[dev]);

  // ---- schedule into the static host stage: [status = 0 | SeqInfo[batch] | units]
  std::memset(g_stage, 0, kStatusBytes);
  SeqInfo* seqs = reinterpret_cast<SeqInfo*>(g_stage + kStatusBytes);
  PrefillUnit* units = reinterpret_cast<PrefillUnit*>(g_stage + kStatusBytes + kSeqBytes);
  size_t nu = 0;
  for (int32_t b = 0, cq = 0, ckv = 0; b < batch; cq += sl[b], ckv += kl[b], ++b) seqs[b] = SeqInfo{cq, sl[b], kl[b], ckv};
  prefill_units(batch, sl, kl, maskType, headNum, kvHeadNum, shape, [&](const PrefillUnit& u) { units[nu++] = u; });
  // longest first; ties in a fixed order so every call gets the same schedule
  std::sort(units, units + nu, [](const PrefillUnit& a, const PrefillUnit& c) {
    const int64_t ca = prefill_unit_cost(a), cc = prefill_unit_cost(c);
    if (ca != cc) return ca > cc;
    if (a.b != c.b) return a.b < c.b;
    if (a.q0[0] != c.q0[0]) return a.q0[0] < c.q0[0];
    return a.head[0] < c.head[0];
  });

  CUtensorMap tmQ, tmK, tmV;
  if (!encode_rows_heads_d(&tmQ, query->data, dt, n_tokens, headNum, d, 128, false) ||
      !encode_rows_heads_d(&tmK, key->data, dt, key->dims[0], kvHeadNum, d, shape.tile_keys, false) ||
      !encode_rows_heads_d(&tmV, value->data, dt, key->dims[0], kvHeadNum, d, shape.tile_keys, true))
    return nfail(ALA_CUDA_ERROR, "%s: cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)", fn);

  const size_t bytes = kStatusBytes + kSeqBytes + nu * sizeof(PrefillUnit);
  // pageable source on a stream that is not being captured: the copy is staged before this call
  // returns, so g_stage may be rewritten by the next call
  if (cudaMemcpyAsync(scratch, g_stage, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return nfail(ALA_CUDA_ERROR, "%s: schedule upload failed: %s", fn, cudaGetErrorString(cudaGetLastError()));

  PrefillParams p{};
  p.units = reinterpret_cast<const PrefillUnit*>(scratch + kStatusBytes + kSeqBytes);
  p.seqs = reinterpret_cast<const SeqInfo*>(scratch + kStatusBytes);
  p.block_tables = nullptr;
  p.slopes = alibi ? static_cast<const float*>(slopes->data) : nullptr;
  p.out = attnOut->data;
  p.lse = lse && lse->data ? static_cast<float*>(lse->data) : nullptr;
  p.status = reinterpret_cast<int*>(scratch);
  p.cta_offsets = nullptr;  // one CTA per work unit
  p.n_units = (int32_t)nu;
  p.n_ctas = (int32_t)nu;
  p.max_blocks = 0;
  p.block_size = 0;
  p.oob_row = (int32_t)key->dims[0];
  p.mask_type = maskType;
  p.heads = headNum;
  p.group = group;
  p.scale_log2 = qkScale * 1.4426950408889634f;
  p.d_out = (int32_t)d;
  p.kv_box_rows = shape.tile_keys;  // contiguous K/V: one box per tile
  const cudaError_t e = launch_prefill(dt, prefill_kernel_d(dt, d), tmQ, tmK, tmV, p, st);
  if (e != cudaSuccess) return nfail(ALA_CUDA_ERROR, "%s: kernel launch failed: %s", fn, cudaGetErrorString(e));
  set_last_error("");
  return ALA_OK;
}

extern "C" ALA_API int varlen_attention_noalloc_status(ala_stream_t stream, int32_t* code) {
  NvtxRange nvtx_range("varlen_attention_noalloc_status");
  const char* fn = "varlen_attention_noalloc_status";
  if (!code) return nfail(ALA_NULL_REQUIRED, "%s: code is NULL", fn);
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return nfail(ALA_CUDA_ERROR, "%s: stream sync failed: %s", fn, cudaGetErrorString(cudaGetLastError()));
  int32_t v[2] = {0, 0};
  // a copy out of the library's array by symbol: no allocation (word 1: a range-checking build's report)
  const cudaError_t e = cudaMemcpyFromSymbol(v, g_noalloc_scratch, sizeof v, 0, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return nfail(ALA_CUDA_ERROR, "%s: status read failed: %s", fn, cudaGetErrorString(e));
  *code = v[0] != 0 ? v[0] : v[1];
  set_last_error("");
  return ALA_OK;
}
