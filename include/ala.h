/*
 * ala.h -- C ABI of the B200 (sm_100a) packed-varlen / paged attention library
 * (libala.so).
 *
 * Operation: O = softmax(qkScale * Q K^T + M) V per sequence and head, over
 * query tokens packed back to back (per-sequence lengths instead of padding),
 * with K/V in a contiguous packed tensor or a paged cache read through a block
 * table.  M is never passed or built: it is generated in registers from the
 * mask type's rule.
 *   - formula: nalar.dev article on padding masks, section "Masking mengubah
 *     kelayakan relasi attention" (A = softmax(QK^T/sqrt(d) + M), O = AV; a
 *     masked pair gets zero probability);
 *   - two-phase API, argument names and shapes: ATB "PrefixEncoder" page
 *     (definition and parameter table) and ATB "MLA" page (definition and
 *     parameter table);
 *   - mask rules: ATB "压缩mask" (compressed mask) page, enabling and alibi
 *     sections; ATB "PrefixEncoder" page, parameter table, row maskType;
 *   - packing with cumulative offsets: nalar.dev article, section "Packing
 *     mengeluarkan padding dari representasi".
 *
 * Conventions shared by every entry point
 *   - Tensors are described by ala_tensor: a data pointer, a dtype code, the
 *     number of dims and the dims (row-major, densely packed).  Tensors marked
 *     (host) live in host memory and are read during *_get_workspace_size;
 *     every other tensor lives in device memory.
 *   - Ownership: the caller owns every tensor and the workspace.  The library
 *     allocates no device memory.  An ala_op owns host copies of the metadata
 *     and the schedule; later changes to host tensors do not affect it.  The
 *     device pointers captured in the op must stay valid while it is used.
 *   - *_get_workspace_size validates everything it can without touching the
 *     GPU, builds the schedule and returns the workspace size in bytes plus a
 *     new op.  The execute call (same name without the suffix) enqueues the
 *     work asynchronously on `stream`; the workspace must stay untouched until
 *     the stream has passed the call.  An op may be executed any number of
 *     times; free it with ala_op_destroy.
 *   - Every function returns an ala_status and never aborts; the text of the
 *     last error on the calling thread is returned by ala_last_error().
 *     Device faults surface at the caller's next synchronisation.  Kernel
 *     waits are bounded: a pipeline stall ends the kernel and leaves a nonzero
 *     code that ala_workspace_status() reads back.
 *   - Unused cache slots (past kvSeqLen in a sequence's last block, spare
 *     blocks) may hold any FINITE values; they never contribute.
 */
#ifndef ALA_H
#define ALA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ALA_API __attribute__((visibility("default")))
#else
#define ALA_API
#endif

typedef struct CUstream_st* ala_stream_t; /* same type as cudaStream_t */

/* dtype codes */
enum { ALA_F16 = 0, ALA_BF16 = 1, ALA_F32 = 2, ALA_I32 = 3, ALA_I8 = 4 };

typedef struct ala_tensor {
  void* data;
  int32_t dtype;
  int32_t ndim;
  int64_t dims[4];
} ala_tensor;

typedef enum ala_status {
  ALA_OK = 0,
  ALA_NULL_REQUIRED = 1,      /* a required tensor or pointer is NULL            */
  ALA_INVALID_SHAPE = 2,      /* dims inconsistent with each other or the params */
  ALA_INVALID_DTYPE = 3,      /* dtype not allowed for that argument              */
  ALA_INVALID_PARAM = 4,      /* scalar parameter or metadata out of range        */
  ALA_UNSUPPORTED = 5,        /* valid per the pages, not built here              */
  ALA_WORKSPACE_TOO_SMALL = 6,
  ALA_CUDA_ERROR = 7,         /* a CUDA runtime/driver call failed                */
  ALA_DEVICE_TIMEOUT = 8      /* a kernel wait ran out (ala_workspace_status)     */
} ala_status;

/* PrefixEncoder mask types (ATB "PrefixEncoder" page, parameter table, row
 * maskType), plus ALA_MASK_NONE for varlen_attention only. */
enum {
  ALA_MASK_NONE = 0,              /* every key of the sequence allowed              */
  ALA_MASK_ALIBI_COMPRESS = 3,    /* causal, bias slope_h*(j - iabs)                 */
  ALA_MASK_ALIBI_COMPRESS_SQRT = 4, /* causal, bias -slope_h*sqrt(iabs - j)          */
  ALA_MASK_ALIBI_COMPRESS_LEFT_ALIGN = 5, /* causal, bias slope_h*j                  */
  ALA_MASK_CAUSAL = 9             /* causal, generated inside                        */
};
/* Causal here means j <= iabs with iabs = i + (kvSeqLen_b - seqLen_b): the new
 * tokens are the last seqLen_b of the kvSeqLen_b keys (prefix offset). */

/* MLA enums (ATB "MLA" page, parameter table, rows maskType/calcType/cacheMode). */
enum { ALA_MLA_MASK_UNDEFINED = 0, ALA_MLA_MASK_SPEC = 1, ALA_MLA_MASK_FREE = 2 };
enum { ALA_MLA_CALC_UNDEFINED = 0, ALA_MLA_CALC_SPEC = 1, ALA_MLA_CALC_RING = 2, ALA_MLA_CALC_PREFILL = 3 };
enum { ALA_MLA_CACHE_KVCACHE = 0, ALA_MLA_CACHE_KROPE_CTKV = 1, ALA_MLA_CACHE_INT8_NZ = 2, ALA_MLA_CACHE_NZ = 3 };

typedef struct ala_op ala_op;

/* Text of the last error on the calling thread ("" if none). */
ALA_API const char* ala_last_error(void);

/* Frees an op (NULL is allowed). */
ALA_API void ala_op_destroy(ala_op* op);

/* Binds `workspace` to `op`: copies the op's schedule (the host metadata the
 * planning call built, with cleared status words) into it and waits for that
 * copy on `stream`.  Later executions of `op` into this same workspace pointer
 * skip the copy (~10 us of host-to-device latency per call) and launch their
 * kernels only; executions into any other workspace copy the schedule as
 * before.  The status words of a bound workspace are not cleared between
 * executions: a code that an execution records there stays until the
 * workspace is bound again (ala_workspace_status reports it), and a wait
 * timeout's code makes later executions return at once without writing their
 * outputs.  While bound, the caller guarantees that nothing else writes to
 * the workspace (an execution of another op into it included: that would
 * replace the schedule this op's executions read) and that it stays
 * allocated; binding a NULL workspace unbinds.  Status: ALA_NULL_REQUIRED (op NULL),
 * ALA_WORKSPACE_TOO_SMALL, ALA_INVALID_PARAM (misaligned: 16 bytes for the
 * prefill ops, 256 for MLA), ALA_CUDA_ERROR. */
ALA_API int ala_op_bind_workspace(ala_op* op, void* workspace, uint64_t workspaceSize, ala_stream_t stream);

/* Reads the device status word of `workspace` for `op` (synchronous copy on
 * the legacy stream after synchronising `stream`).  *code = 0 means every
 * kernel wait completed; 0x101..0x10A identifies the wait that ran out; 0x10B
 * (range-checking build libala_debug.so only) means a block-table entry that
 * was read lay outside [0, numBlocks): that page was read as zeros. */
ALA_API int ala_workspace_status(const ala_op* op, const void* workspace, ala_stream_t stream, int32_t* code);

/* ---------------------------------------------------------------------------
 * PrefixEncoder (ATB "PrefixEncoder" page, definition and parameter table).
 *
 * query       [nTokens, headNum*headSize] or [nTokens, headNum, headSize]
 *             f16/bf16, device.  Tokens of sequence b are packed at
 *             [sum_{c<b} seqLen_c, + seqLen_b).
 * key, value  paged cache [numBlocks, blockSize, kvHeadNum*headSize] or
 *             [numBlocks, blockSize, kvHeadNum, headSize], same dtype, device.
 *             Key position j of sequence b is slot j % blockSize of block
 *             blockTables[b][j / blockSize].  blockSize must be a multiple
 *             of 16 (the kernels gather each key tile in boxes of
 *             gcd(blockSize, keys per tile) rows, each inside one page).
 * blockTables [batch, maxBlockNum] int32, device.  Entries past
 *             ceil(kvSeqLen_b / blockSize) are never read; entries read must
 *             be in [0, numBlocks).
 * mask        NULL, or for maskType 3/4 a [256,256] or [headNum,seqLen,128]
 *             compressed bias, which is accepted and ignored: the bias is
 *             regenerated from the rule.  Must be NULL for 5 and 9.
 * seqLen      [batch] int32, HOST: new query tokens per sequence (>= 0).
 * kvSeqLen    [batch] int32, HOST: keys per sequence = prefix + new tokens
 *             (kvSeqLen_b >= seqLen_b).
 * slopes      [headNum] fp32, device: per-head ALiBi coefficient; required for
 *             maskType 3/4/5, must be NULL for 9.
 * maskType    3, 4, 5 or 9 (see enum above).
 * headNum     > 0; kvHeadNum > 0 and divides headNum (query head h reads kv
 *             head h / (headNum/kvHeadNum)).
 * qkScale     multiplies Q K^T before the bias is added.
 * headSize    a multiple of 8 up to 256 (ALiBi masks: <= 128, per the
 *             compressed-mask page's constraints); 64, 128 and 256 run
 *             natively, others on the next of those with zero-filled extra
 *             dimensions.
 * attnOut     same shape and dtype as query, device, 32-byte aligned.
 * ------------------------------------------------------------------------- */
ALA_API int atb_like_prefix_encoder_get_workspace_size(
    const ala_tensor* query, const ala_tensor* key, const ala_tensor* value, const ala_tensor* blockTables,
    const ala_tensor* mask, const ala_tensor* seqLen, const ala_tensor* kvSeqLen, const ala_tensor* slopes,
    int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale, ala_tensor* attnOut,
    uint64_t* workspaceSize, ala_op** op);

ALA_API int atb_like_prefix_encoder(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream);

/* The same operation with the natural-log lse of every (token, head) row also
 * written, so that attention over a prefix split into chunks can be merged
 * with ala_lse_merge (the MLA page's lse output, applied to this encoder).
 * lse: [nTokens, headNum] (or [nTokens, headNum, 1]) fp32, device, required;
 * for left-aligned ALiBi (maskType 5) it is the lse of the left-aligned
 * scores.  Execute with atb_like_prefix_encoder. */
ALA_API int atb_like_prefix_encoder_lse_get_workspace_size(
    const ala_tensor* query, const ala_tensor* key, const ala_tensor* value, const ala_tensor* blockTables,
    const ala_tensor* mask, const ala_tensor* seqLen, const ala_tensor* kvSeqLen, const ala_tensor* slopes,
    int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale, ala_tensor* attnOut, ala_tensor* lse,
    uint64_t* workspaceSize, ala_op** op);

/* ---------------------------------------------------------------------------
 * varlen_attention: the same operation with K/V packed contiguously instead of
 * paged (the contiguous full-prefill reading of the pages' PA_ENCODER mode).
 *
 * query       [nTokens, headNum, headSize] f16/bf16/f32, device.
 * key, value  [nKvTokens, kvHeadNum, headSize], same dtype, device; keys of
 *             sequence b are packed at [sum_{c<b} kvSeqLen_c, + kvSeqLen_b).
 * seqLen, kvSeqLen, slopes, headNum, kvHeadNum, qkScale, headSize as above;
 *             maskType 0, 3, 4, 5 or 9 (0 or 9 when headSize > 128).
 *             f32 inputs run on tf32 tensor cores (headSize a multiple of 8
 *             up to 64).
 * attnOut     like query, 32-byte aligned.
 * lse         NULL or [nTokens, headNum] fp32, device: natural-log
 *             log-sum-exp of each row's scaled, biased, masked scores.
 * ------------------------------------------------------------------------- */
ALA_API int varlen_attention_get_workspace_size(
    const ala_tensor* query, const ala_tensor* key, const ala_tensor* value, const ala_tensor* seqLen,
    const ala_tensor* kvSeqLen, const ala_tensor* slopes, int maskType, int32_t headNum, int32_t kvHeadNum,
    float qkScale, ala_tensor* attnOut, ala_tensor* lse, uint64_t* workspaceSize, ala_op** op);

ALA_API int varlen_attention(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream);

/* ---------------------------------------------------------------------------
 * varlen_attention_noalloc: varlen_attention in one call that allocates
 * nothing, for callers that cannot call cudaMalloc (runtimes that only hand
 * out pre-sized arenas, hosts whose device allocator belongs to another
 * component).  The pages have no counterpart of this call.
 *
 * Arguments as for varlen_attention_get_workspace_size (query 3-D; lse NULL,
 * [nTokens, headNum] or [nTokens, headNum, 1]), plus the stream; no workspace
 * and no op.  The schedule lives in a 1 MiB array in device global memory
 * owned by the library (every GPU that loads the library keeps it until
 * exit): at most 4096 sequences and as many 128-row work units as fit; larger
 * calls return ALA_UNSUPPORTED with the limit in the message.  Every call
 * rewrites that array (its status word is cleared first), so calls whose GPU
 * work overlaps race on it: order them on one stream or with events.  The
 * schedule is uploaded from a library-owned host buffer that the next call
 * rewrites, so a call on a stream that is being captured returns
 * ALA_UNSUPPORTED.  The first call on each device looks up the array's
 * address (cudaGetSymbolAddress, with that device current).  A successful
 * call allocates no device or host memory.
 * ------------------------------------------------------------------------- */
ALA_API int varlen_attention_noalloc(const ala_tensor* query, const ala_tensor* key, const ala_tensor* value,
                                     const ala_tensor* seqLen, const ala_tensor* kvSeqLen, const ala_tensor* slopes,
                                     int maskType, int32_t headNum, int32_t kvHeadNum, float qkScale,
                                     ala_tensor* attnOut, ala_tensor* lse, ala_stream_t stream);

/* Status word of the last varlen_attention_noalloc call on the current device:
 * synchronises `stream`, then reads the word from the library's array (no
 * allocation).  *code = 0 means every kernel wait completed; nonzero names the
 * wait that ran out, and the output of that call is incomplete.  The pages
 * have no counterpart of this call. */
ALA_API int varlen_attention_noalloc_status(ala_stream_t stream, int32_t* code);

/* ---------------------------------------------------------------------------
 * MLA decode / speculative decode (ATB "MLA" page, definition and parameter
 * table).  key_j = [ctKV_j ; kRope_j] (576 dims), value_j = ctKV_j (512).
 *
 * qNope       [tokens, headNum, 512] bf16/f16 (qRope's dtype), device; with
 *             cacheMode 2 also int8 codes (16-byte aligned).
 * qRope       [tokens, headNum, 64] bf16/f16, device: the compute and output type.
 * ctKV        [numBlocks, blockSize, kvHeadNum, 512], device (ND layout), qRope's
 *             dtype, or int8 codes with cacheMode 2 (16-byte aligned);
 *             blockSize a multiple of 16.
 * kRope       [numBlocks, blockSize, kvHeadNum, 64], device.
 * blockTables [batch, maxBlocks] int32, device (entries read must be valid).
 * contextLens [batch] int32, HOST: keys per batch, including the new tokens.
 * mask        NULL (the speculative mask is generated from the rule), or with
 *             maskType SPEC the page's MASK_TYPE_SPEC mask: [tokens,
 *             maxSeqLen] fp16/bf16, device, maxSeqLen >= every contextLens
 *             entry.  Token t (packed over the batch) then considers every key
 *             j < contextLens of its batch, and mask[t][j] is added to the
 *             scaled score (-inf or a large negative value masks the key); the
 *             generated rule is not applied.  A token whose keys are all
 *             masked with -inf gets output 0 and lse -inf.  Must be NULL with
 *             calcType PREFILL.
 * qSeqLen     [batch] int32, HOST: query tokens per batch; required when
 *             calcType = SPEC, else NULL (one token each).  Token t of batch
 *             b allows keys j <= contextLens_b - qSeqLen_b + t.
 * qkDescale, pvDescale  [headNum] fp32, device, required with cacheMode 2
 *             and NULL otherwise.  Reading of the page's two rows: the score
 *             is qkScale * (qkDescale[h] * qNope.ctKV + qRope.kRope) with qNope
 *             and ctKV taken as stored (int8 codes, or floats), and the output
 *             is pvDescale[h] * sum_j p_j ctKV_j.
 * headNum     128 (multiple of 64 accepted); kvHeadNum must be 1.
 * maskType    UNDEFINED (0) with one token per batch, or SPEC (1).
 * calcType    UNDEFINED (0), SPEC (1), RING (2) or PREFILL (3).
 *             RING (ring attention) computes the same attention over the keys
 *             this call is given and requires lse, so that results over
 *             disjoint key ranges can be merged with ala_lse_merge.
 *             PREFILL (full prefill) requires qSeqLen (the new tokens of each
 *             batch, at the end of its context) and applies the causal rule
 *             token t -> keys j <= contextLens - qSeqLen + t whatever maskType
 *             (UNDEFINED or SPEC) says.
 * cacheMode   KROPE_CTKV (1), or INT8_NZCACHE (2): the int8 latent cache,
 *             kept here in the same ND layout as mode 1 (the page's NZ fractal
 *             layout is Ascend's); 0 and 3 return UNSUPPORTED.
 * attenOut    [tokens, headNum, 512], dtype of qRope, device.
 * lse         NULL or [tokens, headNum, 1] fp32, device (natural log);
 *             required with calcType RING (NULL_REQUIRED otherwise).
 * workspace   256-byte aligned; holds the schedule and, for key ranges split
 *             across CTAs, fp32 partial outputs merged by lse at the end.
 * ------------------------------------------------------------------------- */
ALA_API int atb_like_mla_get_workspace_size(
    const ala_tensor* qNope, const ala_tensor* qRope, const ala_tensor* ctKV, const ala_tensor* kRope,
    const ala_tensor* blockTables, const ala_tensor* contextLens, const ala_tensor* mask,
    const ala_tensor* qSeqLen, const ala_tensor* qkDescale, const ala_tensor* pvDescale, int32_t headNum,
    float qkScale, int32_t kvHeadNum, int maskType, int calcType, uint8_t cacheMode, ala_tensor* attenOut,
    ala_tensor* lse, uint64_t* workspaceSize, ala_op** op);

ALA_API int atb_like_mla(void* workspace, uint64_t workspaceSize, ala_op* op, ala_stream_t stream);

/* ---------------------------------------------------------------------------
 * Merge of two partial attention results over disjoint key ranges by their
 * log-sum-exp (ATB "MLA" page, parameter table, rows calcType (ring mode) and
 * lse).  Per output row r:
 *   lse[r] = log(exp(lseA[r]) + exp(lseB[r])),
 *   out[r] = exp(lseA[r] - lse[r]) outA[r] + exp(lseB[r] - lse[r]) outB[r];
 * a row whose lseA and lseB are both -inf gets lse = -inf and out = 0.
 *
 * outA, outB, out  same shape [..., d] (1 to 4 dims, 1 <= d <= 1024), same
 *                  dtype (bf16, f16 or f32), device; rows = product of the
 *                  leading dims.  Each is normalised over its own keys.
 * lseA, lseB, lse  fp32 with one value per row (any shape of `rows`
 *                  elements, e.g. [tokens, headNum, 1]), device, natural log.
 * out / lse may be the same memory as outA / lseA or outB / lseB (in-place
 * accumulation over a ring).  Runs asynchronously on `stream`; allocates
 * nothing.  Returns a status code before any GPU work on invalid arguments.
 * ------------------------------------------------------------------------- */
ALA_API int ala_lse_merge(const ala_tensor* outA, const ala_tensor* lseA, const ala_tensor* outB,
                          const ala_tensor* lseB, ala_tensor* out, ala_tensor* lse, ala_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ALA_H */
