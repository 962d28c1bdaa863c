// internal.h -- structures shared by the host API (api.cpp) and the kernels.
// Not part of the public interface; the public C-ABI is include/ala.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ala {

// Device status codes written by bounded waits (0 = no error).
enum DeviceStatus : int {
  kDevOk = 0,
  kDevTimeoutQ = 0x101,
  kDevTimeoutKFull = 0x102,
  kDevTimeoutVFull = 0x103,
  kDevTimeoutKEmpty = 0x104,
  kDevTimeoutVEmpty = 0x105,
  kDevTimeoutSFull = 0x106,
  kDevTimeoutSFree = 0x107,
  kDevTimeoutPFull = 0x108,
  kDevTimeoutODone = 0x109,
  kDevTimeoutFinal = 0x10A,
};

// Per-sequence metadata, built on the host from seqLen / kvSeqLen.
struct SeqInfo {
  int32_t cu_q;     // first packed query token of the sequence
  int32_t seq_len;  // query rows
  int32_t kv_len;   // keys (prefix + new tokens)
  int32_t cu_kv;    // first packed key row (contiguous layout only)
};

// One CTA's work: up to two blocks of 128 query rows of one sequence that read
// the same kv head (two query heads of a group, or two consecutive row tiles of
// one head), so every K/V tile the CTA loads serves both.
struct PrefillUnit {
  int32_t b;           // sequence
  int32_t n_blocks;    // 1 or 2
  int32_t q0[2];       // first query row of each block (within the sequence)
  int32_t head[2];     // query head of each block
  int32_t n_tiles[2];  // 128-key tiles each block visits: ceil(min(kv_len, last allowed key + 1) / 128);
                       // n_tiles[1] >= n_tiles[0] when n_blocks == 2
};

struct PrefillParams {
  const PrefillUnit* units;
  const int32_t* cta_offsets;   // [n_ctas + 1]: CTA c runs units [off[c], off[c+1]); null: CTA c runs unit c
  const SeqInfo* seqs;
  const int32_t* block_tables;  // device [batch, max_blocks] or null (contiguous)
  const float* slopes;          // device [heads] or null
  void* out;                    // [nTokens, heads, D]
  float* lse;                   // [nTokens, heads] or null
  int* status;                  // device status word
  int32_t n_units;
  int32_t n_ctas;               // grid size
  int32_t max_blocks;
  int32_t block_size;
  int32_t oob_row;              // a key row index past the cache (TMA fills zeros there)
  int32_t mask_type;
  int32_t heads;
  int32_t group;                // heads / kvHeads
  float scale_log2;             // qkScale * log2(e)
};

// dtype codes as in include/ala.h
enum : int32_t { kF16 = 0, kBF16 = 1, kF32 = 2, kI32 = 3 };

// Launches the prefill kernel for element type `dtype` and head size `d`.
cudaError_t launch_prefill(int32_t dtype, int32_t d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const PrefillParams& p, cudaStream_t stream);
// Dynamic shared memory the prefill kernel needs (0 if the combination is unsupported).
int prefill_smem_bytes(int32_t dtype, int32_t d);

// Merges two partial results (rows x d, each normalised over its own keys) by their lse; out / lse may
// alias the inputs.  d <= 1024.
cudaError_t launch_lse_merge(int32_t dtype, const void* a, const float* lse_a, const void* b, const float* lse_b,
                             void* out, float* lse, int64_t rows, int d, cudaStream_t stream);

}  // namespace ala
