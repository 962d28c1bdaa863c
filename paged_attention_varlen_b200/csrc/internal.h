// internal.h -- structures shared by the host API (api.cpp) and the kernels.
// Not part of the public interface; the public C-ABI is include/ala.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace ala {

// One NVTX range per C-ABI call (named after the entry point), visible in a profiler's timeline; without
// a profiler attached the push and pop cost a function-pointer check.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

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
  kDevBadBlockIndex = 0x10B,  // ALA_DEBUG_BOUNDS builds: a block-table entry read lies outside [0, numBlocks)
};

#ifndef ALA_DEBUG_BOUNDS
#define ALA_DEBUG_BOUNDS 0  // 1: kernels range-check every block-table entry they read (libala_debug.so)
#endif

// Cache row of key position `pos` of a sequence whose block-table row is `bt`: bt[pos / bs] * bs + pos % bs,
// or `oob_row` (one past the cache: the TMA load fills zeros there) for pages at or past `n_pages`.  In an
// ALA_DEBUG_BOUNDS build an entry outside [0, oob_row / bs) records kDevBadBlockIndex in the second status
// word (status[1], which the pipeline's waits do not watch, so the kernel still runs to its end) and reads
// the zero-filled row instead; otherwise such an entry still only ever feeds a bounds-checked TMA load.
__device__ __forceinline__ int paged_row(const int32_t* bt, int pos, int bs, int n_pages, int oob_row, int* status) {
  const int pg = pos / bs;
  if (pg >= n_pages) return oob_row;
  const int32_t blk = bt[pg];
#if ALA_DEBUG_BOUNDS
  if (blk < 0 || (int64_t)blk * bs >= oob_row) {
    atomicCAS(status + 1, 0, kDevBadBlockIndex);
    return oob_row;
  }
#else
  (void)status;
#endif
  return blk * bs + (pos - pg * bs);
}

// Per-sequence metadata, built on the host from seqLen / kvSeqLen.
struct SeqInfo {
  int32_t cu_q;     // first packed query token of the sequence
  int32_t seq_len;  // query rows
  int32_t kv_len;   // keys (prefix + new tokens)
  int32_t cu_kv;    // first packed key row (contiguous layout only)
};

// Keys per K/V tile of the prefill kernel.
constexpr int kPrefillTileKeys = 128;

// One CTA's work: up to two blocks of 128 query rows of one sequence that read
// the same kv head (two query heads of a group, or two consecutive row tiles of
// one head), so every K/V tile the CTA loads serves both.
struct PrefillUnit {
  int32_t b;           // sequence
  int32_t n_blocks;    // 1 or 2
  int32_t q0[2];       // first query row of each block (within the sequence)
  int32_t head[2];     // query head of each block
  int32_t n_tiles[2];  // key tiles each block visits: ceil(min(kv_len, last allowed key + 1) / kPrefillTileKeys);
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
  int32_t d_out;                // head size of the tensors (<= the kernel's D; dims past it are zero-filled)
  int32_t kv_box_rows;          // paged caches: rows per K/V TMA box, gcd(blockSize, keys per tile)
};

// Rows per K/V TMA box for a paged cache: the largest count that divides both the key tile and blockSize,
// so every box lies inside one page (blockSize a multiple of 16 gives at least 16).
inline int kv_box_rows(int block_size, int tile_keys) {
  int a = block_size, b = tile_keys;
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Tiling of the prefill kernel instance that serves kernel head size D (prefill_kernel_d): keys per K/V
// tile and whether a unit holds one block of 128 query rows (D = 256, whose O takes half of tensor memory)
// or up to two.
struct PrefillShape {
  int32_t tile_keys;
  bool one_block;
};
inline PrefillShape prefill_shape(int32_t D) { return D > 128 ? PrefillShape{64, true} : PrefillShape{kPrefillTileKeys, false}; }

// Work units of one prefill request, in sequence order (every prefill entry point uses this list).
// Per sequence b, blocks of 128 query rows; two blocks that read the same kv head form a unit: two
// query heads of a GQA group on the same rows, or, without grouping, two consecutive row tiles of one
// head (one block per unit with shape.one_block).  Each block visits the key tiles up to its last
// allowed key (the causal rule with the prefix offset kvSeqLen - seqLen; every key for mask type 0).
// `emit(const PrefillUnit&)` receives them.
template <class Emit>
inline void prefill_units(int32_t batch, const int32_t* seq_len, const int32_t* kv_len, int mask_type,
                          int32_t heads, int32_t kv_heads, PrefillShape shape, Emit&& emit) {
  const int32_t group = heads / kv_heads;
  const int32_t tk = shape.tile_keys;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t sl = seq_len[b], kl = kv_len[b], off = kl - sl;
    auto tiles_for = [&](int32_t q0) {
      const int32_t last_row = (q0 + 127 < sl - 1) ? q0 + 127 : sl - 1;
      const int32_t causal_end = last_row + off + 1;
      const int32_t kv_end = (mask_type == 0 || kl < causal_end) ? kl : causal_end;
      return (kv_end + tk - 1) / tk;
    };
    if (shape.one_block) {
      for (int32_t h = 0; h < heads; ++h)
        for (int32_t q0 = 0; q0 < sl; q0 += 128) emit(PrefillUnit{b, 1, {q0, q0}, {h, h}, {tiles_for(q0), 0}});
    } else if (group >= 2) {
      for (int32_t q0 = 0; q0 < sl; q0 += 128) {
        const int32_t nt = tiles_for(q0);
        for (int32_t g = 0; g < kv_heads; ++g)
          for (int32_t i = 0; i < group; i += 2) {
            const int32_t h = g * group + i;
            const bool two = i + 1 < group;
            emit(PrefillUnit{b, two ? 2 : 1, {q0, q0}, {h, two ? h + 1 : h}, {nt, two ? nt : 0}});
          }
      }
    } else {
      for (int32_t h = 0; h < heads; ++h)
        for (int32_t q0 = 0; q0 < sl; q0 += 256) {
          const bool two = q0 + 128 < sl;
          emit(PrefillUnit{b, two ? 2 : 1, {q0, q0 + 128}, {h, h}, {tiles_for(q0), two ? tiles_for(q0 + 128) : 0}});
        }
    }
  }
}

// Number of units prefill_units emits (no list is built).
inline int64_t prefill_unit_count(int32_t batch, const int32_t* seq_len, int32_t heads, int32_t kv_heads,
                                  PrefillShape shape) {
  const int32_t group = heads / kv_heads;
  int64_t n = 0;
  for (int32_t b = 0; b < batch; ++b)
    n += shape.one_block ? (int64_t)heads * ((seq_len[b] + 127) / 128)
         : group >= 2    ? (int64_t)((seq_len[b] + 127) / 128) * kv_heads * ((group + 1) / 2)
                         : (int64_t)heads * ((seq_len[b] + 255) / 256);
  return n;
}

// Scheduling cost of a unit: its key tiles plus about one tile of fixed work (Q load, epilogue).
inline int64_t prefill_unit_cost(const PrefillUnit& u) { return (int64_t)u.n_tiles[0] + u.n_tiles[1] + 1; }

// Tensor map over a [rows, heads, d] tensor (d innermost): box of 128 bytes of d, one head and
// `box_rows` rows, 128-byte swizzle (32-byte atoms for a 32-bit MN-major operand).  Defined in api.cpp.
bool encode_rows_heads_d(CUtensorMap* map, void* base, int32_t dtype, int64_t rows, int64_t heads, int64_t d,
                         int box_rows, bool mn_major_operand);

// dtype codes as in include/ala.h
enum : int32_t { kF16 = 0, kBF16 = 1, kF32 = 2, kI32 = 3 };

// Head size D of the prefill kernel instance that serves head size `d` of element type `dtype` (0 if none
// does): 16-bit types take d a multiple of 8 up to 256 (D = 64, 128 or 256), fp32 a multiple of 8 up to
// 64 (D = 64).  The tensor maps are encoded over the real d, so the dimensions d..D-1 of every Q, K and V
// tile are zero-filled by the TMA loads and contribute nothing; the epilogue stores the first d columns.
int prefill_kernel_d(int32_t dtype, int64_t d);
// The D = 256 instance (prefill_d256.cu): one block of 128 rows per unit, 64-key tiles.
cudaError_t launch_prefill_d256(int32_t dtype, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                const PrefillParams& p, cudaStream_t stream);
// Launches the prefill kernel for element type `dtype` and kernel head size `D` (prefill_kernel_d).
cudaError_t launch_prefill(int32_t dtype, int32_t D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const PrefillParams& p, cudaStream_t stream);

// Merges two partial results (rows x d, each normalised over its own keys) by their lse; out / lse may
// alias the inputs.  d <= 1024.
cudaError_t launch_lse_merge(int32_t dtype, const void* a, const float* lse_a, const void* b, const float* lse_b,
                             void* out, float* lse, int64_t rows, int d, cudaStream_t stream);

}  // namespace ala
