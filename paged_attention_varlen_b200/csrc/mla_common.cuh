// mla_common.cuh -- the MLA schedule's work records, the kernel parameters and small device helpers
// (mla.cu).  Internal to the library.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace ala {
namespace mlak {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only when the max grows by > 2^8

constexpr int kTileKeys = 64;              // keys per staged cache tile
constexpr int kDNope = 512;                // latent (ctKV) dimensions; the rope part adds 64
constexpr int kPlannedSms = 148;           // SMs of the part the schedule is cut for
constexpr int kMinLaneTiles = 4;           // shortest key range worth a lane of its own
constexpr unsigned kFull = 0xffffffffu;

struct MlaPiece {
  int32_t b;         // batch
  int32_t token0;    // first packed query token of the chunk
  int32_t kv_begin;  // first key of the range (a multiple of 32)
  int32_t n_tiles;   // 32-key tiles in the range
  int32_t last;      // last allowed key of the chunk's first token; token t of the chunk allows last + row_step*t
  int32_t part;      // partial slot (rows part*tpc .. +tpc-1 of the partials), or -1: final output
  int32_t n_keys;    // keys of the batch the chunk may read (its pages): last + tpc, or contextLens with a mask
  int32_t row_step;  // 1: the speculative rule; 0: every token reads keys 0..n_keys-1 (explicit mask tensor)
};

struct MlaCombine {
  int32_t token;       // packed query token
  int32_t part_begin;  // its chunk's first partial slot
  int32_t n_parts;
  int32_t t_local;     // token index within the chunk
};

struct MlaParams {
  const MlaPiece* pieces;
  const int32_t* lane_off;  // [n_lanes + 1]: lane l walks pieces [lane_off[l], lane_off[l+1])
  const int32_t* block_tables;
  const uint8_t* q_nope;    // [tokens, heads, 512] (rows go to tensor memory through registers)
  const uint8_t* ct_kv;     // [numBlocks * blockSize, 512] (the L2 prefetch reads raw rows)
  const uint8_t* k_rope;    // [numBlocks * blockSize, 64]
  void* out;                // [tokens, heads, 512] (written by TMA stores and by the combine)
  float* lse;               // [tokens, heads] or null
  float* part_o;            // [parts * tpc, heads, 512]
  float* part_lse;          // [parts * tpc, heads]
  int* status;
  int32_t heads;
  int32_t groups;           // heads / hpc
  int32_t tpc;              // query tokens per CTA row block
  int32_t hpc;              // heads per CTA row block (64 / tpc)
  int32_t max_blocks;
  int32_t block_size;
  int32_t kv_box_rows;      // rows per cache TMA box when a tile spans pages: gcd(blockSize, kTileKeys)
  int32_t oob_row;
  float scale_log2;
  const float* qk_descale;  // [heads], int8 cache only
  const float* pv_descale;  // [heads], int8 cache only
  int32_t qn_int8;          // qNope holds int8 codes (int8 cache only)
  const uint16_t* mask;     // [tokens, mask_cols] additive mask (fp16 or bf16 bits), or null: the rule
  int64_t mask_cols;
  int32_t mask_f16;         // the mask holds fp16 (else bf16)
  int32_t mask_vec;         // rows start 16-byte aligned: 16-byte loads
};

// One fp16 or bf16 mask element (its 16 bits) as a float.
__device__ __forceinline__ float mask_value(uint32_t bits, bool f16) {
  return f16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(bits))) : __uint_as_float(bits << 16);
}

// The additive mask of packed token `token` for keys j0 .. j0+63, in log2 units (times log2 e); keys at or
// past the mask's row length read 0 (they lie past contextLens and are masked by the key limit).
__device__ __forceinline__ void load_mask_log2(const MlaParams& p, int token, int j0, float (&mk)[64]) {
  const uint16_t* row = p.mask + (size_t)token * p.mask_cols;
  const bool f16 = p.mask_f16 != 0;
  if (p.mask_vec && j0 + 64 <= p.mask_cols) {
    const uint4* src = reinterpret_cast<const uint4*>(row + j0);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint4 w = __ldg(src + v);
      const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mk[8 * v + 2 * i] = mask_value(q[i] & 0xffffu, f16) * kLog2e;
        mk[8 * v + 2 * i + 1] = mask_value(q[i] >> 16, f16) * kLog2e;
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 64; ++c) mk[c] = (j0 + c < p.mask_cols) ? mask_value(__ldg(row + j0 + c), f16) * kLog2e : 0.f;
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Warp-uniform wait on all lanes (each lane observes the phase itself).
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, int* status, int code) {
  return __all_sync(kFull, mbar_wait(bar, parity, status, code));
}

}  // namespace mlak
}  // namespace ala
