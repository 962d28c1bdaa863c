// mla.cu -- MLA decode / speculative decode over a paged latent cache for
// sm_100a (ATB "MLA" page, definition and parameter table): per query token
// and head, O = softmax(qkScale * [qNope;qRope] . [ctKV;kRope]^T) ctKV, with
// the speculative causal rule (token t of a batch with qseqlen tokens allows
// keys j <= contextLens - qseqlen + t), plus the natural-log lse.
//
// Rows.  Every MMA has M = 64 rows: tpc consecutive query tokens of one batch
// times 64/tpc heads (tpc = 4, 2 or 1: the largest that divides every batch's
// qseqlen), so the speculative tokens of a batch share each cache tile the CTA
// stages.  The heads / (64/tpc) "groups" of a batch read the same cache tiles;
// L2 serves them once from HBM.
//
// Persistent schedule.  The key tiles of all chunks (a chunk = the tpc tokens
// one CTA row block covers), laid end to end, are cut into equal contiguous
// ranges, one per "lane"; the grid is lanes x groups CTAs (at most one per SM),
// and a CTA walks the pieces of its lane in order.  A chunk cut by a lane
// boundary leaves an fp32 partial (O, lse) per piece, which mla_combine_kernel
// merges by lse (the merge the MLA page's ring mode returns the lse for).
//
// Memory.  qNope (64 rows x 512) sits in tensor memory as the A operand of the
// QK MMAs, so shared memory holds only qRope and a three-deep ring of 64-key
// tiles (ctKV 64 KB + kRope 8 KB each).  Once S(j) is computed, the softmax
// writes P(j) over tile j's kRope block; the PV of the tile reads P and V from
// the same slot.  Tensor memory: lanes 0..15 of each 32-lane quarter hold qNope
// (columns 0..255) and two S buffers (256..319, 384..447); lanes 16..31 hold O
// (columns 0..511).
//
//   warp 4      TMA producer (one thread): ctKV + kRope tiles gathered through
//               the block table (one 3-D box per tile when a tile lies in one
//               page), running ahead across piece boundaries and asking L2 for
//               the tiles after.
//   warp 5      tcgen05 issuer (one thread): S = qNope K^T (TS, A in tensor
//               memory) + qRope kRope^T (SS), and O += P V with V the ctKV part
//               of the tile (two N = 256 halves); it issues the next PV when
//               its P is ready, else the next QK when its tile and S buffer
//               are (QK may lead PV by two tiles).
//   warps 0..3  softmax: lane l < 16 of warp w owns S row 16w + l (scale, mask,
//               online max / sum, P); lane 16 + l owns the O row and rescales
//               it when the max grew by more than 2^8.  At the end of a piece
//               the O rows are normalised into the last tile's slot and one
//               thread writes them out with TMA stores; then the 128 threads
//               load the next chunk's query into tensor memory.
//
// int8 latent cache (the MLA page's INT8 cache mode with its qkDescale and
// pvDescale rows, kept in the ND layout here).  The producer stages each tile's
// int8 ctKV codes (32 KB) in the upper half of the slot's ctKV area, three
// tiles ahead as above; four more warps (6..9) read them, wait until all 128
// have (their T output overwrites that half), and write the tile as T (every
// int8 code is a T value) in the swizzled layout the MMAs read, so the QK and
// PV MMAs are the same T MMAs as above on half the cache bytes.  The
// qRope kRope part goes to its own accumulator (columns 320..383) so that the
// softmax forms qkDescale[h] * qNope.ctKV + qRope.kRope; pvDescale[h] joins the
// 1 / l of the epilogue.  An int8 qNope is converted on its way into tensor memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <type_traits>

#include "internal.h"
#include "mla.h"
#include "mla_common.cuh"
#include "ptx.cuh"

namespace ala {

namespace {

using namespace mlak;

#ifndef ALA_MLA_PREFETCH_TILES
#define ALA_MLA_PREFETCH_TILES 2  // the producer asks L2 for the tiles this far ahead of its loads
#endif

constexpr int kRows = 64;                  // attention rows per CTA: the M of every MMA
constexpr int kBlk = kRows * 128;          // one 64-column block of 64 rows (query rows or keys): 8 KB
constexpr int kQrBytes = kBlk;             // the 64 x 64 qRope rows (qNope lives in tensor memory)
constexpr int kKvBytes = 9 * kBlk;         // 64 keys x 576 x 2 B: ctKV blocks 0..7, kRope block 8
constexpr int kPOff = 8 * kBlk;            // P(j) overwrites tile j's kRope block once S(j) is computed
constexpr int kStages = 3;
// q_full, kv_full[3], kv_empty[3], p_full[3], pv_last, s_full(0), s_free(0), fin, st_full, st_free, cv_full[3],
// cv_read, s_full(1), s_free(1)
constexpr int kNBars = 1 + 3 * kStages + 6 + kStages + 1 + 2;
constexpr int kI8Off = 4 * kBlk;           // int8 cache: the tile's codes ([4][64 keys][128 B], 128B swizzle)
constexpr int kSmem = 1024 + kQrBytes + kStages * kKvBytes + kNBars * 8 + 16;
static_assert(kSmem <= 232448, "shared memory budget");
static_assert(8 * kBlk <= kKvBytes, "the output staging (eight 8 KB boxes) must fit in a ring slot");
// tensor memory: lanes 0..15 of each 32-lane quarter hold qNope (columns 0..255, the A operand of the
// QK MMAs, which must accumulate at lane offset 0) and two S buffers (columns 256..319 and 384..447, so
// that QK(j+1) runs while the softmax works on S(j)); lanes 16..31 hold O (columns 0..511: output
// columns 0..255 and 256..511 as two N = 256 accumulators)
constexpr uint32_t kQnCol = 0;
constexpr uint32_t kSCol = 256;
constexpr uint32_t kSRCol = 320;           // int8 cache: the qRope kRope part of S, lanes 0..15
constexpr uint32_t kSBuf = 128;            // column offset of the second S buffer (and its qRope kRope part)
constexpr int kConvWarp0 = 6;              // int8 cache: warps 6..9 convert ctKV tiles
constexpr uint32_t kOLane = 16;
constexpr uint32_t kTmemCols = 512;


// Four int8 codes (one 32-bit word, the first code in the low byte) to four T values, exactly,
// as two words of packed pairs.  The code v is biased to v + 128 in [0, 255] and placed in the low
// mantissa bits of a float whose unit in the last place is 1 (2^23 in binary32, 2^10 in binary16);
// subtracting that base plus 128 leaves v.  A binary32 integer of magnitude <= 128 has zeros in its
// low 16 bits, so its upper half is the exact bf16.
__device__ __forceinline__ void i8x4_to_pairs(uint32_t w, uint32_t& lo, uint32_t& hi, __nv_bfloat16*) {
  const uint32_t u = w ^ 0x80808080u;
  const uint64_t bias = f2pack(-8388736.f, -8388736.f);  // -(2^23 + 128)
  const uint64_t a = add_x2(f2pack(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                                   __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))), bias);
  const uint64_t b = add_x2(f2pack(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                                   __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))), bias);
  lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(a >> 32), 0x7632);
  hi = __byte_perm(static_cast<uint32_t>(b), static_cast<uint32_t>(b >> 32), 0x7632);
}
__device__ __forceinline__ void i8x4_to_pairs(uint32_t w, uint32_t& lo, uint32_t& hi, __half*) {
  const uint32_t u = w ^ 0x80808080u;
  uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);  // binary16 1024 + (v + 128) for codes 0 and 1
  uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);  // ... and for codes 2 and 3
  const __half2 bias = __half2half2(__ushort_as_half(static_cast<unsigned short>(0x6480u)));  // 1152
  const __half2 ha = __hsub2(*reinterpret_cast<const __half2*>(&a), bias);
  const __half2 hb = __hsub2(*reinterpret_cast<const __half2*>(&b), bias);
  lo = *reinterpret_cast<const uint32_t*>(&ha);
  hi = *reinterpret_cast<const uint32_t*>(&hb);
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

// Loads one chunk's query into place: qNope rows into tensor memory (lanes 0..15 of the warp's
// quarter, by the 128 softmax threads: row 16w + l is token t, head h of the chunk) and the qRope
// rows into shared memory by TMA (thread 0).  Every thread arrives on q_full once.
// Tensor-memory stores are warp-wide: lanes 16..31 write zeros into their columns 0..255, which
// hold O, so this runs only while O is free (before the piece's first PV, after the last epilogue).
// An int8 qNope (int8 cache only) is converted to T exactly on the way.
template <typename T>
__device__ __forceinline__ void load_query(const MlaParams& p, const CUtensorMap* tmQr, uint8_t* sQr,
                                           uint64_t* q_full, uint32_t tmem_warp, int h0, int token0, int t_local,
                                           int head, bool upper) {
  if (threadIdx.x == 0) {
    mbar_expect_tx_only(q_full, kQrBytes);  // thread 0 arrives below, with the others
    tma_load_3d(sQr, tmQr, q_full, 0, h0, token0);
  }
  const size_t row = (size_t)(token0 + t_local) * p.heads + head;
  if (p.qn_int8) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + row * kDNope);
#pragma unroll
    for (int c32 = 0; c32 < 8; ++c32) {  // 32 columns = 64 elements = 64 B of int8 codes per store
      uint32_t r[32];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 w = upper ? make_uint4(0u, 0u, 0u, 0u) : __ldg(src + c32 * 4 + v);
        i8x4_to_pairs(w.x, r[8 * v + 0], r[8 * v + 1], (T*)nullptr);
        i8x4_to_pairs(w.y, r[8 * v + 2], r[8 * v + 3], (T*)nullptr);
        i8x4_to_pairs(w.z, r[8 * v + 4], r[8 * v + 5], (T*)nullptr);
        i8x4_to_pairs(w.w, r[8 * v + 6], r[8 * v + 7], (T*)nullptr);
      }
      tmem_st32(tmem_warp + kQnCol + c32 * 32, r);
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + row * kDNope * 2);
#pragma unroll
    for (int c32 = 0; c32 < 8; ++c32) {  // 32 columns = 64 elements = 128 B of the row per store
      uint32_t r[32];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const uint4 w = upper ? make_uint4(0u, 0u, 0u, 0u) : __ldg(src + c32 * 8 + v);
        r[4 * v + 0] = w.x;
        r[4 * v + 1] = w.y;
        r[4 * v + 2] = w.z;
        r[4 * v + 3] = w.w;
      }
      tmem_st32(tmem_warp + kQnCol + c32 * 32, r);
    }
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(q_full);
}

// KV8: int8 latent cache (warps 6..9 convert the ctKV tiles)
template <typename T, bool KV8>
__global__ void __launch_bounds__(KV8 ? 320 : 192, 1)
    mla_kernel(const __grid_constant__ CUtensorMap tmQr, const __grid_constant__ CUtensorMap tmKV,
               const __grid_constant__ CUtensorMap tmKV3, const __grid_constant__ CUtensorMap tmKR,
               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmPO, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQr = smem;  // the chunk's qRope rows
  uint8_t* sKV = sQr + kQrBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kStages * kKvBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;               // [kStages] tile loaded
  uint64_t* kv_empty = bars + 1 + kStages;    // [kStages] slot free again
  uint64_t* p_full = bars + 1 + 2 * kStages;  // [kStages] P of the slot's tile written
  uint64_t* pv_last = bars + 1 + 3 * kStages; // the last PV of a piece is complete
  // S buffer b (tile G uses b = G % 2): computed / read by all 128 softmax threads
  uint64_t* const s_full0 = pv_last + 1;
  uint64_t* const s_full1 = pv_last + 7 + kStages;
  uint64_t* const s_free0 = pv_last + 2;
  uint64_t* const s_free1 = pv_last + 8 + kStages;
  auto s_full = [=](int b) { return b ? s_full1 : s_full0; };
  auto s_free = [=](int b) { return b ? s_free1 : s_free0; };
  uint64_t* fin = pv_last + 3;
  uint64_t* st_full = pv_last + 4;  // the 128 softmax threads have written a round of output boxes
  uint64_t* st_free = pv_last + 5;  // the stores of a round have read their boxes
  uint64_t* cv_full = pv_last + 6;  // [kStages] int8 cache: the converters have written the slot's ctKV
  uint64_t* cv_read = pv_last + 6 + kStages;  // int8 cache: the 128 converters have read a tile's codes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNBars);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ln = blockIdx.x / p.groups;
  const int h0 = (blockIdx.x - ln * p.groups) * p.hpc;  // first head of this CTA's group
  const int k0 = p.lane_off[ln];
  const int k1 = p.lane_off[ln + 1];
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
      mbar_init(p_full + s, 128);
    }
    mbar_init(pv_last, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 128);
    }
    mbar_init(fin, 1);
    mbar_init(st_full, 128);
    mbar_init(st_free, 1);
    if (KV8) {
      for (int s = 0; s < kStages; ++s) mbar_init(cv_full + s, 128);
      mbar_init(cv_read, 128);
    }
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the combine grid (launched as a programmatic dependent) may be scheduled from now on; it waits for this
  // grid's completion before it reads the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 4) {
    // ------------------------------------------------------------ producer (one elected thread)
    if (elect_one()) {
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmKV3);
      tma_prefetch_desc(&tmKR);
      const int bs = p.block_size;
      const bool whole = bs % kTileKeys == 0;  // a tile lies in one page: one 3-D box holds its ctKV part
      const int box_rows = p.kv_box_rows;  // every box lies inside one page
      int G = 0;  // tiles issued so far by this CTA
      // L2 prefetch cursor (piece kf, tile jf, CTA tile Gf), kept ALA_MLA_PREFETCH_TILES tiles ahead of the loads
      int kf = k0, jf = 0, Gf = 0;
      MlaPiece pf = k0 < k1 ? p.pieces[k0] : MlaPiece{};
      bool ok = true;
      for (int k = k0; k < k1 && ok; ++k) {
        const MlaPiece pc = p.pieces[k];
        const int32_t* bt = p.block_tables + (size_t)pc.b * p.max_blocks;
        const int n_pages = (pc.n_keys + bs - 1) / bs;  // pages holding the keys the chunk may read
        if (k + 1 < k1) {  // the next chunk's qNope rows, for the softmax threads' loads at the piece boundary
          const MlaPiece pn = p.pieces[k + 1];
          const int qes = p.qn_int8 ? 1 : 2;
          for (int t = 0; t < p.tpc; ++t)
            bulk_prefetch_l2(p.q_nope + (((size_t)(pn.token0 + t) * p.heads + h0) * kDNope) * qes, p.hpc * kDNope * qes);
        }
        for (int j = 0; j < pc.n_tiles; ++j) {
          for (; ALA_MLA_PREFETCH_TILES > 0 && kf < k1 && Gf <= G + ALA_MLA_PREFETCH_TILES; ++Gf) {
            const int32_t* btf = p.block_tables + (size_t)pf.b * p.max_blocks;
            const int npf = (pf.n_keys + bs - 1) / bs;
            for (int r0 = 0; r0 < kTileKeys; r0 += box_rows) {
              const int pos = pf.kv_begin + jf * kTileKeys + r0;
              const int row = paged_row(btf, pos, bs, npf, p.oob_row, p.status);
              if (row >= 0 && row < p.oob_row) {  // a block index outside the cache is never touched
                constexpr int kRowBytes = KV8 ? kDNope : 2 * kDNope;
                bulk_prefetch_l2(p.ct_kv + (size_t)row * kRowBytes, box_rows * kRowBytes);
                bulk_prefetch_l2(p.k_rope + (size_t)row * 128, box_rows * 128);
              }
            }
            if (++jf == pf.n_tiles) {
              jf = 0;
              if (++kf < k1) pf = p.pieces[kf];
            }
          }
          const int s = G % kStages;
          if (G >= kStages && !mbar_wait(kv_empty + s, ((G / kStages) - 1) & 1, status, kDevTimeoutKEmpty)) {
            ok = false;
            break;
          }
          uint8_t* dst = sKV + s * kKvBytes;
          mbar_expect_tx(kv_full + s, KV8 ? 5 * kBlk : kKvBytes);  // int8 cache: 32 KB of codes + kRope
          const int j0 = pc.kv_begin + j * kTileKeys;
          for (int r0 = 0; r0 < kTileKeys; r0 += box_rows) {
            const int pos = j0 + r0;
            const int row = paged_row(bt, pos, bs, n_pages, p.oob_row, p.status);  // past the last page: zeros
            if (KV8) {  // the codes, [4 blocks of 128 columns][key][128 B], into the upper half of the ctKV area
              if (whole) {
                tma_load_3d(dst + kI8Off, &tmKV3, kv_full + s, 0, row, 0);
              } else {
                for (int cb = 0; cb < 4; ++cb)
                  tma_load_2d(dst + kI8Off + cb * kBlk + r0 * 128, &tmKV, kv_full + s, cb * 128, row);
              }
            } else if (whole) {
              tma_load_3d(dst, &tmKV3, kv_full + s, 0, row, 0);  // [column block][key][64 elements]
            } else {
              for (int cb = 0; cb < 8; ++cb) tma_load_2d(dst + cb * kBlk + r0 * 128, &tmKV, kv_full + s, cb * 64, row);
            }
            tma_load_2d(dst + 8 * kBlk + r0 * 128, &tmKR, kv_full + s, 0, row);
          }
          ++G;
        }
      }
      // no copy may be in flight when the CTA exits
      for (int t = G - kStages < 0 ? 0 : G - kStages; t < G; ++t)
        mbar_wait(kv_full + (t % kStages), (t / kStages) & 1, status, kDevTimeoutKFull);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (one elected thread)
    if (elect_one()) {
      constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
      constexpr uint32_t idesc_qk = instr_desc(fmt, false, false, kRows, kTileKeys);
      constexpr uint32_t idesc_pv = instr_desc(fmt, false, true, kRows, 256);
      // base descriptors; a step adds its byte offset >> 4 to the start-address field
      const uint64_t dqr = smem_desc_sw128(smem_addr(sQr), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv = smem_desc(smem_addr(sKV), kBlk, 1024, 2);          // ctKV as the MN-major V operand
      const uint64_t dp = smem_desc_sw128(smem_addr(sKV + kPOff), 16, 1024);  // P in the slot's kRope block
      int total = 0;
      for (int k = k0; k < k1; ++k) total += p.pieces[k].n_tiles;
      // QK cursor: piece kq, tile jq of nq, tile Gq of the CTA; PV cursor likewise
      int kq = k0, jq = 0, nq = k0 < k1 ? p.pieces[k0].n_tiles : 0, Gq = 0;
      int kp = k0, jp = 0, np = nq, Gp = 0;
      bool ok = true;
      uint64_t t_prog = global_timer_ns();  // when the idle loop last saw progress
      uint32_t it = 0;
      bool progressed = false;
      while (ok && Gp < total) {
        // PV(Gp) needs P(Gp) and goes first when ready: it frees its ring slot for the producer.
        // QK(Gq) needs its tile, its S buffer (softmax is done with S(Gq-2)) and, first in a piece, the
        // query; it may lead PV by two tiles (two S buffers, three ring slots).
        const int sq = Gq % kStages;
        if (Gp < Gq && mbar_test_wait(p_full + (Gp % kStages), (Gp / kStages) & 1)) {
          tc_fence_after();
          const uint64_t so = (uint64_t)(((Gp % kStages) * kKvBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTileKeys / 16; ++kk) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // V = ctKV columns [256h, 256h+256): four 64-wide column blocks, MN-major; O at lane 16
              mma_ss(tmem + (kOLane << 16) + 256 * h, dp + so + ((kk * 32) >> 4),
                     dv + so + ((4 * h * kBlk + kk * 16 * 128) >> 4), idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u, false);
            }
          }
          // the last tile of a piece: its slot is the epilogue's staging area and is freed by the epilogue
          mma_commit(jp + 1 == np ? pv_last : kv_empty + (Gp % kStages));
          ++Gp;
          if (++jp == np) {
            ++kp;
            jp = 0;
            np = kp < k1 ? p.pieces[kp].n_tiles : 0;
          }
          progressed = true;
        } else if (Gq < total && Gq - Gp < 3 && mbar_test_wait(kv_full + sq, (Gq / kStages) & 1) &&
            (!KV8 || mbar_test_wait(cv_full + sq, (Gq / kStages) & 1)) &&
            (Gq < 2 || mbar_test_wait(s_free(Gq & 1), ((Gq - 2) >> 1) & 1)) &&
            (jq > 0 || mbar_test_wait(q_full, (kq - k0) & 1))) {
          const uint32_t sb = (Gq & 1) * kSBuf;
          tc_fence_after();
          const uint64_t so = (uint64_t)((sq * kKvBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kDNope / 16; ++kk)  // qNope from tensor memory (8 columns per 16 elements)
            mma_ts(tmem + kSCol + sb, tmem + kQnCol + kk * 8,
                   dk + so + (uint64_t)(((kk >> 2) * kBlk + (kk & 3) * 32) >> 4), idesc_qk, kk > 0 ? 1u : 0u, false);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // qRope x kRope from shared memory (own accumulator with an int8 cache)
            mma_ss(tmem + (KV8 ? kSRCol : kSCol) + sb, dqr + (uint64_t)((kk * 32) >> 4),
                   dk + so + (uint64_t)((8 * kBlk + kk * 32) >> 4), idesc_qk, (!KV8 || kk > 0) ? 1u : 0u, false);
          mma_commit(s_full(Gq & 1));
          ++Gq;
          if (++jq == nq) {
            ++kq;
            jq = 0;
            nq = kq < k1 ? p.pieces[kq].n_tiles : 0;
          }
          progressed = true;
        } else if ((++it & 1023u) == 0) {
          const uint64_t now = global_timer_ns();
          if (progressed) {
            t_prog = now;
            progressed = false;
          }
          if (*(volatile int*)status != 0) ok = false;
          else if (now - t_prog > ALA_WAIT_LIMIT_NS) {
            atomicCAS(status, 0, Gq - Gp < 2 && Gq < total ? kDevTimeoutKFull : kDevTimeoutPFull);
            ok = false;
          }
        }
      }
      mma_commit(fin);
      mbar_wait(fin, 0, status, kDevTimeoutFinal);
    }
  } else if (KV8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ int8 ctKV -> T (warps 6..9)
    // Thread ct handles keys kk0 + 8m (m = 0..7) of every tile and, of each, the 16-byte chunks of
    // codes c0 and c0 + 16 (columns 16c .. 16c+15).  Both its shared-memory reads (the codes, 128B
    // swizzle) and its writes hit each 16-byte bank group four times per warp (no conflicts).
    const int ct = threadIdx.x - kConvWarp0 * 32;
    const int kk0 = ct & 7;
    const int c0 = ct >> 3;
    int G = 0;
    bool ok = true;
    for (int k = k0; k < k1 && ok; ++k) {
      const int n_tiles = p.pieces[k].n_tiles;
      for (int j = 0; j < n_tiles; ++j, ++G) {
        const int s = G % kStages;
        if (!wait_all(kv_full + s, (G / kStages) & 1, status, kDevTimeoutKFull)) {
          ok = false;
          break;
        }
        const uint32_t slot = smem_addr(sKV + s * kKvBytes);
        uint4 v[8][2];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = c0 + 16 * h;  // 128-column block c >> 3, its 16-byte chunk c & 7
            v[m][h] = ld_shared_v4(slot + kI8Off + (c >> 3) * kBlk + (kk0 + 8 * m) * 128 + (((c & 7) ^ kk0) << 4));
          }
        }
        // the T tile overwrites the codes: every converter must have read its share first
        mbar_arrive(cv_read);
        if (!wait_all(cv_read, G & 1, status, kDevTimeoutKFull)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t key_row = slot + (kk0 + 8 * m) * 128;  // 128B swizzle of key row r: chunk q at q ^ (r & 7)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = c0 + 16 * h;
            const uint4 w = v[m][h];
            uint32_t o[8];
            i8x4_to_pairs(w.x, o[0], o[1], (T*)nullptr);
            i8x4_to_pairs(w.y, o[2], o[3], (T*)nullptr);
            i8x4_to_pairs(w.z, o[4], o[5], (T*)nullptr);
            i8x4_to_pairs(w.w, o[6], o[7], (T*)nullptr);
            const uint32_t blk = key_row + (c >> 2) * kBlk;  // 64-column block of columns 16c .. 16c+15
            const int q = 2 * (c & 3);                        // their two 16-byte chunks in the block's row
            st_shared_v4(blk + ((q ^ kk0) << 4), make_uint4(o[0], o[1], o[2], o[3]));
            st_shared_v4(blk + (((q + 1) ^ kk0) << 4), make_uint4(o[4], o[5], o[6], o[7]));
          }
        }
        fence_proxy_async_smem();  // visible to the tensor cores
        mbar_arrive(cv_full + s);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // lanes 0..15 of warp w own S row 16w + l; lanes 16..31 own O row 16w + (l - 16)
    const bool upper = lane >= 16;
    const int hr = (warp * 16) + (lane & 15); // row within the CTA: token t_local, head h0 + hl
    const int t_local = hr / p.hpc;
    const int head = h0 + (hr - t_local * p.hpc);
    const uint32_t tmem_warp = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int sw = hr & 7;  // 128-byte swizzle of the row's 16-byte chunks
    const float scale = p.scale_log2;
    const bool has_mask = p.mask != nullptr;
    const bool raw_max = scale > 0.f && !has_mask;  // max of the raw scores, scale folded into the exponent
    const float qk_d = KV8 ? p.qk_descale[head] : 1.f;
    const float pv_d = KV8 ? p.pv_descale[head] : 1.f;
    bool ok = true;
    int G = 0;  // tiles consumed
    int R = 0;  // output staging rounds
    if (k0 < k1) load_query<T>(p, &tmQr, sQr, q_full, tmem_warp, h0, p.pieces[k0].token0, t_local, head, upper);
    for (int k = k0; k < k1 && ok; ++k) {
      const MlaPiece pc = p.pieces[k];
      const int row_last = min(pc.last + pc.row_step * t_local, pc.n_keys - 1);
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; j < pc.n_tiles; ++j, ++G) {
        ok = wait_all(s_full(G & 1), (G >> 1) & 1, status, kDevTimeoutSFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sb = (G & 1) * kSBuf;
        float x[kTileKeys];
        {
          uint32_t regs[2][32];
          tmem_ld32(tmem_warp + kSCol + sb, regs[0]);
          tmem_ld32(tmem_warp + kSCol + sb + 32, regs[1]);
          if constexpr (KV8) {
            // score = qkDescale * (qNope . ctKV) + qRope . kRope
            uint32_t rr[2][32];
            tmem_ld32(tmem_warp + kSRCol + sb, rr[0]);
            tmem_ld32(tmem_warp + kSRCol + sb + 32, rr[1]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < kTileKeys; ++c)
              x[c] = fmaf(qk_d, __uint_as_float(regs[c >> 5][c & 31]), __uint_as_float(rr[c >> 5][c & 31]));
          } else {
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < kTileKeys; ++c) x[c] = __uint_as_float(regs[c >> 5][c & 31]);
          }
        }
        const int lim = row_last - (pc.kv_begin + j * kTileKeys);  // columns c <= lim are allowed
        if (has_mask) {
          // the explicit mask is added after the scale (log2 units); lanes 16..31 hold no score row
          float mk[kTileKeys];
          if (!upper) {
            load_mask_log2(p, pc.token0 + t_local, pc.kv_begin + j * kTileKeys, mk);
          } else {
#pragma unroll
            for (int c = 0; c < kTileKeys; ++c) mk[c] = 0.f;
          }
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] = fmaf(x[c], scale, mk[c]);
        } else if (!raw_max) {
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] *= scale;
        }
        if (__any_sync(kFull, lim < kTileKeys - 1)) {  // only a range's last tiles can hold masked keys
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTileKeys; c += 8) {
          mx0 = max3(mx0, x[c], x[c + 1]);
          mx1 = max3(mx1, x[c + 2], x[c + 3]);
          mx2 = max3(mx2, x[c + 4], x[c + 5]);
          mx3 = max3(mx3, x[c + 6], x[c + 7]);
        }
        float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        if (raw_max) mx *= scale;
        const float m_new = fmaxf(m_run, mx);
        float alpha = 1.f;
        if (m_new - m_run > kRescaleThreshold) {  // false while both are -inf
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        // lanes 16..31 scale the O rows whose S rows lanes 0..15 own
        const float a_row = __shfl_sync(kFull, alpha, lane & 15);
        if (j >= 1 && __any_sync(kFull, a_row != 1.f)) {
          // O must hold P(j-1) V(j-1) before it is scaled, and no MMA may run while the warp-wide
          // tensor-memory stores rewrite this quarter (lanes 0..15 store back qNope and both S buffers
          // unchanged): QK(j+1) of this piece, which may already be running into the other S buffer, is
          // waited for; QK(j+2) is not issued before s_free below, and PV(j) waits for P(j).  (A next
          // piece's first QK waits for its query, which is loaded after this piece.)
          ok = wait_all(kv_empty + ((G - 1) % kStages), ((G - 1) / kStages) & 1, status, kDevTimeoutODone);
          if (ok && j + 1 < pc.n_tiles)
            ok = wait_all(s_full((G + 1) & 1), ((G + 1) >> 1) & 1, status, kDevTimeoutSFull);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 2
          for (int c32 = 0; c32 < 512 / 32; ++c32) {
            uint32_t regs[32];
            const uint32_t addr = tmem_warp + c32 * 32;
            tmem_ld32(addr, regs);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) regs[c] = upper ? __float_as_uint(__uint_as_float(regs[c]) * a_row) : regs[c];
            tmem_st32(addr, regs);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(s_free(G & 1));
        const float m_base = (m_run == -INFINITY) ? 0.f : m_run;
        // P = 2^(x*scale - m), a pair of columns at a time (-inf masked keys give exactly 0)
        const uint64_t scale2 = f2pack(raw_max ? scale : 1.f, raw_max ? scale : 1.f);
        const uint64_t negm2 = f2pack(-m_base, -m_base);
        uint64_t acc0 = f2pack(0.f, 0.f), acc1 = f2pack(0.f, 0.f);
        uint32_t pk[kTileKeys / 2];
#pragma unroll
        for (int c = 0; c < kTileKeys; c += 2) {
          float e0, e1;
          f2unpack(fma_x2(f2pack(x[c], x[c + 1]), scale2, negm2), e0, e1);
          e0 = fast_exp2(e0);
          e1 = fast_exp2(e1);
          if ((c >> 1) & 1) acc1 = add_x2(acc1, f2pack(e0, e1));
          else acc0 = add_x2(acc0, f2pack(e0, e1));
          pk[c >> 1] = pack2(e0, e1, (T*)nullptr);
        }
        float s0, s1;
        f2unpack(add_x2(acc0, acc1), s0, s1);
        l_run = l_run * alpha + (s0 + s1);
        if (!upper) {
          // P row hr into this tile's kRope block (S(j) is computed, so the block is dead): 64 keys x 16 bit
          const uint32_t prow = smem_addr(sKV + (G % kStages) * kKvBytes + kPOff) + hr * 128;
#pragma unroll
          for (int ch = 0; ch < kTileKeys / 8; ++ch)
            st_shared_v4(prow + ((ch ^ sw) << 4), make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full + (G % kStages));
      }
      if (!ok) break;
      // ---- epilogue of the piece: O / l staged in the last tile's slot, TMA stores, then the next query
      const int s_last = (G - 1) % kStages;
      ok = wait_all(pv_last, (k - k0) & 1, status, kDevTimeoutODone);
      if (!ok) break;
      tc_fence_after();
      const float l_row = __shfl_sync(kFull, l_run, lane & 15);
      const float m_row = __shfl_sync(kFull, m_run, lane & 15);
      // a row whose allowed keys all lie before this range (possible only in a partial) contributes nothing
      const bool empty = !(l_row > 0.f);
      const float inv_l = empty ? 0.f : pv_d / l_row;  // pv_d = 1 unless the cache is int8
      const float lse_row = empty ? -INFINITY : (m_row == -INFINITY ? 0.f : m_row) * kLn2 + logf(l_row);
      uint8_t* stage = sKV + s_last * kKvBytes;
      const uint32_t stage_row = smem_addr(stage) + hr * 128;  // this row in each 8 KB staging box
      const bool final_out = pc.part < 0;
      const int n_rounds = final_out ? 1 : 2;
      for (int r = 0; r < n_rounds && ok; ++r, ++R) {
        // the previous round's boxes must have been read by its stores
        if (R > 0 && !(ok = wait_all(st_free, (R - 1) & 1, status, kDevTimeoutFinal))) break;
        if (final_out) {
          // output in T: box b holds columns 64b .. 64b+63 of the 64 rows (lanes 16..31 hold all of O)
#pragma unroll 1
          for (int b = 0; b < 8; ++b) {
            uint32_t ra[32], rb[32];
            tmem_ld32(tmem_warp + b * 64, ra);
            tmem_ld32(tmem_warp + b * 64 + 32, rb);
            tmem_ld_wait();
            if (upper) {
              const uint32_t box = stage_row + b * kBlk;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const uint32_t* q = c < 4 ? ra + 8 * c : rb + 8 * (c - 4);
                uint4 v;
                v.x = pack2(__uint_as_float(q[0]) * inv_l, __uint_as_float(q[1]) * inv_l, (T*)nullptr);
                v.y = pack2(__uint_as_float(q[2]) * inv_l, __uint_as_float(q[3]) * inv_l, (T*)nullptr);
                v.z = pack2(__uint_as_float(q[4]) * inv_l, __uint_as_float(q[5]) * inv_l, (T*)nullptr);
                v.w = pack2(__uint_as_float(q[6]) * inv_l, __uint_as_float(q[7]) * inv_l, (T*)nullptr);
                st_shared_v4(box + ((c ^ sw) << 4), v);
              }
            }
          }
        } else {
          // fp32 partial, round r: box b holds columns 256r + 32b .. +31
#pragma unroll 1
          for (int b = 0; b < 8; ++b) {
            uint32_t ra[32];
            tmem_ld32(tmem_warp + 256 * r + 32 * b, ra);
            tmem_ld_wait();
            if (upper) {
              const uint32_t box = stage_row + b * kBlk;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                st_shared_v4(box + ((c ^ sw) << 4),
                             make_uint4(__float_as_uint(__uint_as_float(ra[4 * c + 0]) * inv_l),
                                        __float_as_uint(__uint_as_float(ra[4 * c + 1]) * inv_l),
                                        __float_as_uint(__uint_as_float(ra[4 * c + 2]) * inv_l),
                                        __float_as_uint(__uint_as_float(ra[4 * c + 3]) * inv_l)));
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(st_full);
        if (threadIdx.x == 0) {
          if (mbar_wait(st_full, R & 1, status, kDevTimeoutFinal)) {
            for (int b = 0; b < 8; ++b) {
              if (final_out)
                tma_store_3d(&tmO, stage + b * kBlk, 64 * b, h0, pc.token0);
              else
                tma_store_3d(&tmPO, stage + b * kBlk, 256 * r + 32 * b, h0, pc.part * p.tpc);
            }
            bulk_commit_group();
            bulk_wait_read_all();
          }
          mbar_arrive(st_free);
        }
      }
      if (!ok) break;
      if (!upper) {
        if (final_out) {
          if (p.lse) p.lse[(size_t)(pc.token0 + t_local) * p.heads + head] = lse_row;
        } else {
          p.part_lse[((size_t)pc.part * p.tpc + t_local) * p.heads + head] = lse_row;
        }
      }
      // O has been read: the next chunk's query may go in (its qNope stores clobber O)
      tc_fence_before();
      if (k + 1 < k1) {
        const MlaPiece pn = p.pieces[k + 1];
        load_query<T>(p, &tmQr, sQr, q_full, tmem_warp, h0, pn.token0, t_local, head, upper);
      }
      // the staging slot goes back to the producer once the stores have read it
      if (threadIdx.x == 0) {
        ok = mbar_wait(st_free, (R - 1) & 1, status, kDevTimeoutFinal);
        mbar_arrive(kv_empty + s_last);
      }
      ok = __all_sync(kFull, ok);
    }
    if (threadIdx.x == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge of the partial results of one token's key ranges by their lse:
// lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.
// One CTA per (token, 8 heads); one warp per head, 16 output columns per lane.
template <typename T>
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaCombine* work, const MlaParams p) {
  // launched as a programmatic dependent of mla_kernel: wait until that grid has completed and its writes
  // (the partials) are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const MlaCombine w = work[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y * 8 + warp;
  if (head >= p.heads) return;
  auto row = [&](int s) { return ((size_t)(w.part_begin + s) * p.tpc + w.t_local) * p.heads + head; };
  float m = -INFINITY;
  for (int s = 0; s < w.n_parts; ++s) m = fmaxf(m, p.part_lse[row(s)]);
  // a row with no allowed key in any part (possible only with an explicit mask) gets O = 0, lse = -inf
  const bool none = m == -INFINITY;
  float l = 0.f;
  for (int s = 0; s < w.n_parts && !none; ++s) l += __expf(p.part_lse[row(s)] - m);
  const float lse = none ? -INFINITY : m + __logf(l);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < w.n_parts && !none; ++s) {
    const size_t pr = row(s);
    const float wgt = __expf(p.part_lse[pr] - lse);  // 0 for a part whose rows saw no allowed key
    const float4* src = reinterpret_cast<const float4*>(p.part_o + pr * kDNope);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = src[i * 32 + lane];
      acc[i * 4 + 0] += wgt * v.x;
      acc[i * 4 + 1] += wgt * v.y;
      acc[i * 4 + 2] += wgt * v.z;
      acc[i * 4 + 3] += wgt * v.w;
    }
  }
  T* orow = reinterpret_cast<T*>(p.out) + ((size_t)w.token * p.heads + head) * kDNope;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint2 v;
    v.x = pack2(acc[i * 4 + 0], acc[i * 4 + 1], (T*)nullptr);
    v.y = pack2(acc[i * 4 + 2], acc[i * 4 + 3], (T*)nullptr);
    *reinterpret_cast<uint2*>(orow + (i * 32 + lane) * 4) = v;
  }
  if (lane == 0 && p.lse) p.lse[(size_t)w.token * p.heads + head] = lse;
}

int mfail(char* err, size_t n, int st, const char* msg) {
  snprintf(err, n, "%s", msg);
  return st;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// rank-2 or rank-3 map with a 128-byte inner box and 128B swizzle
bool encode(CUtensorMap* map, void* base, int32_t dtype, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType t = dtype == ALA_F16   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                : dtype == ALA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dtype == ALA_I8  ? CU_TENSOR_MAP_DATA_TYPE_UINT8  // int8 codes move as bytes
                                                   : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(map, t, rank, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  const bool kv8 = cacheMode == ALA_MLA_CACHE_INT8_NZ;
  if (cacheMode != ALA_MLA_CACHE_KROPE_CTKV && !kv8)
    return mfail(err, n, ALA_UNSUPPORTED, "cacheMode must be KROPE_CTKV (1) or INT8_NZCACHE (2, int8 ctKV in the ND layout)");
  if (calcType == ALA_MLA_CALC_RING || calcType == ALA_MLA_CALC_PREFILL)
    return mfail(err, n, ALA_UNSUPPORTED, "calcType RING and PREFILL are not built");
  if (calcType != ALA_MLA_CALC_UNDEFINED && calcType != ALA_MLA_CALC_SPEC)
    return mfail(err, n, ALA_INVALID_PARAM, "calcType must be 0..3");
  if (maskType == 3 || maskType == 4 || maskType == 5)
    return mfail(err, n, ALA_INVALID_PARAM, "ALiBi masks apply only to the encoder paths");
  if (maskType != ALA_MLA_MASK_UNDEFINED && maskType != ALA_MLA_MASK_SPEC)
    return mfail(err, n, maskType == ALA_MLA_MASK_FREE ? ALA_UNSUPPORTED : ALA_INVALID_PARAM,
                 "maskType must be UNDEFINED (0) or SPEC (1)");
  if (kv8) {
    if (!qkDescale || !qkDescale->data || !pvDescale || !pvDescale->data)
      return mfail(err, n, ALA_NULL_REQUIRED, "qkDescale and pvDescale are required with the int8 cache (cacheMode 2)");
    if (qkDescale->dtype != ALA_F32 || pvDescale->dtype != ALA_F32)
      return mfail(err, n, ALA_INVALID_DTYPE, "qkDescale and pvDescale must be fp32");
    if (qkDescale->ndim != 1 || qkDescale->dims[0] != headNum || pvDescale->ndim != 1 || pvDescale->dims[0] != headNum)
      return mfail(err, n, ALA_INVALID_SHAPE, "qkDescale and pvDescale must be [headNum]");
  } else if ((qkDescale && qkDescale->data) || (pvDescale && pvDescale->data)) {
    return mfail(err, n, ALA_INVALID_PARAM, "qkDescale/pvDescale are passed only with the int8 cache (cacheMode 2)");
  }
  if (headNum <= 0) return mfail(err, n, ALA_INVALID_PARAM, "headNum must be > 0");
  if (headNum % 64 != 0) return mfail(err, n, ALA_UNSUPPORTED, "headNum must be a multiple of 64");
  if (kvHeadNum != 1) return mfail(err, n, ALA_UNSUPPORTED, "kvHeadNum must be 1");
  if (!std::isfinite(qkScale)) return mfail(err, n, ALA_INVALID_PARAM, "qkScale must be finite");
  const int32_t dt = qRope->dtype;  // the MMA and output type
  if (dt != ALA_BF16 && dt != ALA_F16) return mfail(err, n, ALA_INVALID_DTYPE, "qRope must be bf16 or f16");
  if (kv8) {
    if (ctKV->dtype != ALA_I8) return mfail(err, n, ALA_INVALID_DTYPE, "ctKV must be int8 with cacheMode 2");
    if (qNope->dtype != ALA_I8 && qNope->dtype != dt)
      return mfail(err, n, ALA_INVALID_DTYPE, "qNope must be int8 or qRope's dtype with cacheMode 2");
    if (kRope->dtype != dt || attenOut->dtype != dt)
      return mfail(err, n, ALA_INVALID_DTYPE, "kRope and attenOut must have qRope's dtype");
    // the converter and query loads read 16-byte pieces
    if (reinterpret_cast<uintptr_t>(ctKV->data) % 16 || reinterpret_cast<uintptr_t>(qNope->data) % 16)
      return mfail(err, n, ALA_INVALID_PARAM, "ctKV and qNope must be 16-byte aligned");
  } else if (qNope->dtype != dt || ctKV->dtype != dt || kRope->dtype != dt || attenOut->dtype != dt) {
    return mfail(err, n, ALA_INVALID_DTYPE, "qNope, ctKV, kRope and attenOut must have qRope's dtype");
  }
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
  if (!(bs > 0 && bs % 16 == 0)) return mfail(err, n, ALA_UNSUPPORTED, "blockSize must be a multiple of 16");
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
  // the explicit MASK_TYPE_SPEC mask (MLA page, parameter table, rows mask and maskType): [tokens, maxSeqLen]
  const bool has_mask = mask && mask->data;
  if (has_mask) {
    if (maskType != ALA_MLA_MASK_SPEC)
      return mfail(err, n, ALA_INVALID_PARAM, "a mask tensor is passed only with maskType SPEC (1)");
    if (mask->dtype != ALA_F16 && mask->dtype != ALA_BF16)
      return mfail(err, n, ALA_INVALID_DTYPE, "mask must be fp16 or bf16");
    if (mask->ndim != 2 || mask->dims[0] != tokens || mask->dims[1] < 1)
      return mfail(err, n, ALA_INVALID_SHAPE, "mask must be [tokens, maxSeqLen]");
    if (reinterpret_cast<uintptr_t>(mask->data) % 2) return mfail(err, n, ALA_INVALID_PARAM, "mask must be 2-byte aligned");
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
    if (has_mask && cl[b] > mask->dims[1])
      return mfail(err, n, ALA_INVALID_SHAPE, "the mask's maxSeqLen is shorter than a contextLens entry");
    sum_q += q;
  }
  if (sum_q != tokens) return mfail(err, n, ALA_INVALID_SHAPE, "sum(qseqlen) != tokens");
  if (ctKV->dims[0] * bs >= ((int64_t)1 << 31)) return mfail(err, n, ALA_UNSUPPORTED, "cache has more than 2^31 rows");

  plan->dtype = dt;
  plan->kv8 = kv8;
  plan->qn_int8 = kv8 && qNope->dtype == ALA_I8;
  plan->qk_descale = kv8 ? static_cast<const float*>(qkDescale->data) : nullptr;
  plan->pv_descale = kv8 ? static_cast<const float*>(pvDescale->data) : nullptr;
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
  plan->mask = has_mask ? static_cast<const uint16_t*>(mask->data) : nullptr;
  plan->mask_cols = has_mask ? mask->dims[1] : 0;
  plan->mask_f16 = has_mask && mask->dtype == ALA_F16;

  // ---- row blocks: tpc tokens x hpc heads, tpc the largest of 4, 2, 1 dividing every qseqlen
  int32_t tpc = 4;
  for (; tpc > 1; tpc >>= 1) {
    bool divides = true;
    for (int32_t b = 0; b < batch; ++b) divides = divides && plan->qs[b] % tpc == 0;
    if (divides) break;
  }
  const int32_t hpc = kRows / tpc;
  const int32_t groups = headNum / hpc;
  const int32_t ctas_per_lane = groups;
  plan->tpc = tpc;
  plan->hpc = hpc;
  plan->groups = groups;

  // ---- chunks and their 32-key tiles, end to end
  struct Chunk {
    int32_t b, token0, last, tiles, n_keys, row_step;
  };
  std::vector<Chunk> chunks;
  int64_t total_tiles = 0;
  for (int32_t b = 0, token = 0; b < batch; token += plan->qs[b], ++b) {
    for (int32_t t0 = 0; t0 < plan->qs[b]; t0 += tpc) {
      // the rule: token t0 + t of the chunk allows keys 0 .. last + t; with an explicit mask every token
      // reads keys 0 .. contextLens - 1 and the mask decides
      const int32_t last = has_mask ? cl[b] - 1 : cl[b] - plan->qs[b] + t0;
      const int32_t n_keys = has_mask ? cl[b] : last + tpc;
      const int32_t tiles = (n_keys + kTileKeys - 1) / kTileKeys;
      chunks.push_back(Chunk{b, token + t0, last, tiles, n_keys, has_mask ? 0 : 1});
      total_tiles += tiles;
    }
  }
  // ---- lanes: equal contiguous ranges of that sequence, one CTA per lane and group
  const int64_t lanes_max = std::max<int64_t>(1, kPlannedSms / ctas_per_lane);
  const int64_t per_lane = std::max<int64_t>(kMinLaneTiles, (total_tiles + lanes_max - 1) / lanes_max);
  std::vector<MlaPiece> pieces;
  std::vector<int32_t> piece_lane;
  std::vector<MlaCombine> comb;
  int32_t parts = 0, lane_id = 0;
  int64_t pos = 0, lane_end = per_lane;
  for (const Chunk& ch : chunks) {
    const size_t first = pieces.size();
    for (int32_t t = 0; t < ch.tiles;) {
      const int32_t take = (int32_t)std::min<int64_t>(lane_end - pos, ch.tiles - t);
      pieces.push_back(MlaPiece{ch.b, ch.token0, t * kTileKeys, take, ch.last, -1, ch.n_keys, ch.row_step});
      piece_lane.push_back(lane_id);
      pos += take;
      t += take;
      if (pos == lane_end) {
        ++lane_id;
        lane_end += per_lane;
      }
    }
    const int32_t np = (int32_t)(pieces.size() - first);
    if (np > 1) {
      for (int32_t i = 0; i < np; ++i) pieces[first + i].part = parts + i;
      for (int32_t t = 0; t < tpc; ++t) comb.push_back(MlaCombine{ch.token0 + t, parts, np, t});
      parts += np;
    }
  }
  const int32_t n_lanes = pieces.empty() ? 0 : piece_lane.back() + 1;
  std::vector<int32_t> lane_off(n_lanes + 1, 0);
  for (int32_t l = 0, i = 0; l <= n_lanes; ++l) {
    while (i < (int32_t)pieces.size() && piece_lane[i] < l) ++i;
    lane_off[l] = i;
  }
  plan->n_lanes = n_lanes;
  plan->n_work = n_lanes * ctas_per_lane;
  plan->n_splits_total = parts;
  plan->n_combine = (int32_t)comb.size();
  auto align = [](uint64_t x) { return (x + 255) / 256 * 256; };
  plan->off_work = 256;
  plan->off_lanes = align(plan->off_work + sizeof(MlaPiece) * std::max<size_t>(pieces.size(), 1));
  plan->off_rows = align(plan->off_lanes + sizeof(int32_t) * lane_off.size());
  plan->off_part_lse = align(plan->off_rows + sizeof(MlaCombine) * std::max<size_t>(comb.size(), 1));
  const uint64_t part_rows = (uint64_t)parts * tpc * headNum;
  plan->off_part_o = align(plan->off_part_lse + sizeof(float) * part_rows);
  plan->ws_size = align(plan->off_part_o + sizeof(float) * part_rows * kDNope);
  plan->image_size = plan->off_part_lse;  // only the schedule is uploaded; partials are written by the kernel
  plan->image.assign(plan->image_size, 0);
  std::memcpy(plan->image.data() + plan->off_work, pieces.data(), sizeof(MlaPiece) * pieces.size());
  std::memcpy(plan->image.data() + plan->off_lanes, lane_off.data(), sizeof(int32_t) * lane_off.size());
  std::memcpy(plan->image.data() + plan->off_rows, comb.data(), sizeof(MlaCombine) * comb.size());
  return ALA_OK;
}

int mla_upload(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t n) {
  if (!plan->pinned) {
    if (cudaHostAlloc(&plan->pinned, plan->image_size, cudaHostAllocDefault) == cudaSuccess)
      std::memcpy(plan->pinned, plan->image.data(), plan->image_size);
    else {
      plan->pinned = nullptr;
      cudaGetLastError();
    }
  }
  if (cudaMemcpyAsync(workspace, plan->pinned ? plan->pinned : plan->image.data(), plan->image_size,
                      cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return mfail(err, n, ALA_CUDA_ERROR, "schedule upload failed");
  return ALA_OK;
}

int mla_run(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t n) {
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return mfail(err, n, ALA_INVALID_PARAM, "workspace must be 256-byte aligned");
  if (plan->n_work == 0) return ALA_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const cuuint32_t tpc = (cuuint32_t)plan->tpc, hpc = (cuuint32_t)plan->hpc;
  if (!plan->maps_ready) {
    const int es = 2;
    const cuuint64_t rows = (cuuint64_t)plan->num_blocks * plan->block_size;
    const cuuint32_t box_rows = (cuuint32_t)kv_box_rows(plan->block_size, kTileKeys);
    cuuint64_t qn_dims[3] = {512, (cuuint64_t)plan->heads, (cuuint64_t)plan->tokens};
    cuuint64_t qn_str[2] = {512 * es, (cuuint64_t)plan->heads * 512 * es};
    cuuint64_t qr_dims[3] = {64, (cuuint64_t)plan->heads, (cuuint64_t)plan->tokens};
    cuuint64_t qr_str[2] = {64 * es, (cuuint64_t)plan->heads * 64 * es};
    cuuint32_t q_box[3] = {64, hpc, tpc};
    cuuint64_t kv_dims[2] = {512, rows};
    cuuint64_t kv_str[1] = {512 * es};
    cuuint64_t kr_dims[2] = {64, rows};
    cuuint64_t kr_str[1] = {64 * es};
    cuuint32_t kv_box[2] = {64, box_rows};
    // ctKV seen as (64 elements, rows, 8 column blocks): one box is a whole 64-key tile, laid out
    // [column block][key][64 elements] as the 128B-swizzled K-major operand wants it
    cuuint64_t kv3_dims[3] = {64, rows, 8};
    cuuint64_t kv3_str[2] = {512 * es, 64 * es};
    cuuint32_t kv3_box[3] = {64, (cuuint32_t)kTileKeys, 8};
    // int8 codes: 512 bytes a row, seen as 128-byte column blocks (4 per row), same boxes of keys
    cuuint64_t k8_dims[2] = {512, rows};
    cuuint64_t k8_str[1] = {512};
    cuuint32_t k8_box[2] = {128, box_rows};
    cuuint64_t k83_dims[3] = {128, rows, 4};
    cuuint64_t k83_str[2] = {512, 128};
    cuuint32_t k83_box[3] = {128, (cuuint32_t)kTileKeys, 4};
    const bool kv_ok = plan->kv8 ? (encode(&plan->tmKV3, plan->ct_kv, ALA_I8, 3, k83_dims, k83_str, k83_box) &&
                                    encode(&plan->tmKV, plan->ct_kv, ALA_I8, 2, k8_dims, k8_str, k8_box))
                                 : (encode(&plan->tmKV3, plan->ct_kv, plan->dtype, 3, kv3_dims, kv3_str, kv3_box) &&
                                    encode(&plan->tmKV, plan->ct_kv, plan->dtype, 2, kv_dims, kv_str, kv_box));
    if (!kv_ok || !encode(&plan->tmQr, plan->q_rope, plan->dtype, 3, qr_dims, qr_str, q_box) ||
        !encode(&plan->tmKR, plan->k_rope, plan->dtype, 2, kr_dims, kr_str, kv_box) ||
        !encode(&plan->tmO, plan->out, plan->dtype, 3, qn_dims, qn_str, q_box))
      return mfail(err, n, ALA_CUDA_ERROR, "cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)");
    plan->maps_ready = true;
  }
  if (plan->n_splits_total == 0) {
    plan->tmPO = plan->tmO;  // never used: every piece writes the final output
  } else if (plan->tmPO_base != ws + plan->off_part_o) {
    cuuint64_t po_dims[3] = {512, (cuuint64_t)plan->heads, (cuuint64_t)plan->n_splits_total * tpc};
    cuuint64_t po_str[2] = {512 * 4, (cuuint64_t)plan->heads * 512 * 4};
    cuuint32_t po_box[3] = {32, hpc, tpc};
    if (!encode(&plan->tmPO, ws + plan->off_part_o, ALA_F32, 3, po_dims, po_str, po_box))
      return mfail(err, n, ALA_CUDA_ERROR, "cuTensorMapEncodeTiled failed for the partial-output map");
    plan->tmPO_base = ws + plan->off_part_o;
  }
  // a bound workspace already holds the schedule and status words that only a failed execution sets
  // (ala_op_bind_workspace); any other workspace gets both copied in
  if (workspace != plan->bound_ws) {
    const int st = mla_upload(plan, workspace, stream, err, n);
    if (st != ALA_OK) return st;
  }
  MlaParams p{};
  p.pieces = reinterpret_cast<const MlaPiece*>(ws + plan->off_work);
  p.lane_off = reinterpret_cast<const int32_t*>(ws + plan->off_lanes);
  p.block_tables = plan->block_tables;
  p.q_nope = static_cast<const uint8_t*>(plan->q_nope);
  p.ct_kv = static_cast<const uint8_t*>(plan->ct_kv);
  p.k_rope = static_cast<const uint8_t*>(plan->k_rope);
  p.out = plan->out;
  p.lse = plan->lse;
  p.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
  p.part_lse = reinterpret_cast<float*>(ws + plan->off_part_lse);
  p.status = reinterpret_cast<int*>(ws);
  p.heads = plan->heads;
  p.groups = plan->groups;
  p.tpc = plan->tpc;
  p.hpc = plan->hpc;
  p.max_blocks = plan->max_blocks;
  p.block_size = plan->block_size;
  p.kv_box_rows = kv_box_rows(plan->block_size, kTileKeys);
  p.oob_row = (int32_t)(plan->num_blocks * plan->block_size);
  p.scale_log2 = plan->qk_scale * kLog2e;
  p.qk_descale = plan->qk_descale;
  p.pv_descale = plan->pv_descale;
  p.qn_int8 = plan->qn_int8 ? 1 : 0;
  p.mask = plan->mask;
  p.mask_cols = plan->mask_cols;
  p.mask_f16 = plan->mask_f16 ? 1 : 0;
  p.mask_vec = (reinterpret_cast<uintptr_t>(plan->mask) % 16 == 0 && plan->mask_cols % 8 == 0) ? 1 : 0;
  const bool f16 = plan->dtype == ALA_F16;
  auto kern = plan->kv8 ? (f16 ? mla_kernel<__half, true> : mla_kernel<__nv_bfloat16, true>)
                        : (f16 ? mla_kernel<__half, false> : mla_kernel<__nv_bfloat16, false>);
  const int threads = plan->kv8 ? 320 : 192;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e == cudaSuccess) {
    kern<<<plan->n_work, threads, kSmem, stream>>>(plan->tmQr, plan->tmKV, plan->tmKV3, plan->tmKR, plan->tmO,
                                                   plan->tmPO, p);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && plan->n_combine > 0) {
    auto ck = plan->dtype == ALA_F16 ? mla_combine_kernel<__half> : mla_combine_kernel<__nv_bfloat16>;
    // a programmatic dependent launch: the combine grid is scheduled during mla_kernel's tail instead of
    // after it, and griddepcontrol.wait holds it until mla_kernel has completed
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan->n_combine, (plan->heads + 7) / 8);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, ck, reinterpret_cast<const MlaCombine*>(ws + plan->off_rows), p);
  }
  if (e != cudaSuccess) return mfail(err, n, ALA_CUDA_ERROR, cudaGetErrorString(e));
  return ALA_OK;
}

MlaPlan::~MlaPlan() {
  if (pinned) cudaFreeHost(pinned);
}

}  // namespace ala
