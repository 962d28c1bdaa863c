// mla_wide.cu -- MLA decode with 128 query rows per CTA for sm_100a (ATB "MLA"
// page, definition and parameter table): per query token and head,
// O = softmax(qkScale * [qNope;qRope] . [ctKV;kRope]^T (+ mask)) ctKV and its lse,
// for requests with one query token per CTA row block (decode, or speculative
// tokens whose counts share no factor 2 or 4) over a 16-bit latent cache.
//
// Why 128 rows.  The 128 heads of a token are one M = 128 tensor-core tile, which
// runs at twice the rate of the M = 64 tiles of mla.cu.  The fp32 output of 128
// rows x 512 latent columns would fill all 512 tensor-memory columns, so a pair
// of CTAs serves the token: CTA `half` owns output columns [256 half, +256).
// Both compute the whole score tile S = Q K^T themselves (the QK work is done
// twice, the P V work once), so nothing is exchanged between them; each stages
// the full cache tile (the pair's second read comes from L2).
//
// Tensor memory (128 lanes = 128 heads):
//   columns   0..127  qNope dims 0..255 (16-bit pairs): the A operand of the
//                     first half of the QK MMAs (TS form);
//   columns 128..255  S, double buffered (64 columns each); P(j) is written
//                     over S(j) as 16-bit pairs and read from there by the
//                     P V MMAs (TS form);
//   columns 256..511  this CTA's half of O.
// Shared memory: qNope dims 256..511 and qRope (SS A operands, 80 KB) and a
// two-deep ring of 64-key tiles (ctKV 64 KB + kRope 8 KB each).  A slot is
// loaded and released in two parts: part A (the other half's ctKV columns and
// kRope, 40 KB) is dead once the tile's QK has completed, part B (this CTA's
// ctKV columns, the V of its P V, 32 KB) once the P V has.  The QK of tile
// j+2 reuses the S buffer of tile j only after P(j) V has completed, so it
// starts with the MMAs over part A, loaded long before, while part B is still
// on its way.
//
//   warp 4      TMA producer (one thread): per piece the query's shared-memory
//               part, then the tiles gathered through the block table, and
//               L2 prefetches ahead of them.
//   warp 5      tcgen05 issuer (one thread): QK(j+1) ahead of PV(j); the
//               S buffer of QK(j) is reused once PV(j-2) has completed.
//   warps 0..3  softmax: thread r owns row r (head h0 + r): scale, mask,
//               online max and sum, P over S, the O rescale when the max grew
//               by more than 2^8; at the end of a piece it loads the next
//               piece's qNope into tensor memory, then normalises its O half,
//               stages it in the last tile's slot and one thread writes it out
//               with TMA stores (fp32 partials when the piece's key range was
//               split across CTAs, merged by lse afterwards).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "internal.h"
#include "mla_common.cuh"
#include "ptx.cuh"

namespace ala {
namespace mlak {

namespace {

constexpr int kWRows = 128;
constexpr int kWBlkK = kTileKeys * 128;  // one 64-column block of a 64-key tile: 8 KB
constexpr int kWBlkQ = kWRows * 128;     // one 64-column block of the 128 query rows: 16 KB
constexpr int kWQnBytes = 4 * kWBlkQ;    // qNope dims 256..511 of the 128 rows
constexpr int kWQrBytes = kWBlkQ;        // qRope
constexpr int kWKvBytes = 9 * kWBlkK;    // ctKV blocks 0..7 + kRope
constexpr int kWStages = 2;
// q_full, q_free, full_a[2], full_b[2], empty_a[2], empty_b[2], s_full[2], p_full[2], pv_done[2], o_free,
// st_full, st_free, fin
constexpr int kWNBars = 2 + 7 * kWStages + 4;
constexpr int kWPartA = 5 * kWBlkK;  // part A bytes: four ctKV column blocks + kRope
constexpr int kWPartB = 4 * kWBlkK;  // part B bytes: four ctKV column blocks
constexpr int kWSmem = 1024 + kWQnBytes + kWQrBytes + kWStages * kWKvBytes + kWNBars * 8 + 16;
static_assert(kWSmem <= 232448, "shared memory budget");
static_assert(4 * kWBlkQ <= kWKvBytes, "the output staging (four 16 KB boxes) must fit in a ring slot");
constexpr uint32_t kWQnCol = 0;
constexpr uint32_t kWSCol = 128;
constexpr uint32_t kWOCol = 256;
constexpr uint32_t kWTmemCols = 512;

#ifndef ALA_MLA_WIDE_PREFETCH_TILES
#define ALA_MLA_WIDE_PREFETCH_TILES 3  // the producer asks L2 for the tiles this far ahead of its loads
#endif

template <typename T>
__global__ void __launch_bounds__(192, 1)
    mla_wide_kernel(const __grid_constant__ CUtensorMap tmQn, const __grid_constant__ CUtensorMap tmQr,
                    const __grid_constant__ CUtensorMap tmKV, const __grid_constant__ CUtensorMap tmKV3,
                    const __grid_constant__ CUtensorMap tmKR, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmPO, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQn = smem;                 // qNope dims 256..511: four 16 KB column blocks
  uint8_t* sQr = sQn + kWQnBytes;      // qRope
  uint8_t* sKV = sQr + kWQrBytes;      // [kWStages][kWKvBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kWStages * kWKvBytes);
  uint64_t* q_full = bars;             // the piece's query is in place (128 TMEM stores + the TMA bytes)
  uint64_t* q_free = bars + 1;         // every QK of the piece has completed
  uint64_t* full_a = bars + 2;         // [2] part A of the slot's tile has landed
  uint64_t* full_b = bars + 4;         // [2] part B has landed
  uint64_t* empty_a = bars + 6;        // [2] part A is free (the tile's QK has completed)
  uint64_t* empty_b = bars + 8;        // [2] part B is free (the tile's P V has completed)
  uint64_t* s_full = bars + 10;        // [2] per S buffer
  uint64_t* p_full = bars + 12;        // [2] per S buffer: P written over S
  uint64_t* pv_done = bars + 14;       // [2] per S buffer: the P V of that buffer's tile has completed
  uint64_t* o_free = bars + 16;        // the epilogue has read O
  uint64_t* st_full = bars + 17;
  uint64_t* st_free = bars + 18;
  uint64_t* fin = bars + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kWNBars);

  const int warp = threadIdx.x >> 5;
  const int half = blockIdx.x & 1;                 // output columns [256 half, 256 half + 256)
  const int cb_own = 4 * half;                     // the ctKV column blocks of this CTA's V (part B)
  const int cb_other = 4 - cb_own;                 // the other half's column blocks (part A, with kRope)
  const int pair = blockIdx.x >> 1;
  const int ln = pair / p.groups;
  const int h0 = (pair - ln * p.groups) * kWRows;  // first head of this CTA's rows
  const int k0 = p.lane_off[ln];
  const int k1 = p.lane_off[ln + 1];
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 129);
    mbar_init(q_free, 1);
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(full_a + s, 1);
      mbar_init(full_b + s, 1);
      mbar_init(empty_a + s, 1);
      mbar_init(empty_b + s, 1);
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 128);
      mbar_init(pv_done + s, 1);
    }
    mbar_init(o_free, 128);
    mbar_init(st_full, 128);
    mbar_init(st_free, 1);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kWTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer (one elected thread)
    if (elect_one()) {
      tma_prefetch_desc(&tmQn);
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmKV3);
      tma_prefetch_desc(&tmKR);
      const int bs = p.block_size;
      const bool whole = bs % kTileKeys == 0;  // a tile lies in one page: one 3-D box holds its ctKV part
      const int box_rows = bs < kTileKeys ? bs : kTileKeys;
      int G = 0;  // tiles issued so far by this CTA
      int kf = k0, jf = 0, Gf = 0;  // L2 prefetch cursor: piece, tile, CTA tile
      MlaPiece pf = k0 < k1 ? p.pieces[k0] : MlaPiece{};
      bool ok = true;
      for (int k = k0; k < k1 && ok; ++k) {
        const MlaPiece pc = p.pieces[k];
        const int32_t* bt = p.block_tables + (size_t)pc.b * p.max_blocks;
        const int n_pages = (pc.n_keys + bs - 1) / bs;  // pages holding the keys the piece may read
        // the query's shared-memory part, once the previous piece's QKs have completed
        if (k > k0 && !mbar_wait(q_free, (k - 1 - k0) & 1, status, kDevTimeoutQ)) {
          ok = false;
          break;
        }
        mbar_expect_tx(q_full, kWQnBytes + kWQrBytes);
        for (int cb = 0; cb < 4; ++cb) tma_load_3d(sQn + cb * kWBlkQ, &tmQn, q_full, 256 + 64 * cb, h0, pc.token0);
        tma_load_3d(sQr, &tmQr, q_full, 0, h0, pc.token0);
        if (k + 1 < k1) {  // the next piece's qNope rows, for the softmax threads' loads at the piece boundary
          const uint8_t* qn = p.q_nope + ((size_t)p.pieces[k + 1].token0 * p.heads + h0) * kDNope * 2;
          for (int c = 0; c < 4; ++c) bulk_prefetch_l2(qn + c * 32768, 32768);
        }
        for (int j = 0; j < pc.n_tiles; ++j) {
          for (; kf < k1 && Gf <= G + ALA_MLA_WIDE_PREFETCH_TILES; ++Gf) {
            const int32_t* btf = p.block_tables + (size_t)pf.b * p.max_blocks;
            const int npf = (pf.n_keys + bs - 1) / bs;
            for (int r0 = 0; r0 < kTileKeys; r0 += box_rows) {
              const int pos = pf.kv_begin + jf * kTileKeys + r0;
              const int row = paged_row(btf, pos, bs, npf, p.oob_row, p.status);
              if (row >= 0 && row < p.oob_row) {  // a block index outside the cache is never touched
                bulk_prefetch_l2(p.ct_kv + (size_t)row * (2 * kDNope), box_rows * 2 * kDNope);
                bulk_prefetch_l2(p.k_rope + (size_t)row * 128, box_rows * 128);
              }
            }
            if (++jf == pf.n_tiles) {
              jf = 0;
              if (++kf < k1) pf = p.pieces[kf];
            }
          }
          const int s = G % kWStages;
          uint8_t* dst = sKV + s * kWKvBytes;
          const int j0 = pc.kv_begin + j * kTileKeys;
          // part A (other half's columns, kRope) once the previous tile in the slot has finished its QK; part B
          // (this CTA's columns) once it has finished its P V
          for (int part = 0; part < 2 && ok; ++part) {
            uint64_t* empty = part == 0 ? empty_a : empty_b;
            uint64_t* full = (part == 0 ? full_a : full_b) + s;
            if (G >= kWStages && !mbar_wait(empty + s, ((G / kWStages) - 1) & 1, status, kDevTimeoutKEmpty)) {
              ok = false;
              break;
            }
            mbar_expect_tx(full, part == 0 ? kWPartA : kWPartB);
            const int cb0 = part == 0 ? cb_other : cb_own;
            for (int r0 = 0; r0 < kTileKeys; r0 += box_rows) {
              const int row = paged_row(bt, j0 + r0, bs, n_pages, p.oob_row, p.status);  // past the last page: zeros
              if (whole) {
                tma_load_3d(dst + cb0 * kWBlkK, &tmKV3, full, 0, row, cb0);  // [4 column blocks][key][64 elements]
              } else {
                for (int cb = cb0; cb < cb0 + 4; ++cb)
                  tma_load_2d(dst + cb * kWBlkK + r0 * 128, &tmKV, full, cb * 64, row);
              }
              if (part == 0) tma_load_2d(dst + 8 * kWBlkK + r0 * 128, &tmKR, full, 0, row);
            }
          }
          if (!ok) break;
          ++G;
        }
      }
      // no copy may be in flight when the CTA exits
      for (int t = G - kWStages < 0 ? 0 : G - kWStages; t < G; ++t) {
        mbar_wait(full_a + (t % kWStages), (t / kWStages) & 1, status, kDevTimeoutKFull);
        mbar_wait(full_b + (t % kWStages), (t / kWStages) & 1, status, kDevTimeoutKFull);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (one elected thread)
    if (elect_one()) {
      constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
      constexpr uint32_t idesc_qk = instr_desc(fmt, false, false, kWRows, kTileKeys);
      constexpr uint32_t idesc_pv = instr_desc(fmt, false, true, kWRows, 256);
      // base descriptors; a step adds its byte offset >> 4 to the start-address field
      const uint64_t dqn = smem_desc_sw128(smem_addr(sQn), 16, 1024);
      const uint64_t dqr = smem_desc_sw128(smem_addr(sQr), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv = smem_desc(smem_addr(sKV), kWBlkK, 1024, 2);  // ctKV as the MN-major V operand
      int total = 0;
      for (int k = k0; k < k1; ++k) total += p.pieces[k].n_tiles;
      // QK cursor: piece kq, tile jq of nq, CTA tile Gq; PV cursor likewise
      int kq = k0, jq = 0, nq = k0 < k1 ? p.pieces[k0].n_tiles : 0, Gq = 0;
      int kp = k0, jp = 0, np = nq, Gp = 0;
      bool ok = true;
      uint64_t t_prog = global_timer_ns();
      uint32_t it = 0;
      bool progressed = false;
      // the three groups of QK MMAs into S buffer d_s of slot offset so (the first one issued starts the sum)
      auto qk_ts = [&](uint32_t d_s, uint64_t so, bool first) {  // qNope dims 0..255 from tensor memory
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_ts(d_s, tmem + kWQnCol + kk * 8, dk + so + (uint64_t)(((kk >> 2) * kWBlkK + (kk & 3) * 32) >> 4),
                 idesc_qk, (first && kk == 0) ? 0u : 1u, false);
      };
      auto qk_ss = [&](uint32_t d_s, uint64_t so, bool first) {  // qNope dims 256..511 from shared memory
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          mma_ss(d_s, dqn + (uint64_t)(((kk >> 2) * kWBlkQ + (kk & 3) * 32) >> 4),
                 dk + so + (uint64_t)(((4 + (kk >> 2)) * kWBlkK + (kk & 3) * 32) >> 4), idesc_qk,
                 (first && kk == 0) ? 0u : 1u, false);
      };
      auto qk_rope = [&](uint32_t d_s, uint64_t so) {  // qRope x kRope
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(d_s, dqr + (uint64_t)((kk * 32) >> 4), dk + so + (uint64_t)((8 * kWBlkK + kk * 32) >> 4), idesc_qk, 1u,
                 false);
      };
      bool qk_a = false;  // the part-A MMAs of QK(Gq) are issued, the part-B ones not yet
      while (ok && Gp < total) {
        // QK(Gq) needs its S buffer (PV(Gq-2), which read P over it, has completed), first in a piece the
        // query, and leads PV by at most one tile; its MMAs over part A go first, those over part B once
        // that part has landed.  PV(Gp) needs P(Gp) and, first in a piece after the CTA's first, the
        // previous epilogue's read of O.
        const int bq = Gq & 1;
        const uint32_t d_s = tmem + kWSCol + 64 * bq;
        const uint64_t so_q = (uint64_t)((bq * kWKvBytes) >> 4);
        if (qk_a && mbar_test_wait(full_b + bq, (Gq >> 1) & 1)) {
          tc_fence_after();
          if (half == 0) qk_ts(d_s, so_q, false);  // this CTA's column blocks: dims 0..255
          else qk_ss(d_s, so_q, false);            // dims 256..511
          mma_commit(s_full + bq);
          const bool last = jq + 1 == nq;
          if (last) mma_commit(q_free);  // the piece's last QK: its query may be replaced
          else mma_commit(empty_a + bq);  // a piece's last slot is the epilogue's staging area instead
          qk_a = false;
          ++Gq;
          if (++jq == nq) {
            ++kq;
            jq = 0;
            nq = kq < k1 ? p.pieces[kq].n_tiles : 0;
          }
          progressed = true;
        } else if (!qk_a && Gq < total && Gq - Gp < 2 && mbar_test_wait(full_a + bq, (Gq >> 1) & 1) &&
                   (Gq < 2 || mbar_test_wait(pv_done + bq, ((Gq - 2) >> 1) & 1)) &&
                   (jq > 0 || mbar_test_wait(q_full, (kq - k0) & 1))) {
          tc_fence_after();
          if (half == 0) qk_ss(d_s, so_q, true);  // the other half's column blocks
          else qk_ts(d_s, so_q, true);
          qk_rope(d_s, so_q);
          qk_a = true;
          progressed = true;
        } else if (Gp < Gq && mbar_test_wait(p_full + (Gp & 1), (Gp >> 1) & 1) &&
                   (jp > 0 || kp == k0 || mbar_test_wait(o_free, (kp - 1 - k0) & 1))) {
          tc_fence_after();
          const int bp = Gp & 1;
          const uint64_t so = (uint64_t)((bp * kWKvBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTileKeys / 16; ++kk)
            // O (this half's 256 columns) += P (tensor memory, over S) x V (ctKV columns [256 half, +256))
            mma_ts(tmem + kWOCol, tmem + kWSCol + 64 * bp + kk * 8,
                   dv + so + (uint64_t)((4 * half * kWBlkK + kk * 16 * 128) >> 4), idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u,
                   false);
          mma_commit(pv_done + bp);
          // part B returns to the producer; a piece's last slot is the epilogue's staging area instead
          if (jp + 1 < np) mma_commit(empty_b + bp);
          ++Gp;
          if (++jp == np) {
            ++kp;
            jp = 0;
            np = kp < k1 ? p.pieces[kp].n_tiles : 0;
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
  } else {
    // ------------------------------------------------------------ softmax / epilogue: thread r owns row r
    const int r = threadIdx.x;
    const int head = h0 + r;
    const uint32_t tmem_warp = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int sw = r & 7;  // 128-byte swizzle of the row's 16-byte chunks
    const float scale = p.scale_log2;
    const bool has_mask = p.mask != nullptr;
    const bool raw_max = scale > 0.f && !has_mask;  // max of the raw scores, scale folded into the exponent
    // the row's qNope dims 0..255 into tensor memory columns 0..127 (16-bit pairs)
    auto load_qnope = [&](int token) {
      const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + ((size_t)token * p.heads + head) * kDNope * 2);
#pragma unroll
      for (int c32 = 0; c32 < 4; ++c32) {
        uint32_t rg[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 w = __ldg(src + c32 * 8 + v);
          rg[4 * v + 0] = w.x;
          rg[4 * v + 1] = w.y;
          rg[4 * v + 2] = w.z;
          rg[4 * v + 3] = w.w;
        }
        tmem_st32(tmem_warp + kWQnCol + c32 * 32, rg);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_full);
    };
    bool ok = true;
    int G = 0;  // tiles consumed
    int R = 0;  // output staging rounds
    if (k0 < k1) load_qnope(p.pieces[k0].token0);
    for (int k = k0; k < k1 && ok; ++k) {
      const MlaPiece pc = p.pieces[k];
      const int row_last = min(pc.last, pc.n_keys - 1);  // one token per chunk
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; j < pc.n_tiles; ++j, ++G) {
        const int b = G & 1;
        ok = wait_all(s_full + b, (G >> 1) & 1, status, kDevTimeoutSFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_col = tmem_warp + kWSCol + 64 * b;
        float x[kTileKeys];
        {
          uint32_t regs[2][32];
          tmem_ld32(s_col, regs[0]);
          tmem_ld32(s_col + 32, regs[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] = __uint_as_float(regs[c >> 5][c & 31]);
        }
        const int j0 = pc.kv_begin + j * kTileKeys;
        const int lim = row_last - j0;  // columns c <= lim are allowed
        if (has_mask) {
          float mk[kTileKeys];
          load_mask_log2(p, pc.token0, j0, mk);
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] = fmaf(x[c], scale, mk[c]);
        } else if (!raw_max) {
#pragma unroll
          for (int c = 0; c < kTileKeys; ++c) x[c] *= scale;
        }
        if (__any_sync(kFull, lim < kTileKeys - 1)) {  // only a range's last tile can hold masked keys
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
        if (j >= 1 && __any_sync(kFull, alpha != 1.f)) {
          // O must hold P(j-1) V(j-1) before it is scaled; PV(j) cannot start before P(j) below
          ok = wait_all(pv_done + (b ^ 1), ((G - 1) >> 1) & 1, status, kDevTimeoutODone);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 2
          for (int c32 = 0; c32 < 256 / 32; ++c32) {
            uint32_t regs[32];
            const uint32_t addr = tmem_warp + kWOCol + c32 * 32;
            tmem_ld32(addr, regs);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) regs[c] = __float_as_uint(__uint_as_float(regs[c]) * alpha);
            tmem_st32(addr, regs);
          }
        }
        const float m_base = (m_run == -INFINITY) ? 0.f : m_run;
        // P = 2^(x*scale - m), a pair of columns at a time (-inf masked keys give exactly 0), over S
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
        tmem_st32(s_col, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + b);
      }
      if (!ok) break;
      // ---- the next piece's qNope (every QK of this piece has completed: its last S was consumed)
      if (k + 1 < k1) {
        ok = wait_all(q_free, (k - k0) & 1, status, kDevTimeoutQ);
        if (!ok) break;
        tc_fence_after();
        load_qnope(p.pieces[k + 1].token0);
      }
      // ---- epilogue of the piece: O / l staged in the last tile's slot, TMA stores
      const int s_last = (G - 1) & 1;
      ok = wait_all(pv_done + s_last, ((G - 1) >> 1) & 1, status, kDevTimeoutODone);
      if (!ok) break;
      tc_fence_after();
      // a row whose allowed keys all lie outside this range (possible only in a partial or with a mask)
      const bool empty = !(l_run > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l_run;
      const float lse_row = empty ? -INFINITY : (m_run == -INFINITY ? 0.f : m_run) * kLn2 + logf(l_run);
      uint8_t* stage = sKV + s_last * kWKvBytes;
      const uint32_t stage_row = smem_addr(stage) + r * 128;  // this row in each 16 KB staging box
      const bool final_out = pc.part < 0;
      const int n_rounds = final_out ? 1 : 2;
      for (int rd = 0; rd < n_rounds && ok; ++rd, ++R) {
        // the previous round's boxes must have been read by its stores
        if (R > 0 && !(ok = wait_all(st_free, (R - 1) & 1, status, kDevTimeoutFinal))) break;
        if (final_out) {
          // output in T: box bx holds this half's columns 64 bx .. 64 bx + 63 of the 128 rows
#pragma unroll 1
          for (int bx = 0; bx < 4; ++bx) {
            uint32_t ra[32], rb[32];
            tmem_ld32(tmem_warp + kWOCol + bx * 64, ra);
            tmem_ld32(tmem_warp + kWOCol + bx * 64 + 32, rb);
            tmem_ld_wait();
            const uint32_t box = stage_row + bx * kWBlkQ;
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
        } else {
          // fp32 partial, round rd: box bx holds this half's columns 128 rd + 32 bx .. +31
#pragma unroll 1
          for (int bx = 0; bx < 4; ++bx) {
            uint32_t ra[32];
            tmem_ld32(tmem_warp + kWOCol + 128 * rd + 32 * bx, ra);
            tmem_ld_wait();
            const uint32_t box = stage_row + bx * kWBlkQ;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              st_shared_v4(box + ((c ^ sw) << 4),
                           make_uint4(__float_as_uint(__uint_as_float(ra[4 * c + 0]) * inv_l),
                                      __float_as_uint(__uint_as_float(ra[4 * c + 1]) * inv_l),
                                      __float_as_uint(__uint_as_float(ra[4 * c + 2]) * inv_l),
                                      __float_as_uint(__uint_as_float(ra[4 * c + 3]) * inv_l)));
          }
        }
        if (rd + 1 == n_rounds) {
          // every read of O is done: the next piece's P V may overwrite it
          tc_fence_before();
          mbar_arrive(o_free);
        }
        fence_proxy_async_smem();
        mbar_arrive(st_full);
        if (threadIdx.x == 0) {
          if (mbar_wait(st_full, R & 1, status, kDevTimeoutFinal)) {
            for (int bx = 0; bx < 4; ++bx) {
              if (final_out)
                tma_store_3d(&tmO, stage + bx * kWBlkQ, 256 * half + 64 * bx, h0, pc.token0);
              else
                tma_store_3d(&tmPO, stage + bx * kWBlkQ, 256 * half + 128 * rd + 32 * bx, h0, pc.part);
            }
            bulk_commit_group();
            bulk_wait_read_all();
          }
          mbar_arrive(st_free);
        }
      }
      if (!ok) break;
      if (half == 0) {  // both halves hold the same lse; one writes it
        if (final_out) {
          if (p.lse) p.lse[(size_t)pc.token0 * p.heads + head] = lse_row;
        } else {
          p.part_lse[(size_t)pc.part * p.heads + head] = lse_row;
        }
      }
      // the staging slot goes back to the producer once the stores have read it
      if (threadIdx.x == 0) {
        ok = mbar_wait(st_free, (R - 1) & 1, status, kDevTimeoutFinal);
        mbar_arrive(empty_a + s_last);
        mbar_arrive(empty_b + s_last);
      }
      ok = __all_sync(kFull, ok);
    }
    if (threadIdx.x == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kWTmemCols);
  }
}

}  // namespace

int mla_wide_smem_bytes() { return kWSmem; }

cudaError_t launch_mla_wide(int32_t dtype, int grid, const CUtensorMap& tmQn, const CUtensorMap& tmQr,
                            const CUtensorMap& tmKV, const CUtensorMap& tmKV3, const CUtensorMap& tmKR,
                            const CUtensorMap& tmO, const CUtensorMap& tmPO, const MlaParams& p, cudaStream_t stream) {
  auto kern = dtype == kF16 ? mla_wide_kernel<__half> : mla_wide_kernel<__nv_bfloat16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kWSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 192, kWSmem, stream>>>(tmQn, tmQr, tmKV, tmKV3, tmKR, tmO, tmPO, p);
  return cudaGetLastError();
}

}  // namespace mlak
}  // namespace ala
