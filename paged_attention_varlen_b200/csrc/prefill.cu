// prefill.cu -- masked attention over packed variable-length sequences for
// sm_100a, with K/V read from a contiguous packed tensor or from a paged cache
// through a block table (ATB "PrefixEncoder" page, definition and parameter
// table; nalar.dev padding-mask article, sections on packing and on fused
// kernels that apply the mask rule without materialising it).
//
// One CTA computes up to two blocks of 128 query rows that read the same kv
// head (two query heads of a GQA group, or two consecutive row tiles of one
// head), so each K/V tile staged in shared memory serves 256 rows.
//
//   warps 8, 10  TMA producers: warp 8 both Q tiles of each unit and the K
//                tiles (128 keys, 2-deep ring), warp 10 the V tiles (3-deep
//                ring, 2-deep for sqrt ALiBi, whose bias tables take that
//                room); paged rows are gathered page by page through the
//                block table.
//   warp 9       tcgen05 issuer.  Per key tile j and block b:
//                  S_b = Q_b K_j^T        (SS MMA into TMEM columns of S_b)
//                  O_b += P_b V_j         (TS MMA: P_b read from TMEM)
//                in the order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so the
//                tensor core works on one block while the other block's
//                softmax runs.  P_b V_j goes in two halves of 64 keys: the
//                first starts as soon as the softmax has written P for keys
//                0..63, while it still computes the rest.
//   warps 0..3,  softmax of block 0 / block 1: thread r owns row r (TMEM lane
//   4..7         r).  It reads its S row, applies qkScale, the ALiBi bias and
//                the causal / prefix-offset rule in registers (the mask is
//                never materialised), updates the running max and sum, rescales
//                O_b in TMEM only when the max grew by more than 2^8, and writes
//                P_b (16-bit, or fp32 for tf32) over S_b in TMEM.  At the end it
//                normalises O_b and stores it.
//
// Key tiles wholly above the prefix-shifted causal diagonal, or past the
// sequence's kvSeqLen, are never visited: the host gives each block the number
// of tiles up to its last allowed key.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace ala {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

template <typename T>
struct ElemFmt;
template <>
struct ElemFmt<__half> {
  static constexpr uint32_t fmt = 0;
};
template <>
struct ElemFmt<__nv_bfloat16> {
  static constexpr uint32_t fmt = 1;
};
template <>
struct ElemFmt<float> {
  static constexpr uint32_t fmt = 2;  // tf32 tensor-core inputs
};

// SQ: the instance carries the per-warp tables of the sqrt-ALiBi bias (maskType 4).  Their 10 KB take the
// room of a third V slot, so the other mask types run on an instance with a 3-deep V ring: a K or V tile
// arrives ~5000 cycles after its TMA load is issued, and two slots leave the MMA warp waiting for it.
template <typename T, int D, bool SQ>
struct Cfg {
  static constexpr int ES = sizeof(T);
  static constexpr int AW = 128 / ES;    // elements in one 128-byte swizzled row
  static constexpr int UK = 32 / ES;     // K extent of one MMA instruction
  static constexpr int BLK = 128 * 128;  // bytes of one 128-row x 128-byte swizzle column block
  static constexpr int NSK = 2;           // K ring depth
  static constexpr int NSV = SQ ? 2 : 3;  // V ring depth
  static constexpr int Q_BYTES = 128 * D * ES;
  static constexpr int KV_BYTES = 128 * D * ES;
  static constexpr int TBL_FLOATS = 160;  // per-warp sqrt-bias table: lane - column + 127 in [0, 159)
  static constexpr int TBL_BYTES = SQ ? 8 * 2 * TBL_FLOATS * 4 : 0;
  // q_full, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], and per block s_full, p_full, pv_done, o_done,
  // p_lo; fin, q_empty
  static constexpr int N_BARS = 1 + 2 * NSK + 2 * NSV + 2 * 5 + 2;
  static constexpr int SMEM = 1024 + 2 * Q_BYTES + (NSK + NSV) * KV_BYTES + TBL_BYTES + N_BARS * 8 + 16;
  static constexpr uint32_t IDESC_QK = instr_desc(ElemFmt<T>::fmt, false, false, 128, 128);
  static constexpr uint32_t IDESC_PV = instr_desc(ElemFmt<T>::fmt, false, true, 128, D);
  static constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D, 256+2D)
  static_assert(D % AW == 0, "head size must fill whole swizzle rows");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "tensor memory budget");
};

// One 32-byte store (address 32-byte aligned): whole sectors, half the instructions of 16-byte stores.
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                             uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2), "r"(a3),
               "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

// One 16-byte store (address 16-byte aligned): rows of a 16-bit head size that is an odd multiple of 8.
__device__ __forceinline__ void st_global_v4(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2), "r"(a3) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// P = 2^(u) for one row's 128 scores, u = x*scale - m taken a pair of columns at a
// time with packed f32x2 arithmetic; writes P over S in TMEM (16-bit pairs, or
// fp32 for tf32) and returns the row sum.  Masked keys hold -inf, which ex2 maps
// to exactly 0.
template <typename T>
__device__ __forceinline__ float exp_rows(const float (&x)[128], uint64_t scale2, uint64_t negm2, uint32_t s_col,
                                          uint64_t* p_lo) {
  constexpr bool kHalf = sizeof(T) == 2;
  constexpr int CHUNK = kHalf ? 64 : 32;  // columns per 32-register TMEM store
  uint64_t acc[4] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
#pragma unroll
  for (int h = 0; h < 128 / CHUNK; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int cc = 0; cc < CHUNK / 2; ++cc) {
      const int c0 = h * CHUNK + 2 * cc;
      float e0, e1;
      f2unpack(fma_x2(f2pack(x[c0], x[c0 + 1]), scale2, negm2), e0, e1);
      e0 = fast_exp2(e0);
      e1 = fast_exp2(e1);
      acc[cc & 3] = add_x2(acc[cc & 3], f2pack(e0, e1));
      if constexpr (kHalf) {
        pk[cc] = pack2(e0, e1, (T*)nullptr);
      } else {
        pk[2 * cc] = __float_as_uint(e0);
        pk[2 * cc + 1] = __float_as_uint(e1);
      }
    }
    tmem_st32(s_col + h * 32, pk);
    if (h == 128 / CHUNK / 2 - 1) {
      // P of keys 0..63 is in place: the first half of P*V may start while the rest is computed
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_lo);
    }
  }
  const uint64_t a = add_x2(add_x2(acc[0], acc[1]), add_x2(acc[2], acc[3]));
  float s0, s1;
  f2unpack(a, s0, s1);
  return s0 + s1;
}

template <typename T, int D>
__device__ __forceinline__ void load_kv_tile(const CUtensorMap* map, uint8_t* dst, uint64_t* full, int j,
                                             const SeqInfo& si, const PrefillParams& p, const int32_t* bt,
                                             int n_pages, int kvh, bool leader) {
  using C = Cfg<T, D, false>;
  const bool paged = bt != nullptr;
  const int bs = p.block_size;
  const int box_rows = paged ? p.kv_box_rows : 128;  // paged: every box lies inside one page
  const int j0 = j * 128;
  for (int r0 = 0; r0 < 128; r0 += box_rows) {
    // contiguous rows, or the page's row through the block table (past the last page: zero fill)
    const int row = paged ? paged_row(bt, j0 + r0, bs, n_pages, p.oob_row, p.status) : si.cu_kv + j0 + r0;
    if (leader) {
#pragma unroll
      for (int cb = 0; cb < D / C::AW; ++cb) tma_load_3d(dst + cb * C::BLK + r0 * 128, map, full, cb * C::AW, kvh, row);
    }
  }
}

template <typename T, int D, bool SQ>
__global__ void __launch_bounds__(384, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = Cfg<T, D, SQ>;
  constexpr int NSK = C::NSK, NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                        // [2][Q_BYTES]
  uint8_t* sK = sQ + 2 * C::Q_BYTES;         // [NSK][KV_BYTES]
  uint8_t* sV = sK + NSK * C::KV_BYTES;      // [NSV][KV_BYTES]
  float* sTbl = reinterpret_cast<float*>(sV + NSV * C::KV_BYTES);  // SQ: [8 warps][2][TBL_FLOATS]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sTbl) + C::TBL_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;          // [NSK]
  uint64_t* k_empty = k_full + NSK;     // [NSK]
  uint64_t* v_full = k_empty + NSK;     // [NSV]
  uint64_t* v_empty = v_full + NSV;     // [NSV]
  uint64_t* s_full = v_empty + NSV;     // [2] per block
  uint64_t* p_full = s_full + 2;        // [2] per block: P of keys 64..127 written (all of P)
  uint64_t* pv_done = p_full + 2;       // [2] per block
  uint64_t* o_done = pv_done + 2;       // [2] per block
  uint64_t* p_lo = o_done + 2;          // [2] per block: P of keys 0..63 written
  uint64_t* fin = p_lo + 2;
  uint64_t* q_empty = fin + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::N_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // this CTA's work units: a host-balanced list (persistent grid), or unit blockIdx.x alone
  const int u_begin = p.cta_offsets ? p.cta_offsets[blockIdx.x] : blockIdx.x;
  const int u_end = p.cta_offsets ? p.cta_offsets[blockIdx.x + 1] : blockIdx.x + 1;
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 128);
      mbar_init(p_lo + s, 128);
      mbar_init(pv_done + s, 1);
      mbar_init(o_done + s, 1);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Barrier phases run on across units: the K and V rings by a global tile counter g (slot g % depth,
  // phase g / depth), the per-block S/P/PV barriers by each block's tile counter, q_full / q_empty and
  // o_done by unit counters.
  //
  // register split: the softmax warpgroups take 216 per thread, warps 8..11 keep 72
  // (256*216 + 128*72 = 64512 = 384*168, all the registers the block is launched with)
  if (warp >= 8) {
    regs_decrease<72>();
    if (warp == 8 || warp == 10) {
      // ------------------------------------------------------------ producers
      // warp 8 loads the K tiles and each unit's Q tiles, warp 10 the V tiles, so a K load never waits
      // behind a V slot.  Each walks the schedule (warp-uniform values); one elected lane issues the copies.
      const bool is_k = warp == 8;
      const int depth = is_k ? NSK : NSV;
      uint8_t* ring = is_k ? sK : sV;
      uint64_t* full_bar = is_k ? k_full : v_full;
      uint64_t* empty_bar = is_k ? k_empty : v_empty;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(map);
        if (is_k) tma_prefetch_desc(&tmQ);
      }
      bool ok = true;
      uint32_t kv_iter = 0;  // K/V tiles loaded so far (all units)
      uint32_t issued = 0;   // loads this warp issued
      int q_loads = 0;
      for (int ui = u_begin; ui < u_end && ok; ++ui) {
        const PrefillUnit u = p.units[ui];
        const SeqInfo si = p.seqs[u.b];
        const int nb = u.n_blocks;
        const int nmax = (nb > 1 && u.n_tiles[1] > u.n_tiles[0]) ? u.n_tiles[1] : u.n_tiles[0];
        const int kvh = u.head[0] / p.group;
        const int32_t* bt = p.block_tables ? p.block_tables + (size_t)u.b * p.max_blocks : nullptr;
        const int n_pages = bt ? (si.kv_len + p.block_size - 1) / p.block_size : 0;
        for (int j = 0; j < nmax && ok; ++j) {
          const uint32_t g = kv_iter + j;
          const int s = g % depth;
          if (g >= (uint32_t)depth &&
              !__all_sync(0xffffffffu, mbar_wait(empty_bar + s, ((g / depth) - 1) & 1, status,
                                                 is_k ? kDevTimeoutKEmpty : kDevTimeoutVEmpty))) {
            ok = false;
            break;
          }
          if (leader) mbar_expect_tx(full_bar + s, C::KV_BYTES);
          load_kv_tile<T, D>(map, ring + s * C::KV_BYTES, full_bar + s, j, si, p, bt, n_pages, kvh, leader);
          issued = g + 1;
          if (is_k && j == 0) {
            // Q after the unit's first K tile, so both latencies overlap; the Q buffers are free
            // once the previous unit's last QK has finished
            if (q_loads > 0 && !__all_sync(0xffffffffu, mbar_wait(q_empty, (q_loads - 1) & 1, status, kDevTimeoutQ))) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_expect_tx(q_full, nb * C::Q_BYTES);
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                if (b >= nb) break;
#pragma unroll
                for (int cb = 0; cb < D / C::AW; ++cb)
                  tma_load_3d(sQ + b * C::Q_BYTES + cb * C::BLK, &tmQ, q_full, cb * C::AW, b ? u.head[1] : u.head[0],
                              si.cu_q + (b ? u.q0[1] : u.q0[0]));
              }
            }
            ++q_loads;
          }
        }
        kv_iter += nmax;
      }
      // never leave the CTA while loads this warp issued are still landing in shared memory
      for (uint32_t g = issued >= (uint32_t)depth ? issued - depth : 0; g < issued; ++g)
        mbar_wait(full_bar + (g % depth), (g / depth) & 1, status, is_k ? kDevTimeoutKFull : kDevTimeoutVFull);
      if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1, status, kDevTimeoutQ);
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      // the whole warp walks the schedule with warp-uniform descriptors; one elected lane issues
      const bool leader = elect_one();
      // base shared-memory descriptors; a K step adds its byte offset >> 4 to the start-address field
      const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_addr(sK), 16, 1024);
      // V is the MN-major operand: 16-bit types use the 16-byte-chunk swizzle (8-row atoms),
      // tf32 the 32-byte-chunk swizzle (4-row atoms), matching how the V tensor map loads it
      const uint64_t dv = C::ES == 4 ? smem_desc(smem_addr(sV), C::BLK, 512, 1) : smem_desc(smem_addr(sV), C::BLK, 1024, 2);
      constexpr uint64_t kQStep = C::Q_BYTES >> 4, kKVStep = C::KV_BYTES >> 4;
      auto issue_qk = [&](int b, int s) {
        if (leader) {
          const uint64_t a0 = dq + b * kQStep, b0 = dk + s * kKVStep;
#pragma unroll
          for (int kk = 0; kk < D / C::UK; ++kk) {
            const int ke = kk * C::UK;
            const uint64_t off = ((ke / C::AW) * C::BLK + (ke % C::AW) * C::ES) >> 4;
            mma_ss(tmem + b * 128, a0 + off, b0 + off, C::IDESC_QK, kk > 0, C::ES == 4);
          }
        }
      };
      auto issue_pv = [&](int b, int s, bool acc, int half) {
        if (leader) {
          const uint64_t v0 = dv + s * kKVStep;
#pragma unroll
          for (int kk = half * 64 / C::UK; kk < (half + 1) * 64 / C::UK; ++kk) {
            // P_b in TMEM over S_b: 8 columns per K step (two 16-bit values per column, or 8 tf32)
            mma_ts(tmem + 256 + b * D, tmem + b * 128 + kk * 8, v0 + ((kk * C::UK * 128) >> 4), C::IDESC_PV,
                   (acc || kk > 0) ? 1u : 0u, C::ES == 4);
          }
        }
      };
      auto commit = [&](uint64_t* bar) {
        if (leader) mma_commit(bar);
      };
      auto wait_all = [&](uint64_t* bar, uint32_t parity, int code) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, code));
      };
      bool ok = true;
      uint32_t kv_iter = 0;
      uint32_t sp0 = 0, sp1 = 0;  // tiles block 0 / 1 processed in earlier units
      for (int ui = u_begin; ui < u_end && ok; ++ui) {
        const int it = ui - u_begin;
        const PrefillUnit u = p.units[ui];
        const int nb = u.n_blocks;
        const int n0 = u.n_tiles[0];
        const int n1 = nb > 1 ? u.n_tiles[1] : 0;
        const int nmax = n0 > n1 ? n0 : n1;
        if (!wait_all(q_full, it & 1, kDevTimeoutQ) ||
            !wait_all(k_full + (kv_iter % NSK), (kv_iter / NSK) & 1, kDevTimeoutKFull)) {
          ok = false;
          break;
        }
        for (int b = 0; b < nb; ++b) {
          // S_b / P_b are free once the previous unit's last P_b * V has completed
          const uint32_t spb = b ? sp1 : sp0;
          if (spb > 0 && !wait_all(pv_done + b, (spb - 1) & 1, kDevTimeoutODone)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_qk(b, kv_iter % NSK);
          commit(s_full + b);
        }
        if (!ok) break;
        commit(k_empty + (kv_iter % NSK));
        if (nmax == 1) commit(q_empty);
        for (int j = 0; j < nmax && ok; ++j) {
          const uint32_t g = kv_iter + j;
          const int sv = g % NSV;  // V ring slot of tile j
          bool v_ready = false;
          for (int b = 0; b < nb && ok; ++b) {
            const int nbt = b == 0 ? n0 : n1;
            if (j >= nbt) continue;
            const uint32_t ph = (b ? sp1 : sp0) + j;  // this block's barrier phase for tile j
            if (!wait_all(p_lo + b, ph & 1, kDevTimeoutPFull)) {
              ok = false;
              break;
            }
            if (!v_ready && !wait_all(v_full + sv, (g / NSV) & 1, kDevTimeoutVFull)) {
              ok = false;
              break;
            }
            v_ready = true;
            tc_fence_after();
            issue_pv(b, sv, j > 0, 0);  // keys 0..63
            if (!wait_all(p_full + b, ph & 1, kDevTimeoutPFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(b, sv, true, 1);   // keys 64..127
            commit(pv_done + b);
            const bool last_pv = (b == nb - 1) || (j >= n1);
            if (last_pv) commit(v_empty + sv);
            if (j == nbt - 1) {
              commit(o_done + b);
              continue;
            }
            // next key tile for this block; S_b / P_b are reused once P_b(j) * V has completed
            const uint32_t g1 = g + 1;
            const int s1 = g1 % NSK;  // K ring slot of tile j + 1
            const bool first_qk = (b == 0) || (j + 1 >= n0);
            if (first_qk && !wait_all(k_full + s1, (g1 / NSK) & 1, kDevTimeoutKFull)) {
              ok = false;
              break;
            }
            if (!wait_all(pv_done + b, ph & 1, kDevTimeoutODone)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(b, s1);
            commit(s_full + b);
            const bool last_qk = (b == nb - 1) || (j + 1 >= n1);
            if (last_qk) {
              commit(k_empty + s1);
              if (j + 1 == nmax - 1) commit(q_empty);  // the unit's last QK: Q buffers free
            }
          }
        }
        sp0 += n0;
        sp1 += n1;
        kv_iter += nmax;
      }
      // all tensor-core work this thread issued has finished before TMEM is released
      commit(fin);
      wait_all(fin, 0, kDevTimeoutFinal);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue of block b
    regs_increase<216>();
    const int b = warp >> 2;
    const int r = threadIdx.x & 127;  // query row in the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + b * 128;
    const uint32_t o_col = tmem + lane_base + 256 + b * D;
    const int mt = p.mask_type;
    const bool alibi = (mt == 3 || mt == 4 || mt == 5);
    const float scale = p.scale_log2;
    const bool raw_max = !alibi && scale > 0.f;  // max of the raw scores, scale folded into the exponent
    float* tbl = sTbl + warp * 2 * C::TBL_FLOATS;
    uint32_t sp = 0;  // tiles this block processed in earlier units (barrier phases)
    uint32_t up = 0;  // units this block took part in (o_done phases)
    bool ok = true;
    for (int ui = u_begin; ui < u_end && ok; ++ui) {
      const PrefillUnit u = p.units[ui];
      if (b >= u.n_blocks) continue;
      const SeqInfo si = p.seqs[u.b];
      const int n = b ? u.n_tiles[1] : u.n_tiles[0];
      const int head = b ? u.head[1] : u.head[0];
      const int q0 = b ? u.q0[1] : u.q0[0];
      const int qi = q0 + r;
      const bool row_valid = qi < si.seq_len;
      const int off = si.kv_len - si.seq_len;
      const int iabs = qi + off;
      const float slope = alibi ? p.slopes[head] : 0.f;
      const float slope_log2 = slope * kLog2e;
      const int last_key = (mt == 0) ? si.kv_len - 1 : min(iabs, si.kv_len - 1);
      const int iabs_w = q0 + (warp & 3) * 32 + off;  // iabs of the warp's first row
      float m_run = -INFINITY;  // running max in log2 units (the one P is computed against)
      float l_run = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t ph = sp + j;
        const int j0 = j * 128;
        float* t = tbl + (ph & 1) * C::TBL_FLOATS;
        if (SQ && mt == 4) {
          // -slope*log2(e)*sqrt(distance) for distance = iabs_w + k - 127 - j0, k = lane - column + 127
          for (int k = lane; k < C::TBL_FLOATS; k += 32) {
            const float dist = static_cast<float>(iabs_w - j0 + k - 127);
            t[k] = -slope_log2 * sqrtf(fmaxf(dist, 0.f));
          }
          __syncwarp();
        }
        ok = __all_sync(0xffffffffu, mbar_wait(s_full + b, ph & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        tc_fence_after();
        float x[128];
        {
          uint32_t sr[4][32];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(s_col + c4 * 32, sr[c4]);
          tmem_ld_wait();  // one wait for all four loads
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        const int lim = last_key - j0;  // columns c <= lim are allowed
        if (mt == 3 || mt == 5) {
          // right- and left-aligned bias differ by a per-row constant; both use (j - iabs)
          const float b0 = slope_log2 * static_cast<float>(j0 - iabs);
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = fmaf(x[c], scale, fmaf(slope_log2, static_cast<float>(c), b0));
        } else if (SQ && mt == 4) {
          const float* tl = t + lane + 127;
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = fmaf(x[c], scale, tl[-c]);
        } else if (!raw_max) {
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] *= scale;
        }
        if (lim < 127) {
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
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
        const float m_base = (m_run == -INFINITY) ? 0.f : m_run;
        // O_b is quiescent here: P_b(j-1) * V completed before S_b(j) was written
        if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c32 = 0; c32 < D / 32; ++c32) {
            uint32_t regs[32];
            tmem_ld32(o_col + c32 * 32, regs);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) regs[c] = __float_as_uint(__uint_as_float(regs[c]) * alpha);
            tmem_st32(o_col + c32 * 32, regs);
          }
        }
        // P = 2^(x*scale - m) (raw scores) or 2^(x - m) (biased scores), written over S in TMEM
        const uint64_t scale2 = f2pack(raw_max ? scale : 1.f, raw_max ? scale : 1.f);
        const uint64_t negm2 = f2pack(-m_base, -m_base);
        const float row_sum = exp_rows<T>(x, scale2, negm2, s_col, p_lo + b);
        l_run = l_run * alpha + row_sum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + b);
      }
      sp += n;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done + b, up & 1, status, kDevTimeoutODone));
      ++up;
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const int d_out = p.d_out;  // columns d_out..D-1 hold zeros (zero-filled Q, K and V dimensions)
      const bool wide_rows = d_out % 16 == 0;  // 16-bit rows 32-byte aligned: 32-byte stores
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(si.cu_q + qi) * p.heads + head) * d_out;
      uint32_t orr[D / 32][32];
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) tmem_ld32(o_col + c32 * 32, orr[c32]);
      tmem_ld_wait();  // one wait for all loads of the row; the next unit's P_b * V may then overwrite O_b
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) {
        const uint32_t(&regs)[32] = orr[c32];
        if (row_valid) {
          // rows are d_out * element size apart, a multiple of 32 bytes: every 32-byte store is aligned
          if constexpr (C::ES == 2) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack2(__uint_as_float(regs[2 * i]) * inv_l, __uint_as_float(regs[2 * i + 1]) * inv_l, (T*)nullptr);
            if (wide_rows) {
#pragma unroll
              for (int v8 = 0; v8 < 2; ++v8) {
                if (c32 * 32 + v8 * 16 >= d_out) break;
                st_global_v8(orow + c32 * 32 + v8 * 16, w[8 * v8], w[8 * v8 + 1], w[8 * v8 + 2], w[8 * v8 + 3],
                             w[8 * v8 + 4], w[8 * v8 + 5], w[8 * v8 + 6], w[8 * v8 + 7]);
              }
            } else {
              // rows 16 bytes apart only (d_out an odd multiple of 8): 16-byte stores
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                if (c32 * 32 + v4 * 8 >= d_out) break;
                st_global_v4(orow + c32 * 32 + v4 * 8, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
              }
            }
          } else {
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {
              if (c32 * 32 + v8 * 8 >= d_out) break;
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(__uint_as_float(regs[v8 * 8 + i]) * inv_l);
              st_global_v8(reinterpret_cast<float*>(orow) + c32 * 32 + v8 * 8, w[0], w[1], w[2], w[3], w[4], w[5],
                           w[6], w[7]);
            }
          }
        }
      }
      if (row_valid && p.lse) {
        float lse = (m_run == -INFINITY ? 0.f : m_run) * kLn2 + logf(l_run);
        if (mt == 5) lse += slope * static_cast<float>(iabs);  // left-aligned bias = right-aligned + slope*iabs
        p.lse[(size_t)(si.cu_q + qi) * p.heads + head] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <typename T, int D, bool SQ>
cudaError_t launch_instance(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const PrefillParams& p, cudaStream_t stream) {
  using C = Cfg<T, D, SQ>;
  // at least 120 KB so a second CTA never shares the SM (each CTA allocates all 512 TMEM columns)
  constexpr int kSmem = C::SMEM > 120 * 1024 ? C::SMEM : 120 * 1024;
  auto kern = prefill_kernel<T, D, SQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  if (p.n_ctas == 0) return cudaSuccess;
  kern<<<p.n_ctas, 384, kSmem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

// maskType 4 (sqrt ALiBi) runs on the instance with the bias tables, every other mask type on the one with
// the deeper V ring
template <typename T, int D>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const PrefillParams& p,
                   cudaStream_t stream) {
  return p.mask_type == 4 ? launch_instance<T, D, true>(tmQ, tmK, tmV, p, stream)
                          : launch_instance<T, D, false>(tmQ, tmK, tmV, p, stream);
}

}  // namespace

int prefill_kernel_d(int32_t dtype, int64_t d) {
  if (dtype == kBF16 || dtype == kF16) {
    if (d <= 0 || d % 8 != 0 || d > 256) return 0;
    return d <= 64 ? 64 : d <= 128 ? 128 : 256;
  }
  if (dtype == kF32) return (d > 0 && d % 8 == 0 && d <= 64) ? 64 : 0;
  return 0;
}

cudaError_t launch_prefill(int32_t dtype, int32_t d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const PrefillParams& p, cudaStream_t stream) {
  if (d == 256) return launch_prefill_d256(dtype, tmQ, tmK, tmV, p, stream);
  if (dtype == kBF16) {
    if (d == 128) return launch<__nv_bfloat16, 128>(tmQ, tmK, tmV, p, stream);
    if (d == 64) return launch<__nv_bfloat16, 64>(tmQ, tmK, tmV, p, stream);
  } else if (dtype == kF16) {
    if (d == 128) return launch<__half, 128>(tmQ, tmK, tmV, p, stream);
    if (d == 64) return launch<__half, 64>(tmQ, tmK, tmV, p, stream);
  } else if (dtype == kF32) {
    if (d == 64) return launch<float, 64>(tmQ, tmK, tmV, p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ala
