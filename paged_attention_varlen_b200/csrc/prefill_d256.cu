// prefill_d256.cu -- the prefill kernel for head sizes 136..256 (kernel head
// size D = 256), 16-bit types, no mask or the causal rule with the prefix offset
// kvSeqLen - seqLen.  The pages bound headSize only for ALiBi compressed masks
// (at most 128: the compressed-mask page, constraints), so head sizes above 128
// take the causal rule or no mask.
//
// O of one 128-row block takes 256 of the 512 tensor-memory columns, so a CTA
// computes one block of 128 query rows (not two, as the D <= 128 kernel does)
// and keeps four S buffers of 64 keys in the other half:
//
//   TMEM columns [64 s, 64 s + 64) S[s] for s = 0..3, [256, 512) O
//   shared memory Q 64 KB, a K ring of 3 x 32 KB and a V ring of 2 x 32 KB
//                (64-key tiles)
//
//   warps 4, 6   TMA producers: warp 4 the K tiles and each unit's Q tile,
//                warp 6 the V tiles; paged rows are gathered page by page
//                through the block table.
//   warp 5       tcgen05 issuer.  Per key tile j:
//                  S[j%4] = Q K_j^T       (SS MMA, M = 128, N = 64)
//                  O     += P V_j         (TS MMA, N = 256: P read from TMEM over S[j%4])
//                in the order PV(j), QK(j+2).  QK(j+2) refills the buffer of
//                tile j-2, whose P V completed well before, so the issuer never
//                waits for the P V it has just issued and the tensor pipe gets
//                PV(j) and QK(j+2) back to back while the softmax works on
//                tile j+1.
//   warps 0..3   softmax: thread r owns row r (TMEM lane r).  It reads its S
//                row, applies qkScale and the causal / prefix-offset rule in
//                registers, updates the running max and sum, rescales O in TMEM
//                only when the max grew by more than 2^8, and writes P (16-bit)
//                over its S buffer.  At the end it normalises O and stores it.
//
// Key tiles wholly above the prefix-shifted causal diagonal, or past the
// sequence's kvSeqLen, are never visited: the host gives each block the number
// of 64-key tiles up to its last allowed key.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace ala {

namespace {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr int D = 256;                     // kernel head size
constexpr int KT = 64;                     // keys per tile
constexpr int AW = 64;                     // 16-bit elements in one 128-byte swizzled row
constexpr int UK = 16;                     // K extent of one MMA instruction (16-bit types)
constexpr int BLK_Q = 128 * 128;           // bytes of one 128-row x 128-byte swizzle column block
constexpr int BLK_KV = KT * 128;           // bytes of one 64-key x 128-byte swizzle column block
constexpr int NSK = 3;                     // K ring depth
constexpr int NSV = 2;                     // V ring depth
constexpr int NSB = 4;                     // S buffers in tensor memory
constexpr int Q_BYTES = 128 * D * 2;
constexpr int KV_BYTES = KT * D * 2;
// q_full, q_empty, fin, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full[NSB], p_full[NSB],
// pv_done[NSB], o_done
constexpr int N_BARS = 3 + 2 * NSK + 2 * NSV + 3 * NSB + 1;
constexpr int SMEM = 1024 + Q_BYTES + (NSK + NSV) * KV_BYTES + N_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 256;
constexpr int kThreads = 224;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(O_COL + D <= TMEM_COLS && NSB * KT <= O_COL, "tensor memory budget");

template <typename T>
struct Fmt;
template <>
struct Fmt<__half> {
  static constexpr uint32_t v = 0;
};
template <>
struct Fmt<__nv_bfloat16> {
  static constexpr uint32_t v = 1;
};

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One 16-byte store (address 16-byte aligned): rows of a 16-bit head size that is an odd multiple of 8.
__device__ __forceinline__ void st_global_v4(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2), "r"(a3) : "memory");
}

// One 32-byte store (address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// P = 2^(x*scale - m) for one row's 64 scores, a pair of columns at a time with packed f32x2 arithmetic;
// writes P (16-bit pairs) over S in TMEM and returns the row sum.  Masked keys hold -inf, which ex2 maps
// to exactly 0.
template <typename T>
__device__ __forceinline__ float exp_row(const float (&x)[KT], uint64_t scale2, uint64_t negm2, uint32_t s_col) {
  uint64_t acc[4] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
  uint32_t pk[32];
#pragma unroll
  for (int cc = 0; cc < KT / 2; ++cc) {
    float e0, e1;
    f2unpack(fma_x2(f2pack(x[2 * cc], x[2 * cc + 1]), scale2, negm2), e0, e1);
    e0 = fast_exp2(e0);
    e1 = fast_exp2(e1);
    acc[cc & 3] = add_x2(acc[cc & 3], f2pack(e0, e1));
    pk[cc] = pack2(e0, e1, (T*)nullptr);
  }
  tmem_st32(s_col, pk);
  const uint64_t a = add_x2(add_x2(acc[0], acc[1]), add_x2(acc[2], acc[3]));
  float s0, s1;
  f2unpack(a, s0, s1);
  return s0 + s1;
}

__device__ __forceinline__ void load_kv_tile(const CUtensorMap* map, uint8_t* dst, uint64_t* full, int j,
                                             const SeqInfo& si, const PrefillParams& p, const int32_t* bt,
                                             int n_pages, int kvh, bool leader) {
  const bool paged = bt != nullptr;
  const int bs = p.block_size;
  const int box_rows = paged ? p.kv_box_rows : KT;  // paged: every box lies inside one page
  const int j0 = j * KT;
  for (int r0 = 0; r0 < KT; r0 += box_rows) {
    // contiguous rows, or the page's row through the block table (past the last page: zero fill)
    const int row = paged ? paged_row(bt, j0 + r0, bs, n_pages, p.oob_row, p.status) : si.cu_kv + j0 + r0;
    if (leader) {
#pragma unroll
      for (int cb = 0; cb < D / AW; ++cb) tma_load_3d(dst + cb * BLK_KV + r0 * 128, map, full, cb * AW, kvh, row);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Q_BYTES;  // [NSK][KV_BYTES]
  uint8_t* sV = sK + NSK * KV_BYTES;  // [NSV][KV_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NSV * KV_BYTES);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* fin = bars + 2;
  uint64_t* k_full = bars + 3;         // [NSK]
  uint64_t* k_empty = k_full + NSK;    // [NSK]
  uint64_t* v_full = k_empty + NSK;    // [NSV]
  uint64_t* v_empty = v_full + NSV;    // [NSV]
  uint64_t* s_full = v_empty + NSV;    // [NSB] S[s] computed
  uint64_t* p_full = s_full + NSB;     // [NSB] P written over S[s]
  uint64_t* pv_done = p_full + NSB;    // [NSB] the P V of S[s]'s tile completed
  uint64_t* o_done = pv_done + NSB;    // the unit's last P V completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + N_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int u_begin = p.cta_offsets ? p.cta_offsets[blockIdx.x] : blockIdx.x;
  const int u_end = p.cta_offsets ? p.cta_offsets[blockIdx.x + 1] : blockIdx.x + 1;
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(fin, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < NSB; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 128);
      mbar_init(pv_done + s, 1);
    }
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  (void)lane;

  // Barrier phases run on across units: the K and V rings by a global tile counter g (slot g % depth,
  // phase g / depth), the S/P/PV barriers by the same counter (buffer g % NSB, phase g / NSB), q_full /
  // q_empty and o_done by unit counters.
  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ producers
    // warp 4 loads K (3-deep ring) and each unit's Q; warp 6 loads V (2-deep ring).  Two warps, so a K
    // load never waits behind a V slot: K(j+3) can start as soon as QK(j) has completed.
    const bool is_k = warp == 4;
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
    uint32_t kv_iter = 0;
    uint32_t issued = 0;
    int q_loads = 0;
    for (int ui = u_begin; ui < u_end && ok; ++ui) {
      const PrefillUnit u = p.units[ui];
      const SeqInfo si = p.seqs[u.b];
      const int n = u.n_tiles[0];
      const int kvh = u.head[0] / p.group;
      const int32_t* bt = p.block_tables ? p.block_tables + (size_t)u.b * p.max_blocks : nullptr;
      const int n_pages = bt ? (si.kv_len + p.block_size - 1) / p.block_size : 0;
      for (int j = 0; j < n && ok; ++j) {
        const uint32_t g = kv_iter + j;
        const int s = g % depth;
        if (g >= (uint32_t)depth &&
            !__all_sync(0xffffffffu, mbar_wait(empty_bar + s, ((g / depth) - 1) & 1, status,
                                               is_k ? kDevTimeoutKEmpty : kDevTimeoutVEmpty))) {
          ok = false;
          break;
        }
        if (leader) mbar_expect_tx(full_bar + s, KV_BYTES);
        load_kv_tile(map, ring + s * KV_BYTES, full_bar + s, j, si, p, bt, n_pages, kvh, leader);
        issued = g + 1;
        if (is_k && j == 0) {
          // Q after the unit's first K tile, so both latencies overlap; the Q buffer is free once the
          // previous unit's last QK has finished
          if (q_loads > 0 && !__all_sync(0xffffffffu, mbar_wait(q_empty, (q_loads - 1) & 1, status, kDevTimeoutQ))) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_expect_tx(q_full, Q_BYTES);
#pragma unroll
            for (int cb = 0; cb < D / AW; ++cb)
              tma_load_3d(sQ + cb * BLK_Q, &tmQ, q_full, cb * AW, u.head[0], si.cu_q + u.q0[0]);
          }
          ++q_loads;
        }
      }
      kv_iter += n;
    }
    // never leave the CTA while loads this warp issued are still landing in shared memory
    for (uint32_t g = issued >= (uint32_t)depth ? issued - depth : 0; g < issued; ++g)
      mbar_wait(full_bar + (g % depth), (g / depth) & 1, status, is_k ? kDevTimeoutKFull : kDevTimeoutVFull);
    if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1, status, kDevTimeoutQ);
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
    const uint64_t dk = smem_desc_sw128(smem_addr(sK), 16, 1024);
    // V is the MN-major operand: 16-byte-chunk swizzle (8-row atoms), as the V tensor map loads it
    const uint64_t dv = smem_desc(smem_addr(sV), BLK_KV, 1024, 2);
    constexpr uint64_t kKVStep = KV_BYTES >> 4;
    constexpr uint32_t kIdescQK = instr_desc(Fmt<T>::v, false, false, 128, KT);
    constexpr uint32_t kIdescPV = instr_desc(Fmt<T>::v, false, true, 128, D);
    auto wait_all = [&](uint64_t* bar, uint32_t parity, int code) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, code));
    };
    // S[g % NSB] = Q K^T of the tile in K ring slot g % NSK
    auto issue_qk = [&](uint32_t g) {
      if (leader) {
        const uint64_t b0 = dk + (g % NSK) * kKVStep;
#pragma unroll
        for (int kk = 0; kk < D / UK; ++kk) {
          const int ke = kk * UK;
          const uint64_t off_q = ((ke / AW) * BLK_Q + (ke % AW) * 2) >> 4;
          const uint64_t off_k = ((ke / AW) * BLK_KV + (ke % AW) * 2) >> 4;
          mma_ss(tmem + (g % NSB) * KT, dq + off_q, b0 + off_k, kIdescQK, kk > 0, false);
        }
        mma_commit(s_full + (g % NSB));
      }
    };
    // O (+)= P V, P in TMEM over S[g % NSB] (8 columns of packed 16-bit pairs per K step of 16 keys)
    auto issue_pv = [&](uint32_t g, bool acc) {
      if (leader) {
        const uint64_t v0 = dv + (g % NSV) * kKVStep;
#pragma unroll
        for (int kk = 0; kk < KT / UK; ++kk)
          mma_ts(tmem + O_COL, tmem + (g % NSB) * KT + kk * 8, v0 + ((kk * UK * 128) >> 4), kIdescPV,
                 (acc || kk > 0) ? 1u : 0u, false);
        mma_commit(pv_done + (g % NSB));
      }
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) mma_commit(bar);
    };
    // QK of tile g: its K tile is loaded and its S buffer is free (the P V of tile g - NSB has completed)
    auto qk_ready = [&](uint32_t g) {
      if (!wait_all(k_full + (g % NSK), (g / NSK) & 1, kDevTimeoutKFull)) return false;
      if (g >= NSB && !wait_all(pv_done + (g % NSB), ((g / NSB) - 1) & 1, kDevTimeoutODone)) return false;
      tc_fence_after();
      return true;
    };
    bool ok = true;
    uint32_t kv_iter = 0;
    for (int ui = u_begin; ui < u_end && ok; ++ui) {
      const int it = ui - u_begin;
      const int n = p.units[ui].n_tiles[0];
      if (!wait_all(q_full, it & 1, kDevTimeoutQ)) {
        ok = false;
        break;
      }
      // each QK releases its K slot; the unit's last one also the Q buffer
      auto qk = [&](int j) {
        if (!qk_ready(kv_iter + j)) return false;
        issue_qk(kv_iter + j);
        commit(k_empty + ((kv_iter + j) % NSK));
        if (j == n - 1) commit(q_empty);
        return true;
      };
      for (int j = 0; j < 2 && j < n && ok; ++j) ok = qk(j);
      for (int j = 0; j < n && ok; ++j) {
        const uint32_t g = kv_iter + j;
        if (!(ok = wait_all(v_full + (g % NSV), (g / NSV) & 1, kDevTimeoutVFull))) break;
        if (!(ok = wait_all(p_full + (g % NSB), (g / NSB) & 1, kDevTimeoutPFull))) break;
        tc_fence_after();
        issue_pv(g, j > 0);
        if (j == n - 1) commit(o_done);
        commit(v_empty + (g % NSV));
        if (j + 2 < n) ok = qk(j + 2);
      }
      kv_iter += n;
    }
    // all tensor-core work this thread issued has finished before TMEM is released
    commit(fin);
    wait_all(fin, 0, kDevTimeoutFinal);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = threadIdx.x;  // query row in the block == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_col = tmem + lane_base + O_COL;
    const bool causal = p.mask_type != 0;
    const float scale = p.scale_log2;
    const bool raw_max = scale > 0.f;  // max of the raw scores, scale folded into the exponent
    uint32_t tp = 0;                   // tiles processed in earlier units (barrier phases)
    uint32_t up = 0;                   // units processed (o_done phases)
    bool ok = true;
    for (int ui = u_begin; ui < u_end && ok; ++ui) {
      const PrefillUnit u = p.units[ui];
      const SeqInfo si = p.seqs[u.b];
      const int n = u.n_tiles[0];
      const int head = u.head[0];
      const int qi = u.q0[0] + r;
      const bool row_valid = qi < si.seq_len;
      const int iabs = qi + si.kv_len - si.seq_len;
      const int last_key = causal ? min(iabs, si.kv_len - 1) : si.kv_len - 1;
      float m_run = -INFINITY;  // running max in log2 units (the one P is computed against)
      float l_run = 0.f;
      for (int j = 0; j < n; ++j) {
        const uint32_t t = tp + j;
        const uint32_t s_col = tmem + lane_base + (t % NSB) * KT;
        const int j0 = j * KT;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full + (t % NSB), (t / NSB) & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        tc_fence_after();
        float x[KT];
        {
          uint32_t sr[2][32];
          tmem_ld32(s_col, sr[0]);
          tmem_ld32(s_col + 32, sr[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < KT; ++c) x[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        if (!raw_max) {
#pragma unroll
          for (int c = 0; c < KT; ++c) x[c] *= scale;
        }
        const int lim = last_key - j0;  // columns c <= lim are allowed
        if (lim < KT - 1) {
#pragma unroll
          for (int c = 0; c < KT; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < KT; c += 8) {
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
        if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O must hold P(j-1) V(j-1) before it is scaled; P(j) V cannot start before P(j) below
          ok = __all_sync(0xffffffffu,
                          mbar_wait(pv_done + ((t - 1) % NSB), ((t - 1) / NSB) & 1, status, kDevTimeoutODone));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c64 = 0; c64 < D / 64; ++c64) {
            uint32_t regs[2][32];
            tmem_ld32(o_col + c64 * 64, regs[0]);
            tmem_ld32(o_col + c64 * 64 + 32, regs[1]);
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
              for (int c = 0; c < 32; ++c) regs[h][c] = __float_as_uint(__uint_as_float(regs[h][c]) * alpha);
              tmem_st32(o_col + c64 * 64 + h * 32, regs[h]);
            }
          }
        }
        const uint64_t scale2 = f2pack(raw_max ? scale : 1.f, raw_max ? scale : 1.f);
        const uint64_t negm2 = f2pack(-m_base, -m_base);
        const float row_sum = exp_row<T>(x, scale2, negm2, s_col);
        l_run = l_run * alpha + row_sum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + (t % NSB));
      }
      tp += n;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, up & 1, status, kDevTimeoutODone));
      ++up;
      if (!ok) break;
      tc_fence_after();
      // O is read before this thread arrives on the next unit's first P, so the next unit's first P V
      // (which overwrites O) cannot start before these loads have completed
      const float inv_l = 1.f / l_run;
      const int d_out = p.d_out;  // columns d_out..D-1 hold zeros (zero-filled Q, K and V dimensions)
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(si.cu_q + qi) * p.heads + head) * d_out;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t orr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(o_col + half * 128 + c * 32, orr[c]);
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v16 = 0; v16 < 8; ++v16) {
            const int col = half * 128 + v16 * 16;
            if (col >= d_out) break;
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              w[i] = pack2(__uint_as_float(orr[v16 >> 1][(v16 & 1) * 16 + 2 * i]) * inv_l,
                           __uint_as_float(orr[v16 >> 1][(v16 & 1) * 16 + 2 * i + 1]) * inv_l, (T*)nullptr);
            if (d_out % 16 == 0) {
              st_global_v8(orow + col, w);  // rows d_out * 2 bytes apart, a multiple of 32 bytes
            } else {
              // rows 16 bytes apart only (d_out an odd multiple of 8): 16-byte stores
              st_global_v4(orow + col, w[0], w[1], w[2], w[3]);
              if (col + 8 < d_out) st_global_v4(orow + col + 8, w[4], w[5], w[6], w[7]);
            }
          }
        }
      }
      if (row_valid && p.lse)
        p.lse[(size_t)(si.cu_q + qi) * p.heads + head] = (m_run == -INFINITY ? 0.f : m_run) * kLn2 + logf(l_run);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <typename T>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const PrefillParams& p,
                   cudaStream_t stream) {
  auto kern = prefill_d256_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  if (p.n_ctas == 0) return cudaSuccess;
  kern<<<p.n_ctas, kThreads, SMEM, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_d256(int32_t dtype, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                const PrefillParams& p, cudaStream_t stream) {
  if (dtype == kBF16) return launch<__nv_bfloat16>(tmQ, tmK, tmV, p, stream);
  if (dtype == kF16) return launch<__half>(tmQ, tmK, tmV, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ala
