// mla_pair.cu -- MLA decode (one query token per batch) with M = 128 rows per
// CTA, for sm_100a (ATB "MLA" page, definition and parameter table): per head,
// O = softmax(qkScale * [qNope;qRope] . [ctKV;kRope]^T) ctKV and the lse.
//
// A cluster of two CTAs serves the 128 heads of one token.  CTA r owns the
// latent dimensions [256r, 256r + 256): it keeps its half of qNope in tensor
// memory (the A operand of the QK MMAs), stages only its half of each ctKV
// tile, computes the QK partial over its dimensions (rank 0 adds qRope kRope),
// and accumulates the 256 output columns of its half.  The two partial score
// tiles are exchanged through distributed shared memory and added, so both
// CTAs run the same softmax on the full scores; each then multiplies P by its
// own half of the tile.  Compared with 64-row CTAs (mla.cu), every MMA has
// M = 128 and each CTA reads half of every cache row, so the tensor work per
// key and head halves and each CTA stages 36 KB per 64 keys instead of 72 KB.
//
// Tensor memory (512 columns, lane = row = head): qNope half at columns
// 0..127 (256 bf16 / fp16 values per row), two score buffers S0, S1 at
// 128..191 and 192..255 (P is written over the buffer once it is read), and
// the output half at 256..511.
//
//   warp 4      TMA producer (one thread): the CTA's half of each 64-key ctKV
//               tile, gathered through the block table (rank 0 also kRope and
//               qRope), three tiles ahead.
//   warp 5      tcgen05 issuer (one thread): S(j) = qNope_half ctKV_half^T
//               (+ qRope kRope^T on rank 0) into S[j & 1], O_half += P(j) V_half.
//   warps 0..3  softmax and epilogue, one row per thread.
//
// Key ranges are cut into lanes as in mla.cu (one cluster per lane and head
// group), and ranges that split a token are merged by lse at the end.
//
// Measured against the 64-row kernel on the bf16 decode workload (batch 64,
// 128 heads): 0.53 ms against 0.23 ms.  The 32 KB score exchange per tile
// through distributed shared memory takes ~4000 cycles (the SM-to-SM network
// moves ~8 bytes per clock per SM here), more than the tensor work the split
// saves, so the planner uses this kernel only when ALA_MLA_PAIR=1 is set.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <type_traits>

#include "internal.h"
#include "mla.h"
#include "ptx.cuh"

namespace ala {

namespace {

constexpr float kPLog2e = 1.4426950408889634f;
constexpr float kPLn2 = 0.6931471805599453f;
constexpr float kPRescale = 8.0f;           // raise the running max only when it grows by more than 2^8

constexpr int kPRows = 128;                 // rows per CTA: the 128 heads of a group
constexpr int kPKeys = 64;                  // keys per tile
constexpr int kPBlk = kPKeys * 128;         // one 64-column block of a tile: 64 keys x 128 B = 8 KB
constexpr int kPSlot = 5 * kPBlk;           // ctKV half (4 blocks) + kRope (rank 0): 40 KB
constexpr int kPStages = 3;
constexpr int kPQr = kPRows * 128;          // qRope rows of the group: 16 KB
constexpr int kPX = kPRows * kPKeys * 4;    // one partial score tile (fp32): 32 KB
// q_full, kv_full[3], kv_empty[3], s_full[2], p_full[2], pv_done[2], pv_last, x_full[2], x_empty[2], fin
constexpr int kPNBars = 1 + 2 * kPStages + 2 + 2 + 2 + 1 + 2 + 2 + 1;
constexpr int kPSmem = 1024 + kPQr + kPStages * kPSlot + 2 * kPX + kPNBars * 8 + 16;
static_assert(kPSmem <= 232448, "shared memory of one CTA");
constexpr uint32_t kPSCol = 128;            // S0 at 128, S1 at 192
constexpr uint32_t kPOCol = 256;
constexpr int kPPlannedSms = 148;
constexpr int kPMinLaneTiles = 4;
constexpr unsigned kPFull = 0xffffffffu;

struct PairPiece {
  int32_t b;         // batch (= its one query token)
  int32_t token0;
  int32_t kv_begin;  // first key of the range (a multiple of 64)
  int32_t n_tiles;
  int32_t last;      // last allowed key of the token
  int32_t part;      // partial slot, or -1: final output
  int32_t pad[2];
};

struct PairCombine {
  int32_t token;
  int32_t part_begin;
  int32_t n_parts;
  int32_t pad;
};

struct PairParams {
  const PairPiece* pieces;
  const int32_t* lane_off;  // [n_lanes + 1]
  const int32_t* block_tables;
  const uint8_t* q_nope;    // [tokens, heads, 512]
  const uint8_t* ct_kv;     // [rows, 512] (the L2 prefetch reads raw rows)
  const uint8_t* k_rope;    // [rows, 64]
  void* out;                // [tokens, heads, 512]
  float* lse;               // [tokens, heads] or null
  float* part_o;            // [parts, heads, 512]
  float* part_lse;          // [parts, heads]
  int* status;
  int32_t heads;
  int32_t groups;           // heads / 128
  int32_t max_blocks;
  int32_t block_size;
  int32_t oob_row;
  float scale_log2;
};

__device__ __forceinline__ uint32_t ppack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t ppack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The same shared-memory offset in the CTA of the cluster with rank `peer`.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(peer));
  return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4p(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// Arrive on an mbarrier of the peer CTA; orders this thread's earlier stores into the peer's memory.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

// Bounded wait on a local barrier that the peer CTA arrives on (acquire at cluster scope).  It polls
// (test_wait) rather than suspending: a suspended thread measured slow to wake on a remote arrival.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* status, int code) {
  const uint32_t a = smem_addr(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((it & 1023u) == 0) {  // the status word and the clock every 1024 polls
      const uint64_t now = global_timer_ns();
      if (it == 0) t0 = now;
      if (*status != 0) return false;
      if (now - t0 > ALA_WAIT_LIMIT_NS) {
        atomicCAS((int*)status, 0, code);
        return false;
      }
    }
  }
}

// Every thread of both CTAs (all arrive, then all wait).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ bool pwait_all(uint64_t* bar, uint32_t parity, int* status, int code) {
  return __all_sync(kPFull, mbar_wait(bar, parity, status, code));
}
__device__ __forceinline__ bool pwait_cluster_all(uint64_t* bar, uint32_t parity, int* status, int code) {
  return __all_sync(kPFull, mbar_wait_cluster(bar, parity, status, code));
}

// This CTA's half of one token's qNope rows into tensor memory (thread t = row t = head h0 + t,
// columns 0..127) and, on rank 0, the group's qRope rows into shared memory by TMA (thread 0).
// Every thread arrives on q_full once.  Runs only while no QK MMA reads qNope or qRope.
__device__ __forceinline__ void pair_load_query(const PairParams& p, const CUtensorMap* tmQr, uint8_t* sQr,
                                                uint64_t* q_full, uint32_t tmem_row, int h0, int token, int head,
                                                uint32_t rank) {
  if (rank == 0 && threadIdx.x == 0) {
    mbar_expect_tx_only(q_full, kPQr);
    tma_load_3d(sQr, tmQr, q_full, 0, h0, token);
  }
  const uint4* src =
      reinterpret_cast<const uint4*>(p.q_nope + (((size_t)token * p.heads + head) * 512 + 256 * rank) * 2);
#pragma unroll
  for (int c32 = 0; c32 < 4; ++c32) {  // 32 columns = 64 elements = 128 B per store
    uint32_t r[32];
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint4 w = __ldg(src + c32 * 8 + v);
      r[4 * v + 0] = w.x;
      r[4 * v + 1] = w.y;
      r[4 * v + 2] = w.z;
      r[4 * v + 3] = w.w;
    }
    tmem_st32(tmem_row + c32 * 32, r);
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(q_full);
}

// Launched in clusters of two CTAs (rank = latent half).
template <typename T>
__global__ void __launch_bounds__(192, 1)
    mla_pair_kernel(const __grid_constant__ CUtensorMap tmQr, const __grid_constant__ CUtensorMap tmKV,
                    const __grid_constant__ CUtensorMap tmKV3, const __grid_constant__ CUtensorMap tmKR,
                    const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQr = smem;
  uint8_t* sKV = sQr + kPQr;
  uint8_t* sX = sKV + kPStages * kPSlot;  // [2][128 rows][64 fp32]: the peer's partial scores
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + 2 * kPX);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kPStages;
  uint64_t* s_full = kv_empty + kPStages;  // [2]
  uint64_t* p_full = s_full + 2;           // [2]
  uint64_t* pv_done = p_full + 2;          // [2]
  uint64_t* pv_last = pv_done + 2;
  uint64_t* x_full = pv_last + 1;          // [2] the peer's partial of S[b] is in sX[b]
  uint64_t* x_empty = x_full + 2;          // [2] the peer has read this CTA's partial of S[b]
  uint64_t* fin = x_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kPNBars);

  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int cl = blockIdx.x >> 1;          // cluster index = lane * groups + group
  const int ln = cl / p.groups;
  const int h0 = (cl - ln * p.groups) * kPRows;
  const int k0 = p.lane_off[ln];
  const int k1 = p.lane_off[ln + 1];
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 128);
      mbar_init(pv_done + b, 1);
      mbar_init(x_full + b, 128);   // the peer's 128 softmax threads
      mbar_init(x_empty + b, 128);
    }
    mbar_init(pv_last, 1);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either arrives on the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer (one elected thread)
    if (elect_one()) {
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmKV3);
      tma_prefetch_desc(&tmKR);
      const int bs = p.block_size;
      const bool whole = bs % kPKeys == 0;  // a tile lies in one page: one 3-D box holds the CTA's half
      const int box_rows = bs < kPKeys ? bs : kPKeys;
      const uint32_t bytes = 4 * kPBlk + (rank == 0 ? kPBlk : 0);
      int G = 0;
      bool ok = true;
      for (int k = k0; k < k1 && ok; ++k) {
        const PairPiece pc = p.pieces[k];
        const int32_t* bt = p.block_tables + (size_t)pc.b * p.max_blocks;
        const int n_pages = (pc.last + 1 + bs - 1) / bs;  // pages holding keys <= the token's last key
        for (int j = 0; j < pc.n_tiles; ++j, ++G) {
          const int s = G % kPStages;
          if (G >= kPStages && !mbar_wait(kv_empty + s, ((G / kPStages) - 1) & 1, status, kDevTimeoutKEmpty)) {
            ok = false;
            break;
          }
          uint8_t* dst = sKV + s * kPSlot;
          mbar_expect_tx(kv_full + s, bytes);
          const int j0 = pc.kv_begin + j * kPKeys;
          for (int r0 = 0; r0 < kPKeys; r0 += box_rows) {
            const int pos = j0 + r0;
            const int pg = pos / bs;
            const int row = pg < n_pages ? bt[pg] * bs + (pos - pg * bs) : p.oob_row;  // past the last page: zeros
            if (whole) {
              tma_load_3d(dst, &tmKV3, kv_full + s, 0, row, 4 * (int)rank);  // blocks 4r..4r+3: [block][key][64]
            } else {
              for (int cb = 0; cb < 4; ++cb)
                tma_load_2d(dst + cb * kPBlk + r0 * 128, &tmKV, kv_full + s, (4 * (int)rank + cb) * 64, row);
            }
            if (rank == 0) tma_load_2d(dst + 4 * kPBlk + r0 * 128, &tmKR, kv_full + s, 0, row);
          }
        }
      }
      // no copy may be in flight when the CTA exits
      for (int t = G - kPStages < 0 ? 0 : G - kPStages; t < G; ++t)
        mbar_wait(kv_full + (t % kPStages), (t / kPStages) & 1, status, kDevTimeoutKFull);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (one elected thread)
    if (elect_one()) {
      constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
      constexpr uint32_t idesc_qk = instr_desc(fmt, false, false, kPRows, kPKeys);
      constexpr uint32_t idesc_pv = instr_desc(fmt, false, true, kPRows, 256);
      const uint64_t dqr = smem_desc_sw128(smem_addr(sQr), 16, 1024);   // qRope rows, K-major
      const uint64_t dk = smem_desc_sw128(smem_addr(sKV), 16, 1024);    // ctKV half (and kRope), K-major
      const uint64_t dv = smem_desc(smem_addr(sKV), kPBlk, 1024, 2);    // ctKV half as the MN-major V operand
      int total = 0;
      for (int k = k0; k < k1; ++k) total += p.pieces[k].n_tiles;
      // QK cursor: piece kq, tile jq of nq, CTA tile Gq; PV cursor likewise
      int kq = k0, jq = 0, nq = k0 < k1 ? p.pieces[k0].n_tiles : 0, Gq = 0;
      int kp = k0, jp = 0, np = nq, Gp = 0;
      bool ok = true;
      uint64_t t_prog = global_timer_ns();
      uint32_t it = 0;
      bool progressed = false;
      while (ok && Gp < total) {
        // QK(Gq) needs its tile, the score buffer Gq & 1 (free once PV(Gq - 2), which read P from it,
        // has completed) and, first in a piece, the query.  PV(Gp) needs P(Gp).
        const int sq = Gq % kPStages;
        const int bq = Gq & 1;
        if (Gq < total && Gq - Gp < 2 && mbar_test_wait(kv_full + sq, (Gq / kPStages) & 1) &&
            (Gq < 2 || mbar_test_wait(pv_done + bq, ((Gq - 2) >> 1) & 1)) &&
            (jq > 0 || mbar_test_wait(q_full, (kq - k0) & 1))) {
          tc_fence_after();
          const uint64_t so = (uint64_t)((sq * kPSlot) >> 4);
          const uint32_t d = tmem + kPSCol + 64 * bq;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)  // 256 dimensions: qNope half from tensor memory (8 columns per 16)
            mma_ts(d, tmem + kk * 8, dk + so + (uint64_t)(((kk >> 2) * kPBlk + (kk & 3) * 32) >> 4), idesc_qk,
                   kk > 0 ? 1u : 0u, false);
          if (rank == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // qRope x kRope from shared memory
              mma_ss(d, dqr + (uint64_t)((kk * 32) >> 4), dk + so + (uint64_t)((4 * kPBlk + kk * 32) >> 4), idesc_qk,
                     1u, false);
          }
          mma_commit(s_full + bq);
          ++Gq;
          if (++jq == nq) {
            ++kq;
            jq = 0;
            nq = kq < k1 ? p.pieces[kq].n_tiles : 0;
          }
          progressed = true;
        } else if (Gp < Gq && mbar_test_wait(p_full + (Gp & 1), (Gp >> 1) & 1)) {
          tc_fence_after();
          const uint64_t so = (uint64_t)(((Gp % kPStages) * kPSlot) >> 4);
          const uint32_t pa = tmem + kPSCol + 64 * (Gp & 1);  // P(Gp): 64 keys as 32 columns of 16-bit pairs
#pragma unroll
          for (int kk = 0; kk < kPKeys / 16; ++kk)
            mma_ts(tmem + kPOCol, pa + kk * 8, dv + so + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                   (jp > 0 || kk > 0) ? 1u : 0u, false);
          mma_commit(pv_done + (Gp & 1));
          mma_commit(kv_empty + (Gp % kPStages));
          if (jp + 1 == np) mma_commit(pv_last);
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
    // ------------------------------------------------------------ softmax / epilogue: thread t = row t = head h0 + t
    const int t = threadIdx.x;
    const int head = h0 + t;
    const uint32_t tmem_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float scale = p.scale_log2;
    const bool raw_max = scale > 0.f;  // max of the raw scores, scale folded into the exponent
    // row t of the exchange buffers: 64 floats as 16 chunks of 16 bytes, chunk c at c ^ (t & 15) so that
    // a warp's 16-byte accesses spread over all bank groups
    const uint32_t xsw = static_cast<uint32_t>(t & 15);
    const uint32_t x_local = smem_addr(sX) + t * 256;
    const uint32_t x_remote = peer_addr(x_local, peer);
    const uint32_t xf_remote = peer_addr(smem_addr(x_full), peer);
    const uint32_t xe_remote = peer_addr(smem_addr(x_empty), peer);
    bool ok = true;
    int G = 0;  // tiles consumed
    if (k0 < k1) pair_load_query(p, &tmQr, sQr, q_full, tmem_row, h0, p.pieces[k0].token0, head, rank);
    for (int k = k0; k < k1 && ok; ++k) {
      const PairPiece pc = p.pieces[k];
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; j < pc.n_tiles; ++j, ++G) {
        const int b = G & 1;
        ok = pwait_all(s_full + b, (G >> 1) & 1, status, kDevTimeoutSFull);
        if (!ok) break;
        tc_fence_after();
        uint32_t r[2][32];
        tmem_ld32(tmem_row + kPSCol + 64 * b, r[0]);
        tmem_ld32(tmem_row + kPSCol + 64 * b + 32, r[1]);
        tmem_ld_wait();
        // this CTA's partial into the peer's buffer b, once the peer has read what went there two tiles ago
        if (G >= 2 && !(ok = pwait_cluster_all(x_empty + b, ((G >> 1) - 1) & 1, status, kDevTimeoutSFree))) break;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t* q = &r[c >> 3][(c & 7) * 4];
          st_cluster_v4(x_remote + b * kPX + ((c ^ xsw) << 4), q[0], q[1], q[2], q[3]);
        }
        mbar_arrive_remote(xf_remote + 8 * b);
        // the peer's partial, added in the same order on both CTAs (fp32 addition commutes)
        if (!(ok = pwait_cluster_all(x_full + b, (G >> 1) & 1, status, kDevTimeoutSFull))) break;
        float x[kPKeys];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 v = ld_shared_v4p(x_local + b * kPX + ((c ^ xsw) << 4));
          const uint32_t* q = &r[c >> 3][(c & 7) * 4];
          x[4 * c + 0] = __uint_as_float(q[0]) + __uint_as_float(v.x);
          x[4 * c + 1] = __uint_as_float(q[1]) + __uint_as_float(v.y);
          x[4 * c + 2] = __uint_as_float(q[2]) + __uint_as_float(v.z);
          x[4 * c + 3] = __uint_as_float(q[3]) + __uint_as_float(v.w);
        }
        mbar_arrive_remote(xe_remote + 8 * b);  // the peer may write its next partial into buffer b
        const int lim = pc.last - (pc.kv_begin + j * kPKeys);  // columns c <= lim are allowed
        if (!raw_max) {
#pragma unroll
          for (int c = 0; c < kPKeys; ++c) x[c] *= scale;
        }
        if (__any_sync(kPFull, lim < kPKeys - 1)) {  // only a range's last tile can hold masked keys
#pragma unroll
          for (int c = 0; c < kPKeys; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kPKeys; c += 8) {
          mx0 = max3(mx0, x[c], x[c + 1]);
          mx1 = max3(mx1, x[c + 2], x[c + 3]);
          mx2 = max3(mx2, x[c + 4], x[c + 5]);
          mx3 = max3(mx3, x[c + 6], x[c + 7]);
        }
        float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        if (raw_max) mx *= scale;
        const float m_new = fmaxf(m_run, mx);
        float alpha = 1.f;
        if (m_new - m_run > kPRescale) {  // false while both are -inf
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        if (j >= 1 && __any_sync(kPFull, alpha != 1.f)) {
          // O must hold P(j-1) V(j-1) before it is scaled; PV(j) waits for P(j), which comes after
          const int g1 = G - 1;
          if (!(ok = pwait_all(pv_done + (g1 & 1), (g1 >> 1) & 1, status, kDevTimeoutODone))) break;
          tc_fence_after();
#pragma unroll 2
          for (int c32 = 0; c32 < 256 / 32; ++c32) {
            uint32_t o[32];
            tmem_ld32(tmem_row + kPOCol + c32 * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem_row + kPOCol + c32 * 32, o);
          }
          tmem_st_wait();
        }
        const float m_base = (m_run == -INFINITY) ? 0.f : m_run;
        // P = 2^(x*scale - m) a pair of columns at a time (-inf masked keys give exactly 0), over S[b]
        const uint64_t scale2 = f2pack(raw_max ? scale : 1.f, raw_max ? scale : 1.f);
        const uint64_t negm2 = f2pack(-m_base, -m_base);
        uint64_t acc0 = f2pack(0.f, 0.f), acc1 = f2pack(0.f, 0.f);
        uint32_t pk[kPKeys / 2];
#pragma unroll
        for (int c = 0; c < kPKeys; c += 2) {
          float e0, e1;
          f2unpack(fma_x2(f2pack(x[c], x[c + 1]), scale2, negm2), e0, e1);
          e0 = fast_exp2(e0);
          e1 = fast_exp2(e1);
          if ((c >> 1) & 1) acc1 = add_x2(acc1, f2pack(e0, e1));
          else acc0 = add_x2(acc0, f2pack(e0, e1));
          pk[c >> 1] = ppack2(e0, e1, (T*)nullptr);
        }
        float s0, s1;
        f2unpack(add_x2(acc0, acc1), s0, s1);
        l_run = l_run * alpha + (s0 + s1);
        tmem_st32(tmem_row + kPSCol + 64 * b, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + b);
      }
      if (!ok) break;
      // every QK of this piece has completed (its scores were read): the next token's query may go in
      if (k + 1 < k1) pair_load_query(p, &tmQr, sQr, q_full, tmem_row, h0, p.pieces[k + 1].token0, head, rank);
      // ---- epilogue: O_half / l of this piece
      if (!(ok = pwait_all(pv_last, (k - k0) & 1, status, kDevTimeoutODone))) break;
      tc_fence_after();
      // a row whose allowed keys all lie before this range (possible only in a partial) contributes nothing
      const bool empty = !(l_run > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l_run;
      const float lse_row = empty ? -INFINITY : (m_run == -INFINITY ? 0.f : m_run) * kPLn2 + logf(l_run);
      if (pc.part < 0) {
        T* orow = reinterpret_cast<T*>(p.out) + ((size_t)pc.token0 * p.heads + head) * 512 + 256 * rank;
#pragma unroll 2
        for (int c32 = 0; c32 < 8; ++c32) {
          uint32_t o[32];
          tmem_ld32(tmem_row + kPOCol + c32 * 32, o);
          tmem_ld_wait();
          uint4* dst = reinterpret_cast<uint4*>(orow + c32 * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(ppack2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l, (T*)nullptr),
                                ppack2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l, (T*)nullptr),
                                ppack2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l, (T*)nullptr),
                                ppack2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l, (T*)nullptr));
        }
        if (rank == 0 && p.lse) p.lse[(size_t)pc.token0 * p.heads + head] = lse_row;
      } else {
        float* prow = p.part_o + ((size_t)pc.part * p.heads + head) * 512 + 256 * rank;
#pragma unroll 2
        for (int c32 = 0; c32 < 8; ++c32) {
          uint32_t o[32];
          tmem_ld32(tmem_row + kPOCol + c32 * 32, o);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(prow + c32 * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v + 0]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                 __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
        if (rank == 0) p.part_lse[(size_t)pc.part * p.heads + head] = lse_row;
      }
      tc_fence_before();  // O has been read before the next piece's first PV overwrites it
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  cluster_sync_all();  // neither CTA leaves while the other may still write into its shared memory
}

// Merge of the partial results of one token's key ranges by their lse:
// lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.
// One CTA per (token, 8 heads); one warp per head, 16 output columns per lane.
template <typename T>
__global__ void __launch_bounds__(256) mla_pair_combine_kernel(const PairCombine* work, const PairParams p) {
  const PairCombine w = work[blockIdx.x];
  const int head = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (head >= p.heads) return;
  float m = -INFINITY;
  for (int s = 0; s < w.n_parts; ++s) m = fmaxf(m, p.part_lse[(size_t)(w.part_begin + s) * p.heads + head]);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float den = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < w.n_parts; ++s) {
      const size_t row = (size_t)(w.part_begin + s) * p.heads + head;
      const float wgt = expf(p.part_lse[row] - m);
      den += wgt;
      const float4* src = reinterpret_cast<const float4*>(p.part_o + row * 512 + lane * 16);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 f = src[v];
        acc[4 * v + 0] += wgt * f.x;
        acc[4 * v + 1] += wgt * f.y;
        acc[4 * v + 2] += wgt * f.z;
        acc[4 * v + 3] += wgt * f.w;
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) + ((size_t)w.token * p.heads + head) * 512 + lane * 16);
#pragma unroll
  for (int v = 0; v < 2; ++v)
    dst[v] = make_uint4(ppack2(acc[8 * v + 0] * inv, acc[8 * v + 1] * inv, (T*)nullptr),
                        ppack2(acc[8 * v + 2] * inv, acc[8 * v + 3] * inv, (T*)nullptr),
                        ppack2(acc[8 * v + 4] * inv, acc[8 * v + 5] * inv, (T*)nullptr),
                        ppack2(acc[8 * v + 6] * inv, acc[8 * v + 7] * inv, (T*)nullptr));
  if (lane == 0 && p.lse) p.lse[(size_t)w.token * p.heads + head] = m == -INFINITY ? -INFINITY : m + logf(den);
}

typedef CUresult (*PairEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// rank-2 or rank-3 16-bit map with a 128-byte inner box and 128B swizzle
bool pair_encode(CUtensorMap* map, void* base, int32_t dtype, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  static PairEncodeFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<PairEncodeFn>(ptr);
  }
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType t = dtype == ALA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(map, t, rank, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int pfail(char* err, size_t n, int code, const char* msg) {
  if (err && n) {
    std::strncpy(err, msg, n - 1);
    err[n - 1] = 0;
  }
  return code;
}

void fill_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, int ctas, cudaStream_t stream) {
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->gridDim = dim3(ctas, 1, 1);
  cfg->blockDim = dim3(192, 1, 1);
  cfg->dynamicSmemBytes = kPSmem;
  cfg->stream = stream;
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = 2;
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

// Clusters of two 206 KB CTAs that can be resident at once (the grid is cut to fit in one wave).
int pair_max_clusters() {
  static int cached = 0;
  if (cached > 0) return cached;
  int n = 0;
  auto kern = mla_pair_kernel<__nv_bfloat16>;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr;
  fill_config(&cfg, &attr, 2 * (kPPlannedSms / 2), nullptr);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = kPPlannedSms / 2 - 4;  // unknown: leave room for SMs a cluster cannot pair up
  }
  cached = std::min(n, kPPlannedSms / 2);
  return cached;
}

}  // namespace

bool mla_pair_eligible(const MlaPlan* plan) {
  if (plan->kv8 || plan->heads % kPRows != 0) return false;
  for (int32_t q : plan->qs)
    if (q != 1) return false;
  return (reinterpret_cast<uintptr_t>(plan->out) % 16) == 0 && (reinterpret_cast<uintptr_t>(plan->q_nope) % 16) == 0;
}

int mla_pair_plan(MlaPlan* plan, char* err, size_t n) {
  const int32_t groups = plan->heads / kPRows;
  struct Chunk {
    int32_t b, last, tiles;
  };
  std::vector<Chunk> chunks;
  int64_t total_tiles = 0;
  for (int32_t b = 0; b < plan->batch; ++b) {  // one query token per batch: token b
    const int32_t last = plan->ctx[b] - 1;
    const int32_t tiles = (last + kPKeys) / kPKeys;
    chunks.push_back(Chunk{b, last, tiles});
    total_tiles += tiles;
  }
  const int64_t lanes_max = std::max<int64_t>(1, pair_max_clusters() / groups);
  const int64_t per_lane = std::max<int64_t>(kPMinLaneTiles, (total_tiles + lanes_max - 1) / lanes_max);
  std::vector<PairPiece> pieces;
  std::vector<int32_t> piece_lane;
  std::vector<PairCombine> comb;
  int32_t parts = 0, lane_id = 0;
  int64_t pos = 0, lane_end = per_lane;
  for (const Chunk& ch : chunks) {
    const size_t first = pieces.size();
    for (int32_t t = 0; t < ch.tiles;) {
      const int32_t take = (int32_t)std::min<int64_t>(lane_end - pos, ch.tiles - t);
      pieces.push_back(PairPiece{ch.b, ch.b, t * kPKeys, take, ch.last, -1, {0, 0}});
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
      comb.push_back(PairCombine{ch.b, parts, np, 0});
      parts += np;
    }
  }
  const int32_t n_lanes = pieces.empty() ? 0 : piece_lane.back() + 1;
  std::vector<int32_t> lane_off(n_lanes + 1, 0);
  for (int32_t l = 0, i = 0; l <= n_lanes; ++l) {
    while (i < (int32_t)pieces.size() && piece_lane[i] < l) ++i;
    lane_off[l] = i;
  }
  plan->pair = true;
  plan->tpc = 1;
  plan->hpc = kPRows;
  plan->groups = groups;
  plan->n_lanes = n_lanes;
  plan->n_work = n_lanes * groups;  // clusters
  plan->n_splits_total = parts;
  plan->n_combine = (int32_t)comb.size();
  auto align = [](uint64_t x) { return (x + 255) / 256 * 256; };
  plan->off_work = 256;
  plan->off_lanes = align(plan->off_work + sizeof(PairPiece) * std::max<size_t>(pieces.size(), 1));
  plan->off_rows = align(plan->off_lanes + sizeof(int32_t) * lane_off.size());
  plan->off_part_lse = align(plan->off_rows + sizeof(PairCombine) * std::max<size_t>(comb.size(), 1));
  const uint64_t part_rows = (uint64_t)parts * plan->heads;
  plan->off_part_o = align(plan->off_part_lse + sizeof(float) * part_rows);
  plan->ws_size = align(plan->off_part_o + sizeof(float) * part_rows * 512);
  plan->image_size = plan->off_part_lse;
  plan->image.assign(plan->image_size, 0);
  std::memcpy(plan->image.data() + plan->off_work, pieces.data(), sizeof(PairPiece) * pieces.size());
  std::memcpy(plan->image.data() + plan->off_lanes, lane_off.data(), sizeof(int32_t) * lane_off.size());
  std::memcpy(plan->image.data() + plan->off_rows, comb.data(), sizeof(PairCombine) * comb.size());
  if (plan->pinned) {  // a page-locked copy of an earlier schedule
    cudaFreeHost(plan->pinned);
    plan->pinned = nullptr;
  }
  plan->maps_ready = false;
  (void)err;
  (void)n;
  return ALA_OK;
}

int mla_pair_run(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t n) {
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return pfail(err, n, ALA_INVALID_PARAM, "workspace must be 256-byte aligned");
  if (plan->n_work == 0) return ALA_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (!plan->maps_ready) {
    const cuuint64_t rows = (cuuint64_t)plan->num_blocks * plan->block_size;
    const cuuint32_t box_rows = (cuuint32_t)std::min(plan->block_size, kPKeys);
    cuuint64_t qr_dims[3] = {64, (cuuint64_t)plan->heads, (cuuint64_t)plan->tokens};
    cuuint64_t qr_str[2] = {128, (cuuint64_t)plan->heads * 128};
    cuuint32_t qr_box[3] = {64, (cuuint32_t)kPRows, 1};
    cuuint64_t kv_dims[2] = {512, rows};
    cuuint64_t kv_str[1] = {1024};
    cuuint32_t kv_box[2] = {64, box_rows};
    cuuint64_t kr_dims[2] = {64, rows};
    cuuint64_t kr_str[1] = {128};
    // ctKV as (64 elements, rows, 8 column blocks): a box of 4 blocks is a CTA's half of a 64-key tile,
    // laid out [column block][key][64 elements]
    cuuint64_t kv3_dims[3] = {64, rows, 8};
    cuuint64_t kv3_str[2] = {1024, 128};
    cuuint32_t kv3_box[3] = {64, (cuuint32_t)kPKeys, 4};
    if (!pair_encode(&plan->tmQr, plan->q_rope, plan->dtype, 3, qr_dims, qr_str, qr_box) ||
        !pair_encode(&plan->tmKV, plan->ct_kv, plan->dtype, 2, kv_dims, kv_str, kv_box) ||
        !pair_encode(&plan->tmKR, plan->k_rope, plan->dtype, 2, kr_dims, kr_str, kv_box) ||
        !pair_encode(&plan->tmKV3, plan->ct_kv, plan->dtype, 3, kv3_dims, kv3_str, kv3_box))
      return pfail(err, n, ALA_CUDA_ERROR, "cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)");
    plan->maps_ready = true;
  }
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
    return pfail(err, n, ALA_CUDA_ERROR, "schedule upload failed");
  PairParams p{};
  p.pieces = reinterpret_cast<const PairPiece*>(ws + plan->off_work);
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
  p.max_blocks = plan->max_blocks;
  p.block_size = plan->block_size;
  p.oob_row = (int32_t)(plan->num_blocks * plan->block_size);
  p.scale_log2 = plan->qk_scale * kPLog2e;
  const bool f16 = plan->dtype == ALA_F16;
  auto kern = f16 ? mla_pair_kernel<__half> : mla_pair_kernel<__nv_bfloat16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr;
    fill_config(&cfg, &attr, 2 * plan->n_work, stream);
    e = cudaLaunchKernelEx(&cfg, kern, plan->tmQr, plan->tmKV, plan->tmKV3, plan->tmKR, p);
  }
  if (e == cudaSuccess && plan->n_combine > 0) {
    auto ck = f16 ? mla_pair_combine_kernel<__half> : mla_pair_combine_kernel<__nv_bfloat16>;
    dim3 grid(plan->n_combine, (plan->heads + 7) / 8);
    ck<<<grid, 256, 0, stream>>>(reinterpret_cast<const PairCombine*>(ws + plan->off_rows), p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return pfail(err, n, ALA_CUDA_ERROR, cudaGetErrorString(e));
  return ALA_OK;
}

}  // namespace ala
