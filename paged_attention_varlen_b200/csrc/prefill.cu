// prefill.cu -- masked attention over packed variable-length sequences for
// sm_100a, with K/V read from a contiguous packed tensor or from a paged cache
// through a block table (ATB "PrefixEncoder" page, definition and parameter
// table; nalar.dev padding-mask article, sections on packing and on fused
// kernels that apply the mask rule without materialising it).
//
// One CTA computes 128 query rows of one query head of one sequence:
//
//   warp 4      TMA producer: Q tile once, then K and V tiles (128 keys each)
//               into a STAGES-deep ring; paged K/V rows are gathered page by
//               page through the block table.
//   warp 5      tcgen05 issuer: S = Q K^T into one of two TMEM buffers, then
//               O += P V into the TMEM accumulator; completion is signalled
//               with tcgen05.commit on mbarriers.
//   warps 0..3  softmax: thread r owns query row r (TMEM lane r).  It reads its
//               S row from TMEM, applies qkScale, the ALiBi bias and the mask
//               rule in registers (the mask is never materialised), keeps the
//               online max / sum, rescales O in TMEM when the running max grows
//               by more than 2^8, writes P to shared memory in the swizzled
//               operand layout, and finally normalises O and stores it.
//
// Key tiles wholly above the prefix-shifted causal diagonal, or past the
// sequence's kvSeqLen, are never visited: the host gives each unit the
// number of tiles up to its last allowed key.
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

template <typename T, int D, int STAGES>
struct Cfg {
  static constexpr int ES = sizeof(T);
  static constexpr int AW = 128 / ES;    // elements in one 128-byte swizzled row
  static constexpr int UK = 32 / ES;     // K extent of one MMA instruction
  static constexpr int BM = 128;         // query rows per CTA
  static constexpr int BN = 128;         // keys per tile
  static constexpr int BLK = 128 * 128;  // bytes of one 128-row x 128-byte swizzle column block
  static constexpr int Q_BYTES = BM * D * ES;
  static constexpr int KV_BYTES = BN * D * ES;
  static constexpr int P_BYTES = BM * BN * ES;
  static constexpr int N_BARS = 1 + 4 * STAGES + 7;
  static constexpr int SMEM = 1024 + Q_BYTES + 2 * STAGES * KV_BYTES + P_BYTES + N_BARS * 8 + 16;
  static constexpr uint32_t IDESC_QK = instr_desc(ElemFmt<T>::fmt, false, false, 128, 128);
  static constexpr uint32_t IDESC_PV = instr_desc(ElemFmt<T>::fmt, false, true, 128, D);
  static constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128) S1 [128,256) O [256, 256+D)
  static constexpr uint32_t O_COL = 256;
  static_assert(D % AW == 0, "head size must fill whole swizzle rows");
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Write 16 bytes of row r's operand data into a 128B-swizzled K-major block.
__device__ __forceinline__ void st_swizzled16(uint8_t* block, int r, int chunk, uint4 v) {
  uint8_t* dst = block + r * 128 + ((chunk ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(dst) = v;
}

template <typename T, int D, int STAGES>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = Cfg<T, D, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;
  uint8_t* sV = sK + STAGES * C::KV_BYTES;
  uint8_t* sP = sV + STAGES * C::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + C::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + STAGES;
  uint64_t* k_empty = bars + 1 + 2 * STAGES;
  uint64_t* v_empty = bars + 1 + 3 * STAGES;
  uint64_t* s_full = bars + 1 + 4 * STAGES;  // [2]
  uint64_t* s_free = s_full + 2;             // [2]
  uint64_t* p_full = s_full + 4;
  uint64_t* o_done = s_full + 5;
  uint64_t* fin = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::N_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const PrefillUnit u = p.units[blockIdx.x];
  const SeqInfo si = p.seqs[u.b];
  const int n = u.n_tiles;
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int kvh = u.head / p.group;
      mbar_expect_tx(q_full, C::Q_BYTES);
      for (int cb = 0; cb < D / C::AW; ++cb)
        tma_load_3d(sQ + cb * C::BLK, &tmQ, q_full, cb * C::AW, u.head, si.cu_q + u.q0);

      const bool paged = p.block_tables != nullptr;
      const int bs = p.block_size;
      const int box_rows = paged ? (bs < 128 ? bs : 128) : 128;
      const int n_pages = paged ? (si.kv_len + bs - 1) / bs : 0;
      const int32_t* bt = paged ? p.block_tables + (size_t)u.b * p.max_blocks : nullptr;
      bool ok = true;
      int issued[2] = {0, 0};  // tiles whose K (0) / V (1) load was issued
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % STAGES;
        const uint32_t par = ((j / STAGES) - 1) & 1;
        for (int kv = 0; kv < 2; ++kv) {
          uint64_t* empty = kv ? v_empty + s : k_empty + s;
          uint64_t* full = kv ? v_full + s : k_full + s;
          const CUtensorMap* map = kv ? &tmV : &tmK;
          uint8_t* dst = (kv ? sV : sK) + s * C::KV_BYTES;
          if (j >= STAGES && !mbar_wait(empty, par, status, kv ? kDevTimeoutVEmpty : kDevTimeoutKEmpty)) {
            ok = false;
            break;
          }
          mbar_expect_tx(full, C::KV_BYTES);
          const int j0 = j * 128;
          for (int r0 = 0; r0 < 128; r0 += box_rows) {
            int row;
            if (!paged) {
              row = si.cu_kv + j0 + r0;
            } else {
              const int pos = j0 + r0;
              const int pg = pos / bs;
              row = pg < n_pages ? bt[pg] * bs + (pos % bs) : p.oob_row;
            }
            for (int cb = 0; cb < D / C::AW; ++cb)
              tma_load_3d(dst + cb * C::BLK + r0 * 128, map, full, cb * C::AW, kvh, row);
          }
          issued[kv] = j + 1;
        }
      }
      // never leave the CTA while loads it issued are still landing in shared memory
      for (int kv = 0; kv < 2; ++kv)
        for (int j = issued[kv] - STAGES < 0 ? 0 : issued[kv] - STAGES; j < issued[kv]; ++j)
          mbar_wait((kv ? v_full : k_full) + j % STAGES, (j / STAGES) & 1, status,
                    kv ? kDevTimeoutVFull : kDevTimeoutKFull);
      mbar_wait(q_full, 0, status, kDevTimeoutQ);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_addr(sQ);
      const uint32_t p_base = smem_addr(sP);
      bool ok = mbar_wait(q_full, 0, status, kDevTimeoutQ);
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          const int s = j % STAGES;
          const int sb = j & 1;
          if (!mbar_wait(k_full + s, (j / STAGES) & 1, status, kDevTimeoutKFull)) break;
          if (j >= 2 && !mbar_wait(s_free + sb, ((j - 2) >> 1) & 1, status, kDevTimeoutSFree)) break;
          tc_fence_after();
          const uint32_t k_base = smem_addr(sK + s * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / C::UK; ++kk) {
            const int ke = kk * C::UK;
            const uint32_t off = (ke / C::AW) * C::BLK + (ke % C::AW) * C::ES;
            mma_ss(tmem + sb * 128, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + off, 16, 1024),
                   C::IDESC_QK, kk > 0, C::ES == 4);
          }
          mma_commit(k_empty + s);
          mma_commit(s_full + sb);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % STAGES;
          if (!mbar_wait(v_full + s, (jj / STAGES) & 1, status, kDevTimeoutVFull)) break;
          if (!mbar_wait(p_full, jj & 1, status, kDevTimeoutPFull)) break;
          tc_fence_after();
          const uint32_t v_base = smem_addr(sV + s * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < 128 / C::UK; ++kk) {
            const int ke = kk * C::UK;
            const uint32_t poff = (ke / C::AW) * C::BLK + (ke % C::AW) * C::ES;
            // V is the MN-major operand: 16-bit types use the 16-byte-chunk swizzle (8-row atoms),
            // tf32 the 32-byte-chunk swizzle (4-row atoms), matching how the V tensor map loads it
            const uint64_t vdesc = C::ES == 4 ? smem_desc(v_base + ke * 128, C::BLK, 512, 1)
                                              : smem_desc(v_base + ke * 128, C::BLK, 1024, 2);
            mma_ss(tmem + C::O_COL, smem_desc_sw128(p_base + poff, 16, 1024), vdesc, C::IDESC_PV,
                   (jj > 0 || kk > 0) ? 1u : 0u, C::ES == 4);
          }
          mma_commit(v_empty + s);
          mma_commit(o_done);
        }
      }
      // all tensor-core work this thread issued has finished before TMEM is released
      mma_commit(fin);
      mbar_wait(fin, 0, status, kDevTimeoutFinal);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = threadIdx.x;  // query row in the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int qi = u.q0 + r;
    const bool row_valid = qi < si.seq_len;
    const int iabs = qi + (si.kv_len - si.seq_len);
    const int mt = p.mask_type;
    const bool alibi = (mt == 3 || mt == 4 || mt == 5);
    const float slope = alibi ? p.slopes[u.head] : 0.f;
    const float slope_log2 = slope * kLog2e;
    // last allowed key of this row (inclusive)
    const int last_key = (mt == 0) ? si.kv_len - 1 : min(iabs, si.kv_len - 1);
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full + sb, (j >> 1) & 1, status, kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t regs[32];
        tmem_ld32(tmem + lane_base + sb * 128 + c4 * 32, regs);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c4 * 32 + c] = __uint_as_float(regs[c]);
      }
      tc_fence_before();
      mbar_arrive(s_free + sb);

      const int j0 = j * 128;
      const int lim = last_key - j0;  // columns c <= lim are allowed
      const float scale = p.scale_log2;
      if (mt == 3 || mt == 5) {
        // right- and left-aligned bias differ by a per-row constant; both use (j - iabs)
        const float b0 = slope_log2 * static_cast<float>(j0 - iabs);
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = fmaf(x[c], scale, fmaf(slope_log2, static_cast<float>(c), b0));
      } else if (mt == 4) {
        const float d0 = static_cast<float>(iabs - j0);
#pragma unroll
        for (int c = 0; c < 128; ++c)
          x[c] = fmaf(x[c], scale, -slope_log2 * sqrtf(fmaxf(d0 - static_cast<float>(c), 0.f)));
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] *= scale;
      }
      if (lim < 127) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
      }
      float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, x[c]);
        mx1 = fmaxf(mx1, x[c + 1]);
        mx2 = fmaxf(mx2, x[c + 2]);
        mx3 = fmaxf(mx3, x[c + 3]);
      }
      const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      const float m_new = fmaxf(m_run, mx);
      float alpha = 1.f;
      if (m_new - m_run > kRescaleThreshold) {  // false while both are -inf
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float m_base = (m_run == -INFINITY) ? 0.f : m_run;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        x[c] = fast_exp2(x[c] - m_base);
        x[c + 1] = fast_exp2(x[c + 1] - m_base);
        sum0 += x[c];
        sum1 += x[c + 1];
      }
      l_run = l_run * alpha + (sum0 + sum1);

      // O and the P buffer are owned by the previous P*V until it completes
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status, kDevTimeoutODone));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c32 = 0; c32 < D / 32; ++c32) {
            uint32_t regs[32];
            const uint32_t addr = tmem + lane_base + C::O_COL + c32 * 32;
            tmem_ld32(addr, regs);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) regs[c] = __float_as_uint(__uint_as_float(regs[c]) * alpha);
            tmem_st32(addr, regs);
          }
          tmem_st_wait();
        }
      }
      // P -> shared memory, K-major 128B-swizzled operand layout
      if constexpr (C::ES == 2) {
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {  // 16 chunks of 8 elements
          uint4 v;
          v.x = pack2(x[ch * 8 + 0], x[ch * 8 + 1], (T*)nullptr);
          v.y = pack2(x[ch * 8 + 2], x[ch * 8 + 3], (T*)nullptr);
          v.z = pack2(x[ch * 8 + 4], x[ch * 8 + 5], (T*)nullptr);
          v.w = pack2(x[ch * 8 + 6], x[ch * 8 + 7], (T*)nullptr);
          st_swizzled16(sP + (ch >> 3) * C::BLK, r, ch & 7, v);
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < 32; ++ch) {  // 32 chunks of 4 fp32 (read as tf32)
          uint4 v = make_uint4(__float_as_uint(x[ch * 4 + 0]), __float_as_uint(x[ch * 4 + 1]),
                               __float_as_uint(x[ch * 4 + 2]), __float_as_uint(x[ch * 4 + 3]));
          st_swizzled16(sP + (ch >> 3) * C::BLK, r, ch & 7, v);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }

    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (n - 1) & 1, status, kDevTimeoutODone));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(si.cu_q + qi) * p.heads + u.head) * D;
#pragma unroll
      for (int c32 = 0; c32 < D / 32; ++c32) {
        uint32_t regs[32];
        tmem_ld32(tmem + lane_base + C::O_COL + c32 * 32, regs);
        tmem_ld_wait();
        if (row_valid) {
          if constexpr (C::ES == 2) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 v;
              v.x = pack2(__uint_as_float(regs[v4 * 8 + 0]) * inv_l, __uint_as_float(regs[v4 * 8 + 1]) * inv_l,
                          (T*)nullptr);
              v.y = pack2(__uint_as_float(regs[v4 * 8 + 2]) * inv_l, __uint_as_float(regs[v4 * 8 + 3]) * inv_l,
                          (T*)nullptr);
              v.z = pack2(__uint_as_float(regs[v4 * 8 + 4]) * inv_l, __uint_as_float(regs[v4 * 8 + 5]) * inv_l,
                          (T*)nullptr);
              v.w = pack2(__uint_as_float(regs[v4 * 8 + 6]) * inv_l, __uint_as_float(regs[v4 * 8 + 7]) * inv_l,
                          (T*)nullptr);
              *reinterpret_cast<uint4*>(orow + c32 * 32 + v4 * 8) = v;
            }
          } else {
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4) {
              float4 v = make_float4(__uint_as_float(regs[v4 * 4 + 0]) * inv_l, __uint_as_float(regs[v4 * 4 + 1]) * inv_l,
                                     __uint_as_float(regs[v4 * 4 + 2]) * inv_l, __uint_as_float(regs[v4 * 4 + 3]) * inv_l);
              *reinterpret_cast<float4*>(reinterpret_cast<float*>(orow) + c32 * 32 + v4 * 4) = v;
            }
          }
        }
      }
      if (row_valid && p.lse) {
        float lse = (m_run == -INFINITY ? 0.f : m_run) * kLn2 + logf(l_run);
        if (mt == 5) lse += slope * static_cast<float>(iabs);  // left-aligned bias = right-aligned + slope*iabs
        p.lse[(size_t)(si.cu_q + qi) * p.heads + u.head] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <typename T, int D, int STAGES>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const PrefillParams& p,
                   cudaStream_t stream) {
  using C = Cfg<T, D, STAGES>;
  // at least 120 KB so a second CTA never shares the SM (each CTA allocates all 512 TMEM columns)
  constexpr int kSmem = C::SMEM > 120 * 1024 ? C::SMEM : 120 * 1024;
  auto kern = prefill_kernel<T, D, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  if (p.n_units == 0) return cudaSuccess;
  kern<<<p.n_units, 192, kSmem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

int prefill_smem_bytes(int32_t dtype, int32_t d) {
  if (dtype == kBF16 || dtype == kF16) {
    if (d == 128) return Cfg<__half, 128, 2>::SMEM;
    if (d == 64) return Cfg<__half, 64, 2>::SMEM;
  } else if (dtype == kF32) {
    if (d == 64) return Cfg<float, 64, 1>::SMEM;
  }
  return 0;
}

cudaError_t launch_prefill(int32_t dtype, int32_t d, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const PrefillParams& p, cudaStream_t stream) {
  if (dtype == kBF16) {
    if (d == 128) return launch<__nv_bfloat16, 128, 2>(tmQ, tmK, tmV, p, stream);
    if (d == 64) return launch<__nv_bfloat16, 64, 2>(tmQ, tmK, tmV, p, stream);
  } else if (dtype == kF16) {
    if (d == 128) return launch<__half, 128, 2>(tmQ, tmK, tmV, p, stream);
    if (d == 64) return launch<__half, 64, 2>(tmQ, tmK, tmV, p, stream);
  } else if (dtype == kF32) {
    if (d == 64) return launch<float, 64, 1>(tmQ, tmK, tmV, p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ala
