// mla.cu -- MLA decode / speculative decode over a paged latent cache for
// sm_100a (ATB "MLA" page, definition and parameter table): per query token
// and head, O = softmax(qkScale * [qNope;qRope] . [ctKV;kRope]^T) ctKV, with
// the speculative causal rule (token t of a batch with qseqlen tokens allows
// keys j <= contextLens - qseqlen + t), plus the natural-log lse.
//
// Work split.  The 512-wide fp32 output of 128 heads would fill all of tensor
// memory, so one CTA handles 64 heads (M = 64 MMAs; the output is kept as two
// 256-column accumulators in the two lane halves of the same TMEM columns) of
// one query token over one range of keys.  The two head groups of a token read
// the same cache tiles, which L2 serves once from HBM.  Long key ranges are
// split so every SM has work; each split leaves an fp32 partial (O, lse) in the
// workspace and mla_combine_kernel merges them by lse (the same merge the MLA
// page's ring mode returns the lse for).
//
//   warp 4      TMA producer: the 64x576 query tile once; then 64-token tiles of
//               ctKV (512) and kRope (64) gathered through the block table into
//               a 2-deep ring.
//   warp 5      tcgen05 issuer: S = Q K^T (64 x 64, K = 576), O += P V with V
//               the ctKV part of the same tile (two N = 256 halves).
//   warps 0..3  softmax: lane l < 16 of warp w owns head 16w + l; it scales and
//               masks its S row in registers, keeps the online max / sum, writes
//               P to shared memory, rescales O when the max grew by more than 2^8,
//               and at the end normalises O (lanes >= 16 hold the upper 256
//               columns of the same heads) and stores it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <type_traits>

#include "internal.h"
#include "mla.h"
#include "ptx.cuh"

namespace ala {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

constexpr int kHeadsPerCta = 64;
constexpr int kTileKeys = 64;
constexpr int kDNope = 512;
constexpr int kBlk = 64 * 128;                     // one 64-row x 128-byte swizzle column block
constexpr int kQBytes = 9 * kBlk;                  // 64 heads x 576 x 2 B
constexpr int kKvBytes = 9 * kBlk;                 // 64 keys x 576 x 2 B
constexpr int kPBytes = kBlk;                      // 64 heads x 64 keys x 2 B
constexpr int kStages = 2;
constexpr int kNBars = 1 + 4 + 5;                  // q_full, kv_full[2], kv_empty[2], s_full, s_free, p_full, o_done, fin
constexpr int kSmem = 1024 + kQBytes + kStages * kKvBytes + kPBytes + kNBars * 8 + 16;
static_assert(kSmem <= 232448, "shared memory budget");
constexpr uint32_t kSCol = 256;                    // S: columns [256, 320), lanes of half 0
constexpr uint32_t kTmemCols = 512;

struct MlaUnit {
  int32_t b;         // batch
  int32_t token;     // packed query token
  int32_t t;         // token index within its batch
  int32_t group;     // head group (heads 64*group .. +63)
  int32_t kv_begin;  // first key of the range (multiple of 64)
  int32_t n_tiles;   // 64-key tiles in the range
  int32_t last_key;  // last allowed key of this token (inclusive)
  int32_t part;      // partial slot, or -1 when this unit writes the final output
};

struct MlaCombine {
  int32_t token;
  int32_t part_begin;
  int32_t n_parts;
  int32_t pad;
};

struct MlaParams {
  const MlaUnit* units;
  const int32_t* block_tables;
  void* out;          // [tokens, heads, 512]
  float* lse;         // [tokens, heads] or null
  float* part_o;      // [parts, heads, 512]
  float* part_lse;    // [parts, heads]
  int* status;
  int32_t heads;
  int32_t max_blocks;
  int32_t block_size;
  int32_t oob_row;
  float scale_log2;
};

__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T>
__global__ void __launch_bounds__(192, 1)
    mla_kernel(const __grid_constant__ CUtensorMap tmQn, const __grid_constant__ CUtensorMap tmQr,
               const __grid_constant__ CUtensorMap tmKV, const __grid_constant__ CUtensorMap tmKR, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kQBytes;
  uint8_t* sP = sKV + kStages * kKvBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kPBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* s_free = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* o_done = bars + 8;
  uint64_t* fin = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNBars);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const MlaUnit u = p.units[blockIdx.x];
  const int n = u.n_tiles;
  int* status = p.status;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
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

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // the whole warp walks the tiles (warp-uniform values); one elected lane issues the copies
    const bool leader = elect_one();
    const int h0 = u.group * kHeadsPerCta;
    if (leader) {
      tma_prefetch_desc(&tmQn);
      tma_prefetch_desc(&tmQr);
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmKR);
      mbar_expect_tx(q_full, kQBytes);
      for (int cb = 0; cb < 8; ++cb) tma_load_3d(sQ + cb * kBlk, &tmQn, q_full, cb * 64, h0, u.token);
      tma_load_3d(sQ + 8 * kBlk, &tmQr, q_full, 0, h0, u.token);
    }
    const int32_t* bt = p.block_tables + (size_t)u.b * p.max_blocks;
    const int bs = p.block_size;
    const int box_rows = bs < kTileKeys ? bs : kTileKeys;
    const int n_pages = (u.last_key + 1 + bs - 1) / bs;
    bool ok = true;
    int issued = 0;
    for (int j = 0; j < n && ok; ++j) {
      const int s = j & 1;
      if (j >= kStages &&
          !__all_sync(0xffffffffu, mbar_wait(kv_empty + s, ((j >> 1) - 1) & 1, status, kDevTimeoutKEmpty))) {
        ok = false;
        break;
      }
      uint8_t* dst = sKV + s * kKvBytes;
      if (leader) mbar_expect_tx(kv_full + s, kKvBytes);
      const int j0 = u.kv_begin + j * kTileKeys;
      for (int r0 = 0; r0 < kTileKeys; r0 += box_rows) {
        const int pos = j0 + r0;
        const int pg = pos / bs;
        const int row = pg < n_pages ? bt[pg] * bs + (pos % bs) : p.oob_row;  // past the last page: zeros
        if (leader) {
          for (int cb = 0; cb < 8; ++cb) tma_load_2d(dst + cb * kBlk + r0 * 128, &tmKV, kv_full + s, cb * 64, row);
          tma_load_2d(dst + 8 * kBlk + r0 * 128, &tmKR, kv_full + s, 0, row);
        }
      }
      issued = j + 1;
    }
    for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j)
      mbar_wait(kv_full + (j & 1), (j >> 1) & 1, status, kDevTimeoutKFull);
    mbar_wait(q_full, 0, status, kDevTimeoutQ);
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp walks the schedule with warp-uniform descriptors; one elected lane issues
    const bool leader = elect_one();
    constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    constexpr uint32_t idesc_qk = instr_desc(fmt, false, false, 64, kTileKeys);
    constexpr uint32_t idesc_pv = instr_desc(fmt, false, true, 64, 256);
    // base descriptors; a step adds its byte offset >> 4 to the start-address field
    const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
    const uint64_t dkv = smem_desc_sw128(smem_addr(sKV), 16, 1024);
    const uint64_t dv = smem_desc(smem_addr(sKV), kBlk, 1024, 2);  // ctKV as the MN-major V operand
    const uint64_t dp = smem_desc_sw128(smem_addr(sP), 16, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity, int code) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, code));
    };
    auto commit = [&](uint64_t* bar) {
      if (leader) mma_commit(bar);
    };
    bool ok = wait_all(q_full, 0, kDevTimeoutQ);
    for (int j = 0; j <= n && ok; ++j) {
      if (j < n) {
        if (!wait_all(kv_full + (j & 1), (j >> 1) & 1, kDevTimeoutKFull)) break;
        if (j >= 1 && !wait_all(s_free, (j - 1) & 1, kDevTimeoutSFree)) break;
        tc_fence_after();
        if (leader) {
          const uint64_t kv0 = dkv + (uint64_t)((j & 1) * kKvBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 576 / 16; ++kk) {
            const uint64_t off = ((kk >> 2) * kBlk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kSCol, dq + off, kv0 + off, idesc_qk, kk > 0, false);
          }
        }
        commit(s_full);
      }
      if (j >= 1) {
        const int jj = j - 1;
        if (!wait_all(p_full, jj & 1, kDevTimeoutPFull)) break;
        tc_fence_after();
        if (leader) {
          const uint64_t v0 = dv + (uint64_t)((jj & 1) * kKvBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < kTileKeys / 16; ++kk) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // V = ctKV columns [256h, 256h+256): four 64-wide column blocks, MN-major
              mma_ss(tmem + ((uint32_t)(16 * h) << 16), dp + ((kk * 32) >> 4),
                     v0 + ((4 * h * kBlk + kk * 16 * 128) >> 4), idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u, false);
            }
          }
        }
        commit(kv_empty + (jj & 1));
        commit(o_done);
      }
    }
    commit(fin);
    wait_all(fin, 0, kDevTimeoutFinal);
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const bool upper = lane >= 16;            // lanes 16..31 hold the upper 256 output columns
    const int hl = (warp * 16) + (lane & 15); // head within the group
    const int head = u.group * kHeadsPerCta + hl;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float scale = p.scale_log2;
    const bool raw_max = scale > 0.f;  // max of the raw scores, scale folded into the exponent
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, j & 1, status, kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      float x[kTileKeys];
#pragma unroll
      for (int c32 = 0; c32 < kTileKeys / 32; ++c32) {
        uint32_t regs[32];
        tmem_ld32(tmem + lane_base + kSCol + c32 * 32, regs);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c32 * 32 + c] = __uint_as_float(regs[c]);
      }
      tc_fence_before();
      mbar_arrive(s_free);
      const int lim = u.last_key - (u.kv_begin + j * kTileKeys);  // columns c <= lim are allowed
      if (!raw_max) {
#pragma unroll
        for (int c = 0; c < kTileKeys; ++c) x[c] *= scale;
      }
      if (__any_sync(0xffffffffu, lim < kTileKeys - 1)) {  // only a range's last tile can hold masked keys
#pragma unroll
        for (int c = 0; c < kTileKeys; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
      }
      float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
      for (int c = 4; c < kTileKeys; c += 8) {
        mx0 = max3(mx0, x[c], x[c + 1]);
        mx1 = max3(mx1, x[c + 2], x[c + 3]);
        mx2 = max3(mx2, x[c + 4], x[c + 5]);
        mx3 = max3(mx3, x[c + 6], x[c + 7]);
      }
      float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      if (raw_max) mx *= scale;
      const float m_new = fmaxf(m_run, mx);
      float alpha = 1.f;
      if (m_new - m_run > kRescaleThreshold) {
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
      }
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
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status, kDevTimeoutODone));
        if (!ok) break;
        tc_fence_after();
        // lanes 16..31 scale the upper half of the heads owned by lanes 0..15
        const float a_row = __shfl_sync(0xffffffffu, alpha, lane & 15);
        if (__any_sync(0xffffffffu, a_row != 1.f)) {
#pragma unroll
          for (int c32 = 0; c32 < 256 / 32; ++c32) {
            uint32_t regs[32];
            const uint32_t addr = tmem + lane_base + c32 * 32;
            tmem_ld32(addr, regs);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) regs[c] = __float_as_uint(__uint_as_float(regs[c]) * a_row);
            tmem_st32(addr, regs);
          }
          tmem_st_wait();
        }
      }
      if (!upper) {
        // P row hl: 64 keys x 16 bit = 128 bytes, K-major 128B-swizzled
        const uint32_t prow = smem_addr(sP) + hl * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(prow + ((ch ^ (hl & 7)) << 4), make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (n - 1) & 1, status, kDevTimeoutODone));
    if (ok) {
      tc_fence_after();
      const float l_row = __shfl_sync(0xffffffffu, l_run, lane & 15);
      const float m_row = __shfl_sync(0xffffffffu, m_run, lane & 15);
      const float inv_l = 1.f / l_row;
      const int col0 = upper ? 256 : 0;
      if (u.part < 0) {
        T* orow = reinterpret_cast<T*>(p.out) + ((size_t)u.token * p.heads + head) * kDNope + col0;
#pragma unroll
        for (int c32 = 0; c32 < 8; ++c32) {
          uint32_t regs[32];
          tmem_ld32(tmem + lane_base + c32 * 32, regs);
          tmem_ld_wait();
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 v;
            v.x = pack2(__uint_as_float(regs[v4 * 8 + 0]) * inv_l, __uint_as_float(regs[v4 * 8 + 1]) * inv_l, (T*)nullptr);
            v.y = pack2(__uint_as_float(regs[v4 * 8 + 2]) * inv_l, __uint_as_float(regs[v4 * 8 + 3]) * inv_l, (T*)nullptr);
            v.z = pack2(__uint_as_float(regs[v4 * 8 + 4]) * inv_l, __uint_as_float(regs[v4 * 8 + 5]) * inv_l, (T*)nullptr);
            v.w = pack2(__uint_as_float(regs[v4 * 8 + 6]) * inv_l, __uint_as_float(regs[v4 * 8 + 7]) * inv_l, (T*)nullptr);
            *reinterpret_cast<uint4*>(orow + c32 * 32 + v4 * 8) = v;
          }
        }
        if (!upper && p.lse) p.lse[(size_t)u.token * p.heads + head] = (m_row == -INFINITY ? 0.f : m_row) * kLn2 + logf(l_row);
      } else {
        float* prow = p.part_o + ((size_t)u.part * p.heads + head) * kDNope + col0;
#pragma unroll
        for (int c32 = 0; c32 < 8; ++c32) {
          uint32_t regs[32];
          tmem_ld32(tmem + lane_base + c32 * 32, regs);
          tmem_ld_wait();
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            *reinterpret_cast<float4*>(prow + c32 * 32 + v4 * 4) =
                make_float4(__uint_as_float(regs[v4 * 4 + 0]) * inv_l, __uint_as_float(regs[v4 * 4 + 1]) * inv_l,
                            __uint_as_float(regs[v4 * 4 + 2]) * inv_l, __uint_as_float(regs[v4 * 4 + 3]) * inv_l);
        }
        if (!upper)
          p.part_lse[(size_t)u.part * p.heads + head] = (m_row == -INFINITY ? 0.f : m_row) * kLn2 + logf(l_row);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge of the partial results of one token's key splits by their lse:
// lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.
// One CTA per (token, 8 heads); one warp per head, 16 output columns per lane.
template <typename T>
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaCombine* work, const MlaParams p) {
  const MlaCombine w = work[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y * 8 + warp;
  if (head >= p.heads) return;
  float m = -INFINITY;
  for (int s = 0; s < w.n_parts; ++s) m = fmaxf(m, p.part_lse[(size_t)(w.part_begin + s) * p.heads + head]);
  float l = 0.f;
  for (int s = 0; s < w.n_parts; ++s) l += __expf(p.part_lse[(size_t)(w.part_begin + s) * p.heads + head] - m);
  const float lse = m + __logf(l);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s = 0; s < w.n_parts; ++s) {
    const size_t pr = (size_t)(w.part_begin + s) * p.heads + head;
    const float wgt = __expf(p.part_lse[pr] - lse);
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

// rank-2 or rank-3 map with a 64-element (128-byte) inner box and 128B swizzle
bool encode(CUtensorMap* map, void* base, int32_t dtype, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dtype == ALA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base,
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
  if (cacheMode != ALA_MLA_CACHE_KROPE_CTKV)
    return mfail(err, n, ALA_UNSUPPORTED, "only cacheMode KROPE_CTKV (1) is built");
  if (calcType == ALA_MLA_CALC_RING || calcType == ALA_MLA_CALC_PREFILL)
    return mfail(err, n, ALA_UNSUPPORTED, "calcType RING and PREFILL are not built");
  if (calcType != ALA_MLA_CALC_UNDEFINED && calcType != ALA_MLA_CALC_SPEC)
    return mfail(err, n, ALA_INVALID_PARAM, "calcType must be 0..3");
  if (maskType == 3 || maskType == 4 || maskType == 5)
    return mfail(err, n, ALA_INVALID_PARAM, "ALiBi masks apply only to the encoder paths");
  if (maskType != ALA_MLA_MASK_UNDEFINED && maskType != ALA_MLA_MASK_SPEC)
    return mfail(err, n, maskType == ALA_MLA_MASK_FREE ? ALA_UNSUPPORTED : ALA_INVALID_PARAM,
                 "maskType must be UNDEFINED (0) or SPEC (1)");
  if (mask && mask->data) return mfail(err, n, ALA_INVALID_PARAM, "mask must be NULL: the spec mask is generated");
  if ((qkDescale && qkDescale->data) || (pvDescale && pvDescale->data))
    return mfail(err, n, ALA_INVALID_PARAM, "qkDescale/pvDescale must be NULL (int8 cache not built)");
  if (headNum <= 0) return mfail(err, n, ALA_INVALID_PARAM, "headNum must be > 0");
  if (headNum % 64 != 0) return mfail(err, n, ALA_UNSUPPORTED, "headNum must be a multiple of 64");
  if (kvHeadNum != 1) return mfail(err, n, ALA_UNSUPPORTED, "kvHeadNum must be 1");
  if (!std::isfinite(qkScale)) return mfail(err, n, ALA_INVALID_PARAM, "qkScale must be finite");
  const int32_t dt = qNope->dtype;
  if (dt != ALA_BF16 && dt != ALA_F16) return mfail(err, n, ALA_INVALID_DTYPE, "qNope must be bf16 or f16");
  if (qRope->dtype != dt || ctKV->dtype != dt || kRope->dtype != dt || attenOut->dtype != dt)
    return mfail(err, n, ALA_INVALID_DTYPE, "qRope, ctKV, kRope and attenOut must have qNope's dtype");
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
  if (!(bs > 0 && bs % 16 == 0 && (kTileKeys % bs == 0 || bs % kTileKeys == 0)))
    return mfail(err, n, ALA_UNSUPPORTED, "blockSize must be a multiple of 16 dividing 64, or a multiple of 64");
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
    sum_q += q;
  }
  if (sum_q != tokens) return mfail(err, n, ALA_INVALID_SHAPE, "sum(qseqlen) != tokens");
  if (ctKV->dims[0] * bs >= ((int64_t)1 << 31)) return mfail(err, n, ALA_UNSUPPORTED, "cache has more than 2^31 rows");

  plan->dtype = dt;
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

  // ---- schedule: per token, its allowed keys split into ranges of chunk_tiles 64-key tiles
  const int groups = headNum / kHeadsPerCta;
  int64_t total_tiles = 0;
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t t = 0; t < plan->qs[b]; ++t) total_tiles += (cl[b] - plan->qs[b] + t + 1 + kTileKeys - 1) / kTileKeys;
  total_tiles *= groups;
  // about three units per SM of a 148-SM part, each at least 8 tiles
  const int64_t target_units = 148 * 3;
  const int32_t chunk_tiles = (int32_t)std::max<int64_t>(8, (total_tiles + target_units - 1) / target_units);
  std::vector<MlaUnit> units;
  std::vector<MlaCombine> comb;
  int32_t token = 0, parts = 0;
  for (int32_t b = 0; b < batch; ++b) {
    for (int32_t t = 0; t < plan->qs[b]; ++t, ++token) {
      const int32_t last = cl[b] - plan->qs[b] + t;
      const int32_t tiles = (last + 1 + kTileKeys - 1) / kTileKeys;
      const int32_t splits = (tiles + chunk_tiles - 1) / chunk_tiles;
      const int32_t part0 = splits > 1 ? parts : -1;
      if (splits > 1) {
        comb.push_back(MlaCombine{token, parts, splits, 0});
        parts += splits;
      }
      for (int32_t s = 0; s < splits; ++s) {
        const int32_t t0 = s * chunk_tiles;
        const int32_t nt = std::min(chunk_tiles, tiles - t0);
        for (int32_t g = 0; g < groups; ++g)
          units.push_back(MlaUnit{b, token, t, g, t0 * kTileKeys, nt, last, splits > 1 ? part0 + s : -1});
      }
    }
  }
  std::stable_sort(units.begin(), units.end(), [](const MlaUnit& a, const MlaUnit& c) { return a.n_tiles > c.n_tiles; });
  plan->n_work = (int32_t)units.size();
  plan->n_splits_total = parts;
  plan->n_combine = (int32_t)comb.size();
  auto align = [](uint64_t x) { return (x + 255) / 256 * 256; };
  plan->off_work = 256;
  plan->off_rows = align(plan->off_work + sizeof(MlaUnit) * std::max<size_t>(units.size(), 1));
  plan->off_part_lse = align(plan->off_rows + sizeof(MlaCombine) * std::max<size_t>(comb.size(), 1));
  plan->off_part_o = align(plan->off_part_lse + sizeof(float) * (uint64_t)parts * headNum);
  plan->ws_size = align(plan->off_part_o + sizeof(float) * (uint64_t)parts * headNum * kDNope);
  plan->image_size = plan->off_part_lse;  // only the schedule is uploaded; partials are written by the kernel
  plan->image.assign(plan->image_size, 0);
  std::memcpy(plan->image.data() + plan->off_work, units.data(), sizeof(MlaUnit) * units.size());
  std::memcpy(plan->image.data() + plan->off_rows, comb.data(), sizeof(MlaCombine) * comb.size());
  return ALA_OK;
}

int mla_run(MlaPlan* plan, void* workspace, cudaStream_t stream, char* err, size_t n) {
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return mfail(err, n, ALA_INVALID_PARAM, "workspace must be 256-byte aligned");
  if (!plan->maps_ready) {
    const int es = 2;
    const cuuint64_t rows = (cuuint64_t)plan->num_blocks * plan->block_size;
    const cuuint32_t kv_box_rows = (cuuint32_t)std::min(plan->block_size, kTileKeys);
    cuuint64_t qn_dims[3] = {512, (cuuint64_t)plan->heads, (cuuint64_t)plan->tokens};
    cuuint64_t qn_str[2] = {512 * es, (cuuint64_t)plan->heads * 512 * es};
    cuuint64_t qr_dims[3] = {64, (cuuint64_t)plan->heads, (cuuint64_t)plan->tokens};
    cuuint64_t qr_str[2] = {64 * es, (cuuint64_t)plan->heads * 64 * es};
    cuuint32_t q_box[3] = {64, kHeadsPerCta, 1};
    cuuint64_t kv_dims[2] = {512, rows};
    cuuint64_t kv_str[1] = {512 * es};
    cuuint64_t kr_dims[2] = {64, rows};
    cuuint64_t kr_str[1] = {64 * es};
    cuuint32_t kv_box[2] = {64, kv_box_rows};
    if (!encode(&plan->tmQn, plan->q_nope, plan->dtype, 3, qn_dims, qn_str, q_box) ||
        !encode(&plan->tmQr, plan->q_rope, plan->dtype, 3, qr_dims, qr_str, q_box) ||
        !encode(&plan->tmKV, plan->ct_kv, plan->dtype, 2, kv_dims, kv_str, kv_box) ||
        !encode(&plan->tmKR, plan->k_rope, plan->dtype, 2, kr_dims, kr_str, kv_box))
      return mfail(err, n, ALA_CUDA_ERROR, "cuTensorMapEncodeTiled failed (pointers must be 16-byte aligned)");
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
    return mfail(err, n, ALA_CUDA_ERROR, "schedule upload failed");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  MlaParams p{};
  p.units = reinterpret_cast<const MlaUnit*>(ws + plan->off_work);
  p.block_tables = plan->block_tables;
  p.out = plan->out;
  p.lse = plan->lse;
  p.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
  p.part_lse = reinterpret_cast<float*>(ws + plan->off_part_lse);
  p.status = reinterpret_cast<int*>(ws);
  p.heads = plan->heads;
  p.max_blocks = plan->max_blocks;
  p.block_size = plan->block_size;
  p.oob_row = (int32_t)(plan->num_blocks * plan->block_size);
  p.scale_log2 = plan->qk_scale * kLog2e;
  auto kern = plan->dtype == ALA_F16 ? mla_kernel<__half> : mla_kernel<__nv_bfloat16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e == cudaSuccess && plan->n_work > 0) {
    kern<<<plan->n_work, 192, kSmem, stream>>>(plan->tmQn, plan->tmQr, plan->tmKV, plan->tmKR, p);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && plan->n_combine > 0) {
    auto ck = plan->dtype == ALA_F16 ? mla_combine_kernel<__half> : mla_combine_kernel<__nv_bfloat16>;
    dim3 grid(plan->n_combine, (plan->heads + 7) / 8);
    ck<<<grid, 256, 0, stream>>>(reinterpret_cast<const MlaCombine*>(ws + plan->off_rows), p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return mfail(err, n, ALA_CUDA_ERROR, cudaGetErrorString(e));
  return ALA_OK;
}

MlaPlan::~MlaPlan() {
  if (pinned) cudaFreeHost(pinned);
}

}  // namespace ala
