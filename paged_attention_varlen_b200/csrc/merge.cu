// merge.cu -- merge of two partial attention results by their log-sum-exp
// (ATB "MLA" page, parameter table, rows calcType and lse: in ring mode the
// operator returns the lse of the keys it saw, so the results over disjoint
// key ranges can be combined).  For one row with partial outputs O_a, O_b
// (each normalised over its own keys) and natural-log lse_a, lse_b:
//   lse = log(exp(lse_a) + exp(lse_b)),
//   O   = exp(lse_a - lse) O_a + exp(lse_b - lse) O_b.
// A row whose two lse are both -inf (no allowed key on either side) gets
// lse = -inf and O = 0.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "internal.h"

namespace ala {

namespace {

__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* d) { *d = __float2bfloat16_rn(v); }
__device__ __forceinline__ void from_f(float v, __half* d) { *d = __float2half_rn(v); }
__device__ __forceinline__ void from_f(float v, float* d) { *d = v; }

// One warp per row; rows are independent, so out / lse may alias either input.
template <typename T>
__global__ void __launch_bounds__(256) lse_merge_kernel(const T* a, const float* lse_a, const T* b, const float* lse_b,
                                                        T* out, float* lse, int64_t rows, int d) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float la = lse_a[row], lb = lse_b[row];
  const float m = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f, l = -INFINITY;
  if (m != -INFINITY) {
    const float s = expf(la - m) + expf(lb - m);  // exp(-inf) = 0
    l = m + logf(s);
    wa = expf(la - l);
    wb = expf(lb - l);
  }
  const T* ra = a + row * d;
  const T* rb = b + row * d;
  T* ro = out + row * d;
  // read every element of the row before writing any, so out may alias a or b
  constexpr int kMaxPerLane = 32;  // d <= 1024
  float acc[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int c = i * 32 + lane;
    acc[i] = c < d ? wa * to_f(ra[c]) + wb * to_f(rb[c]) : 0.f;
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int c = i * 32 + lane;
    if (c < d) from_f(acc[i], ro + c);
  }
  if (lane == 0) lse[row] = l;
}

}  // namespace

cudaError_t launch_lse_merge(int32_t dtype, const void* a, const float* lse_a, const void* b, const float* lse_b,
                             void* out, float* lse, int64_t rows, int d, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (dtype == kBF16)
    lse_merge_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a), lse_a, static_cast<const __nv_bfloat16*>(b), lse_b,
        static_cast<__nv_bfloat16*>(out), lse, rows, d);
  else if (dtype == kF16)
    lse_merge_kernel<__half><<<grid, 256, 0, stream>>>(static_cast<const __half*>(a), lse_a,
                                                       static_cast<const __half*>(b), lse_b,
                                                       static_cast<__half*>(out), lse, rows, d);
  else
    lse_merge_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(a), lse_a,
                                                      static_cast<const float*>(b), lse_b, static_cast<float*>(out),
                                                      lse, rows, d);
  return cudaGetLastError();
}

}  // namespace ala
