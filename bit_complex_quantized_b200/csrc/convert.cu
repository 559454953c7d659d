// Widely-linear transform of a real layer into (U, W) ("Fairy2i write-up" §2.1).
//
// R is [2n][2m] float32 row-major (rows = outputs).  For each complex position
// (i, j): U = (R11+R22)/2 + i (R21-R12)/2, W = (R11-R22)/2 + i (R12+R21)/2.
// The sum or difference is rounded once to float32 and then halved exactly,
// so each output equals the exact value rounded to nearest-even.
//
// HBM-bound: 16 B read + 16 B written per complex position.  Each thread
// handles four consecutive j with 128-bit loads of the four quadrant rows and
// 128-bit stores to the four planes; blockIdx.y walks rows.
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

__device__ __forceinline__ float half_sum(float a, float b) { return __fmul_rn(0.5f, __fadd_rn(a, b)); }
__device__ __forceinline__ float half_diff(float a, float b) { return __fmul_rn(0.5f, __fsub_rn(a, b)); }

__global__ void __launch_bounds__(256) widely_linear_vec4_kernel(const float* __restrict__ R, int64_t n, int64_t m,
                                                                  float* __restrict__ U_re, float* __restrict__ U_im,
                                                                  float* __restrict__ W_re,
                                                                  float* __restrict__ W_im) {
  const int64_t m4 = m >> 2;
  for (int64_t i = blockIdx.y; i < n; i += gridDim.y) {
    const float4* top = reinterpret_cast<const float4*>(R + i * 2 * m);
    const float4* bot = reinterpret_cast<const float4*>(R + (i + n) * 2 * m);
    for (int64_t j4 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j4 < m4; j4 += (int64_t)gridDim.x * blockDim.x) {
      const float4 r11 = __ldcs(top + j4);
      const float4 r12 = __ldcs(top + m4 + j4);
      const float4 r21 = __ldcs(bot + j4);
      const float4 r22 = __ldcs(bot + m4 + j4);
      const int64_t o = i * m4 + j4;
      reinterpret_cast<float4*>(U_re)[o] = make_float4(half_sum(r11.x, r22.x), half_sum(r11.y, r22.y),
                                                       half_sum(r11.z, r22.z), half_sum(r11.w, r22.w));
      reinterpret_cast<float4*>(U_im)[o] = make_float4(half_diff(r21.x, r12.x), half_diff(r21.y, r12.y),
                                                       half_diff(r21.z, r12.z), half_diff(r21.w, r12.w));
      reinterpret_cast<float4*>(W_re)[o] = make_float4(half_diff(r11.x, r22.x), half_diff(r11.y, r22.y),
                                                       half_diff(r11.z, r22.z), half_diff(r11.w, r22.w));
      reinterpret_cast<float4*>(W_im)[o] = make_float4(half_sum(r12.x, r21.x), half_sum(r12.y, r21.y),
                                                       half_sum(r12.z, r21.z), half_sum(r12.w, r21.w));
    }
  }
}

__global__ void __launch_bounds__(256) widely_linear_scalar_kernel(const float* __restrict__ R, int64_t n, int64_t m,
                                                                    float* __restrict__ U_re,
                                                                    float* __restrict__ U_im,
                                                                    float* __restrict__ W_re,
                                                                    float* __restrict__ W_im) {
  for (int64_t i = blockIdx.y; i < n; i += gridDim.y) {
    const float* top = R + i * 2 * m;
    const float* bot = R + (i + n) * 2 * m;
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < m; j += (int64_t)gridDim.x * blockDim.x) {
      const float r11 = top[j], r12 = top[m + j], r21 = bot[j], r22 = bot[m + j];
      const int64_t o = i * m + j;
      U_re[o] = half_sum(r11, r22);
      U_im[o] = half_diff(r21, r12);
      W_re[o] = half_diff(r11, r22);
      W_im[o] = half_sum(r12, r21);
    }
  }
}

}  // namespace

cudaError_t launch_widely_linear(const float* R, int64_t n, int64_t m, float* U_re, float* U_im, float* W_re,
                                 float* W_im, cudaStream_t s) {
  const int threads = 256;
  const bool vec = (m % 4) == 0;
  const int64_t cols = vec ? m / 4 : m;
  int64_t bx = (cols + threads - 1) / threads;
  if (bx > 1024) bx = 1024;
  int64_t by = n < 65535 ? n : 65535;
  dim3 grid((unsigned)bx, (unsigned)by);
  if (vec)
    widely_linear_vec4_kernel<<<grid, threads, 0, s>>>(R, n, m, U_re, U_im, W_re, W_im);
  else
    widely_linear_scalar_kernel<<<grid, threads, 0, s>>>(R, n, m, U_re, U_im, W_re, W_im);
  return cudaGetLastError();
}

}  // namespace ifq
