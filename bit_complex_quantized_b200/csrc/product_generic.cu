// Decode and prefill product for layers whose width K is a multiple of 4 but not of 64
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2).  The tensor-core kernels stream 64-position
// steps through tensor copies whose row strides must be multiples of 16 bytes; a code row of such a
// layer (K/4 bytes) is not, so these layers take this plain CUDA-core kernel instead.  No configured
// workload has such a width: the kernel exists so that every tensor the quantizer accepts
// (K % 4 == 0) can also be multiplied.
//
// One thread per (token, output): for each (stage, branch) the four per-class sums
//     P_rr = sum Br x_re, P_ri = sum Br x_im, P_ir = sum Bi x_re, P_ii = sum Bi x_im
// are formed by signed additions in float64 (no weight multiplies), the scales are applied, and the
// (stage, branch) terms are added in float32 as in the other kernels:
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
// then the optional rotation.  Non-finite activations propagate to the outputs and set
// IFQ_DEV_NONFINITE.
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kGThreads = 128;

struct GenLayer {
  const uint8_t* codes[2];
  const float* scales[2];
  const uint16_t* x[2];
  float* y[2];
  const float* rot[2];
  int64_t N, K;
  int64_t block_begin;  // first block of this layer in the grid's x dimension
  int nbranch;
};

struct GenParams {
  GenLayer L[IFQ_MAX_GROUP];
  int count, T;
  int64_t rows;
  uint32_t* status;
};

__device__ __forceinline__ double bf16d(uint16_t h) { return (double)__uint_as_float((uint32_t)h << 16); }

__global__ void __launch_bounds__(kGThreads) product_generic_kernel(const __grid_constant__ GenParams p) {
  int li = 0;
  while (li + 1 < p.count && (int64_t)blockIdx.x >= p.L[li + 1].block_begin) ++li;
  const GenLayer& L = p.L[li];
  const int64_t n = ((int64_t)blockIdx.x - L.block_begin) * kGThreads + threadIdx.x;
  if (n >= L.N) return;
  for (int64_t m = blockIdx.y; m < p.rows; m += gridDim.y) {
    const uint16_t* xr = L.x[0] + m * L.K;
    const uint16_t* xi = L.x[1] + m * L.K;
    const int64_t kb = L.K / 4;
    float yre = 0.0f, yim = 0.0f;
    bool bad = false;
    for (int t = 0; t < p.T; ++t)
      for (int br = 0; br < L.nbranch; ++br) {
        const uint8_t* row = L.codes[br] + ((int64_t)t * L.N + n) * kb;
        double rr = 0.0, ri = 0.0, ir = 0.0, ii = 0.0;
        for (int64_t q = 0; q < kb; ++q) {
          const uint32_t byte = row[q];
  #pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t k = (byte >> (2 * e)) & 3u;   // bit 0: axis, bit 1: sign
            const double a = bf16d(xr[4 * q + e]), b = bf16d(xi[4 * q + e]);
            const double sa = (k & 2u) ? -a : a, sb = (k & 2u) ? -b : b;
            if (k & 1u) {
              ir += sa;
              ii += sb;
            } else {
              rr += sa;
              ri += sb;
            }
          }
        }
        const float s_re = L.scales[br][2 * t], s_im = L.scales[br][2 * t + 1];
        const float P_rr = (float)rr, P_ri = (float)ri, P_ir = (float)ir, P_ii = (float)ii;
        if (br == 0) {
          yre += s_re * P_rr - s_im * P_ii;
          yim += s_re * P_ri + s_im * P_ir;
        } else {
          yre += s_re * P_rr + s_im * P_ii;
          yim += s_im * P_ir - s_re * P_ri;
        }
      }
    bad = !isfinite(yre) || !isfinite(yim);
    const int64_t off = m * L.N + n;
    if (L.rot[0]) {
      const float cr = L.rot[0][off], ci = L.rot[1][off];
      const float r = cr * yre - ci * yim, im = cr * yim + ci * yre;
      yre = r;
      yim = im;
    }
    L.y[0][off] = yre;
    L.y[1][off] = yim;
    if (bad) set_status(p.status, IFQ_DEV_NONFINITE);
  }
}

}  // namespace

cudaError_t launch_product_generic(const ifq_layer* Ls, int count, int T, int64_t rows, uint32_t* dev_status,
                                   cudaStream_t s) {
  GenParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.rows = rows;
  p.status = dev_status;
  int64_t blocks = 0;
  for (int i = 0; i < count; ++i) {
    GenLayer& a = p.L[i];
    a.codes[0] = Ls[i].codes_u;
    a.codes[1] = Ls[i].codes_w;
    a.scales[0] = Ls[i].scales_u;
    a.scales[1] = Ls[i].scales_w;
    a.nbranch = Ls[i].codes_w ? 2 : 1;
    a.x[0] = Ls[i].x_re;
    a.x[1] = Ls[i].x_im;
    a.y[0] = Ls[i].y_re;
    a.y[1] = Ls[i].y_im;
    a.rot[0] = Ls[i].rot_re;
    a.rot[1] = Ls[i].rot_im;
    a.N = Ls[i].N;
    a.K = Ls[i].K;
    a.block_begin = blocks;
    blocks += (Ls[i].N + kGThreads - 1) / kGThreads;
  }
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  product_generic_kernel<<<dim3((unsigned)blocks, (unsigned)(rows < 65535 ? rows : 65535)), kGThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ifq
