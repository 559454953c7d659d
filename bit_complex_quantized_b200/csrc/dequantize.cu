// Dequantized weights for quantization-aware training: W_hat = sum_t (s_re,t Re b_t
// + i s_im,t Im b_t) as bf16 planes ("Fairy2i write-up" §3.2, §4.1; "iFairy talk
// notes" §2.2.1: training runs the forward pass on the quantized weights, whose
// quantization noise the model learns to absorb, and passes gradients straight
// through).  The straight-through backward is the identity on the gradient, so it
// has no kernel.
//
// Per entry the stage terms are added in float32 in stage order, starting from +0
// (each term is +-s or 0, so the first addition is exact), and the sum is rounded
// once to bf16 (nearest-even).  HBM-bound: T/4 bytes of codes read and 4 bytes of
// bf16 written per complex entry.  Each thread takes four consecutive quads: one
// 32-bit code word per stage in, 32 bytes per plane out (two 16-byte stores), so a
// warp moves 128 contiguous code bytes and 1 KB per plane.  A tensor whose quad
// count is not a multiple of 4 takes the same quads one byte at a time.
#include <cuda_bf16.h>

#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kDThreads = 256;
constexpr int kDQuads = 4;
constexpr int kDQuadsPerBlock = kDThreads * kDQuads;

struct DTensorArg {
  const uint8_t* codes;   // [T][nquads]
  const float* scales;    // [T][2]
  uint16_t* w[2];         // [N][K] bf16: re, im
  int64_t nquads;
  int64_t block_begin;
};

struct DParams {
  DTensorArg t[IFQ_MAX_GROUP];
  int count;
  int T;
};

__device__ __forceinline__ uint32_t bf16_pair(float lo, float hi) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

__global__ void __launch_bounds__(kDThreads) dequant_kernel(const __grid_constant__ DParams p) {
  int ti = 0;
  while (ti + 1 < p.count && (int64_t)blockIdx.x >= p.t[ti + 1].block_begin) ++ti;
  const DTensorArg& D = p.t[ti];
  const int64_t blk = (int64_t)blockIdx.x - D.block_begin;

  float sr[IFQ_MAX_STAGES], si[IFQ_MAX_STAGES];
#pragma unroll
  for (int t = 0; t < IFQ_MAX_STAGES; ++t) {
    sr[t] = t < p.T ? __ldg(D.scales + 2 * t) : 0.0f;
    si[t] = t < p.T ? __ldg(D.scales + 2 * t + 1) : 0.0f;
  }
  const int64_t quad0 = blk * kDQuadsPerBlock + (int64_t)threadIdx.x * kDQuads;  // four consecutive quads
  if (quad0 >= D.nquads) return;
  const bool whole = (D.nquads & 3) == 0;  // 32-bit code words are aligned, and all four quads exist
  uint32_t words[IFQ_MAX_STAGES];          // byte q of word t: quad quad0 + q of stage t
#pragma unroll
  for (int t = 0; t < IFQ_MAX_STAGES; ++t) {
    words[t] = 0u;
    if (t < p.T) {
      const uint8_t* src = D.codes + (int64_t)t * D.nquads + quad0;
      if (whole) {
        words[t] = __ldg(reinterpret_cast<const uint32_t*>(src));
      } else {
#pragma unroll
        for (int q = 0; q < kDQuads; ++q)
          if (quad0 + q < D.nquads) words[t] |= (uint32_t)__ldg(src + q) << (8 * q);
      }
    }
  }
  uint32_t ore[8], oim[8];  // 16 entries per plane as bf16 pairs
#pragma unroll
  for (int h = 0; h < 8; ++h) {  // entries 2h, 2h + 1
    float re[2] = {0.0f, 0.0f}, im[2] = {0.0f, 0.0f};
#pragma unroll
    for (int t = 0; t < IFQ_MAX_STAGES; ++t) {
      if (t >= p.T) break;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t k = (words[t] >> (2 * (2 * h + e))) & 3u;  // 0: 1, 1: i, 2: -1, 3: -i
        const float sc = (k & 1u) ? si[t] : sr[t];
        const float v = (k & 2u) ? -sc : sc;
        if (k & 1u)
          im[e] = __fadd_rn(im[e], v);
        else
          re[e] = __fadd_rn(re[e], v);
      }
    }
    ore[h] = bf16_pair(re[0], re[1]);
    oim[h] = bf16_pair(im[0], im[1]);
  }
  if (whole) {
    uint4* dre = reinterpret_cast<uint4*>(D.w[0] + quad0 * 4);
    uint4* dim = reinterpret_cast<uint4*>(D.w[1] + quad0 * 4);
    dre[0] = make_uint4(ore[0], ore[1], ore[2], ore[3]);
    dre[1] = make_uint4(ore[4], ore[5], ore[6], ore[7]);
    dim[0] = make_uint4(oim[0], oim[1], oim[2], oim[3]);
    dim[1] = make_uint4(oim[4], oim[5], oim[6], oim[7]);
  } else {
#pragma unroll
    for (int q = 0; q < kDQuads; ++q)
      if (quad0 + q < D.nquads) {
        reinterpret_cast<uint2*>(D.w[0])[quad0 + q] = make_uint2(ore[2 * q], ore[2 * q + 1]);
        reinterpret_cast<uint2*>(D.w[1])[quad0 + q] = make_uint2(oim[2 * q], oim[2 * q + 1]);
      }
  }
}

}  // namespace

cudaError_t launch_dequantize(const ifq_dqtensor* t, int count, int T, cudaStream_t s) {
  DParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  int64_t blocks = 0;
  for (int i = 0; i < count; ++i) {
    DTensorArg& a = p.t[i];
    a.codes = t[i].codes;
    a.scales = t[i].scales;
    a.w[0] = t[i].w_re;
    a.w[1] = t[i].w_im;
    a.nquads = t[i].N * t[i].K / 4;
    a.block_begin = blocks;
    blocks += (a.nquads + kDQuadsPerBlock - 1) / kDQuadsPerBlock;
  }
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dequant_kernel<<<(unsigned)blocks, kDThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ifq
