// PhaseQuant with axis scales and recursive residual stages
// ("Fairy2i write-up" §3.1, §3.2, §4.1).
//
// One launch per stage t covers every tensor of the call.  Each thread takes
// four quads (4 consecutive weights = one code byte) strided by 32 within its
// warp, so every load and store instruction of a warp is contiguous:
//   1. residual r_t = w - sum_{u<t} w_hat_u, rebuilt in float64 from w and the
//      already written codes and float32 scales of the earlier stages (w is
//      read again each stage: the per-tensor scale of stage t-1 is a global
//      dependency, and the fp32 weights of a layer do not fit on chip);
//   2. the sector k of r_t by exact comparisons (no atan2);
//   3. four codes packed into one byte;
//   4. per-class sums S_re = sum |Re r| over k even, S_im = sum |Im r| over k
//      odd and the class-0 count, in float64 / integer, reduced per block in a
//      fixed order into workspace partials.
// The last block of a tensor to finish (atomic ticket) reduces the partials in
// block order and writes s_re = S_re/C_re, s_im = S_im/C_im (0 for an empty
// class) rounded to float32, then re-arms the ticket for the next stage.
// No block waits on another, so nothing can hang.
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kQThreads = 256;
constexpr int kQuadsPerThread = 4;
constexpr int kQuadsPerBlock = kQThreads * kQuadsPerThread;

struct QPartial {
  double s_re;
  double s_im;
  unsigned long long c_re;
  unsigned long long pad;
};

struct QTensorArg {
  const float* w_re;
  const float* w_im;
  uint8_t* codes;        // [T][nquads]
  float* scales;         // [T][2]
  QPartial* partials;    // [nblocks]
  unsigned int* ticket;  // one counter
  int64_t nquads;        // N*K/4
  int64_t block_begin;   // first global block of this tensor
  int64_t nblocks;
};

struct QParams {
  QTensorArg t[IFQ_MAX_GROUP];
  int count;
  int stage;  // 0-based stage being computed
  uint32_t* status;
};

// Sector of w = a + ib: 0 -> 1, 1 -> i, 2 -> -1, 3 -> -i.  Ties on a diagonal go
// counter-clockwise, w = 0 -> 0.  Exact in any IEEE precision the inputs fit.
template <typename F>
__device__ __forceinline__ uint32_t phase_sector(F a, F b) {
  const F aa = fabs(a), ab = fabs(b);
  if (b > aa || (a == b && b > F(0))) return 1u;
  if (-a > ab || (b == -a && a < F(0))) return 2u;
  if (-b > aa || (a == b && b < F(0))) return 3u;
  return 0u;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  return v;
}

// Fixed-order block reduction of three values; result valid in thread 0.
__device__ __forceinline__ void block_sum3(double& a, double& b, unsigned long long& c) {
  __shared__ double sa[kQThreads / 32], sb[kQThreads / 32];
  __shared__ unsigned long long sc[kQThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = warp_sum(a);
  b = warp_sum(b);
  c = warp_sum(c);
  if (lane == 0) {
    sa[warp] = a;
    sb[warp] = b;
    sc[warp] = c;
  }
  __syncthreads();
  if (warp == 0) {
    a = lane < kQThreads / 32 ? sa[lane] : 0.0;
    b = lane < kQThreads / 32 ? sb[lane] : 0.0;
    c = lane < kQThreads / 32 ? sc[lane] : 0ull;
    a = warp_sum(a);
    b = warp_sum(b);
    c = warp_sum(c);
  }
  __syncthreads();
}

template <bool FIRST>
__global__ void __launch_bounds__(kQThreads) quant_stage_kernel(const __grid_constant__ QParams p) {
  // Find this block's tensor (at most IFQ_MAX_GROUP entries, uniform per block).
  int ti = 0;
  while (ti + 1 < p.count && (int64_t)blockIdx.x >= p.t[ti + 1].block_begin) ++ti;
  const QTensorArg& T = p.t[ti];
  const int stage = p.stage;
  const int64_t blk = (int64_t)blockIdx.x - T.block_begin;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t quad0 = blk * kQuadsPerBlock + (int64_t)warp * (32 * kQuadsPerThread) + lane;

  double s_prev_re[IFQ_MAX_STAGES], s_prev_im[IFQ_MAX_STAGES];
  if (!FIRST) {
#pragma unroll
    for (int u = 0; u < IFQ_MAX_STAGES; ++u) {
      if (u < stage) {
        s_prev_re[u] = (double)__ldg(T.scales + 2 * u);
        s_prev_im[u] = (double)__ldg(T.scales + 2 * u + 1);
      }
    }
  }

  double S_re = 0.0, S_im = 0.0;
  unsigned long long C_re = 0;
  int bad = 0;

#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
    if (quad >= T.nquads) break;
    const float4 vr = __ldcs(reinterpret_cast<const float4*>(T.w_re) + quad);
    const float4 vi = __ldcs(reinterpret_cast<const float4*>(T.w_im) + quad);
    const float wr[4] = {vr.x, vr.y, vr.z, vr.w};
    const float wi[4] = {vi.x, vi.y, vi.z, vi.w};
    uint32_t prev_bytes[IFQ_MAX_STAGES];
    if (!FIRST) {
#pragma unroll
      for (int u = 0; u < IFQ_MAX_STAGES; ++u)
        if (u < stage) prev_bytes[u] = __ldg(T.codes + (int64_t)u * T.nquads + quad);
    }
    uint32_t byte = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool finite = isfinite(wr[e]) && isfinite(wi[e]);
      bad |= !finite;
      uint32_t k;
      if (FIRST) {
        const float a = finite ? wr[e] : 0.0f;
        const float b = finite ? wi[e] : 0.0f;
        k = phase_sector(a, b);
        if ((k & 1u) == 0u) {
          S_re += (double)fabsf(a);
          ++C_re;
        } else {
          S_im += (double)fabsf(b);
        }
      } else {
        double a = finite ? (double)wr[e] : 0.0;
        double b = finite ? (double)wi[e] : 0.0;
#pragma unroll
        for (int u = 0; u < IFQ_MAX_STAGES; ++u) {
          if (u < stage) {
            const uint32_t ku = (prev_bytes[u] >> (2 * e)) & 3u;
            const double sgn = (ku & 2u) ? -1.0 : 1.0;
            const double br = (ku & 1u) ? 0.0 : sgn;
            const double bi = (ku & 1u) ? sgn : 0.0;
            a = a - s_prev_re[u] * br;
            b = b - s_prev_im[u] * bi;
          }
        }
        k = phase_sector(a, b);
        if ((k & 1u) == 0u) {
          S_re += fabs(a);
          ++C_re;
        } else {
          S_im += fabs(b);
        }
      }
      byte |= k << (2 * e);
    }
    T.codes[(int64_t)stage * T.nquads + quad] = (uint8_t)byte;
  }

  if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(p.status, IFQ_DEV_NONFINITE);

  block_sum3(S_re, S_im, C_re);
  __shared__ int am_last;
  if (threadIdx.x == 0) {
    QPartial part;
    part.s_re = S_re;
    part.s_im = S_im;
    part.c_re = C_re;
    part.pad = 0;
    T.partials[blk] = part;
    __threadfence();
    const unsigned prev = atomicAdd(T.ticket, 1u);
    am_last = (prev == (unsigned)(T.nblocks - 1));
  }
  __syncthreads();
  if (!am_last) return;

  // Last block of this tensor: reduce all partials in a fixed order.
  __threadfence();
  double a = 0.0, b = 0.0;
  unsigned long long c = 0;
  for (int64_t i = threadIdx.x; i < T.nblocks; i += kQThreads) {
    const QPartial* pp = T.partials + i;
    a += __ldcg(&pp->s_re);
    b += __ldcg(&pp->s_im);
    c += __ldcg(&pp->c_re);
  }
  block_sum3(a, b, c);
  if (threadIdx.x == 0) {
    const unsigned long long total = (unsigned long long)T.nquads * 4ull;
    const unsigned long long c_im = total - c;
    const float s_re = c > 0 ? (float)(a / (double)c) : 0.0f;
    const float s_im = c_im > 0 ? (float)(b / (double)c_im) : 0.0f;
    T.scales[2 * stage] = s_re;
    T.scales[2 * stage + 1] = s_im;
    *T.ticket = 0u;  // re-arm for the next stage launch
  }
}

}  // namespace

int64_t quant_blocks_for(int64_t N, int64_t K) {
  const int64_t nquads = N * K / 4;
  return (nquads + kQuadsPerBlock - 1) / kQuadsPerBlock;
}

// Workspace: [tickets: 16 B per tensor, padded to 256 B][partials of tensor 0][tensor 1]...
size_t quant_workspace_bytes(const ifq_qtensor* t, int count) {
  size_t bytes = ((size_t)count * 16 + 255) / 256 * 256;
  for (int i = 0; i < count; ++i) bytes += (size_t)quant_blocks_for(t[i].N, t[i].K) * sizeof(QPartial);
  return bytes;
}

cudaError_t launch_quantize(const ifq_qtensor* t, int count, int T, void* ws, uint32_t* dev_status, cudaStream_t s) {
  QParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.status = dev_status;
  char* base = static_cast<char*>(ws);
  const size_t ticket_bytes = ((size_t)count * 16 + 255) / 256 * 256;
  char* part = base + ticket_bytes;
  int64_t blocks = 0;
  for (int i = 0; i < count; ++i) {
    QTensorArg& a = p.t[i];
    a.w_re = t[i].w_re;
    a.w_im = t[i].w_im;
    a.codes = t[i].codes;
    a.scales = t[i].scales;
    a.nquads = t[i].N * t[i].K / 4;
    a.nblocks = quant_blocks_for(t[i].N, t[i].K);
    a.block_begin = blocks;
    a.ticket = reinterpret_cast<unsigned int*>(base + 16 * i);
    a.partials = reinterpret_cast<QPartial*>(part);
    part += (size_t)a.nblocks * sizeof(QPartial);
    blocks += a.nblocks;
  }
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaMemsetAsync(base, 0, ticket_bytes, s);
  if (e != cudaSuccess) return e;
  for (int st = 0; st < T; ++st) {
    p.stage = st;
    if (st == 0)
      quant_stage_kernel<true><<<(unsigned)blocks, kQThreads, 0, s>>>(p);
    else
      quant_stage_kernel<false><<<(unsigned)blocks, kQThreads, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace ifq
