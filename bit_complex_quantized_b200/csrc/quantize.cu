// PhaseQuant with axis scales and recursive residual stages
// ("Fairy2i write-up" §3.1, §3.2, §4.1).
//
// Work unit: a tile of 1024 quads (4 consecutive weights = one code byte) of
// one tensor.  Each thread of a 256-thread block takes four quads of the tile,
// strided by 32 within its warp, and per stage t:
//   1. rebuilds the residual r_t = w - sum_{u<t} w_hat_u in float64 from w and
//      the already written codes and float32 scales of the earlier stages (w is
//      read again each stage: the per-tensor scale of stage t-1 is a global
//      dependency, and the fp32 weights of a layer do not fit on chip);
//   2. finds the sector k of r_t by exact comparisons (no atan2);
//   3. packs four codes into one byte;
//   4. sums S_re = sum |Re r| over k even, S_im = sum |Im r| over k odd and the
//      class-0 count (float64 / integer); the block reduces them in a fixed
//      order into the tile's partial in the workspace.
// A stage is two launches: quant_stage_kernel (one block per tile) and
// quant_reduce_kernel (one block per tensor: the partials in tile order ->
// s_re = S_re/C_re, s_im = S_im/C_im, 0 for an empty class, rounded to
// float32).  Consecutive launches are chained with programmatic dependent
// launch: a stage kernel loads its weights while the previous reduction runs
// and waits for it only before it needs the earlier scales and codes.  No
// block waits on another block of its own grid.
#include "ifq_common.cuh"
#include "ifq_internal.h"

#include <mutex>

namespace ifq {
namespace {

constexpr int kQThreads = 256;
constexpr int kQuadsPerThread = 4;
constexpr int kQuadsPerBlock = kQThreads * kQuadsPerThread;  // one tile

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
  QPartial* partials;    // [nblocks]: one per tile
  int64_t nquads;        // N*K/4
  int64_t block_begin;   // first global tile of this tensor
  int64_t nblocks;       // tiles
};

struct QParams {
  QTensorArg t[IFQ_MAX_GROUP];
  int64_t tiles;  // tiles of all tensors (tensor-major)
  int count;
  int stage;      // 0-based stage being computed
  uint32_t* status;
};

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Sector of w = a + ib as (cls, sgn) with k = 2 sgn + cls: 0 -> 1, 1 -> i,
// 2 -> -1, 3 -> -i.  Written without branches for finite a, b in any IEEE
// precision:
//   |b| > |a|                       -> cls 1, sign of b
//   |a| > |b|                       -> cls 0, sign of a
//   |a| = |b| > 0 (a diagonal tie)  -> the sector counter-clockwise of it:
//                                      cls 1 iff a, b have the same sign
//   a = b = 0                       -> k = 0
// (the four tie cases: 45 deg -> 1, 135 deg -> 2, -135 deg -> 3, -45 deg -> 0).
template <typename F>
__device__ __forceinline__ uint32_t sector_code(F a, F b) {
  const F aa = fabs(a), ab = fabs(b);
  const bool tie_same = (aa == ab) && (aa > F(0)) && ((a > F(0)) == (b > F(0)));
  const uint32_t cls = (ab > aa) || tie_same;
  const uint32_t sgn = cls ? (b < F(0)) : (a < F(0));
  return 2u * sgn + cls;
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

// One quad (4 weights -> one code byte) of stage PREV (0-based), given the
// earlier stages' code bytes of the quad.  Residual entries are rebuilt in
// float64 one earlier stage at a time: Re r -= s_re Br, Im r -= s_im Bi, i.e.
// add -s or +s when the code is on that axis.  The quad's four class values are
// summed in float32 (at most 3 roundings of a sum of non-negative terms: below
// 2e-7 relative) and that sum is added to the thread's float64 class sums.
// Returns the code byte.
// kChecked: some entry of this thread is NaN or infinite (rare): entries that are
// not finite are taken as 0.  Otherwise no per-entry test is made.
template <int PREV, bool kChecked>
__device__ __forceinline__ uint32_t quad_code(const float (&wr)[4], const float (&wi)[4], const uint32_t (&prev)[8],
                                              const double (&sr)[8], const double (&si)[8], double& S_re,
                                              double& S_im) {
  uint32_t byte = 0;
  float q_re = 0.0f, q_im = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const bool fin = !kChecked || (isfinite(wr[e]) && isfinite(wi[e]));
    uint32_t k;
    float v;
    if (PREV == 0) {
      const float a = fin ? wr[e] : 0.0f, b = fin ? wi[e] : 0.0f;
      k = sector_code(a, b);
      v = (k & 1u) ? fabsf(b) : fabsf(a);
    } else {
      double a = fin ? (double)wr[e] : 0.0, b = fin ? (double)wi[e] : 0.0;
#pragma unroll
      for (int u = 0; u < PREV; ++u) {
        const uint32_t ku = (prev[u] >> (2 * e)) & 3u;
        const double step_r = (ku & 2u) ? sr[u] : -sr[u];  // -s_re * Br for Br = +-1
        const double step_i = (ku & 2u) ? si[u] : -si[u];
        a = (ku & 1u) ? a : a + step_r;
        b = (ku & 1u) ? b + step_i : b;
      }
      k = sector_code(a, b);
      v = (float)((k & 1u) ? fabs(b) : fabs(a));
    }
    q_im += (k & 1u) ? v : 0.0f;
    q_re += (k & 1u) ? 0.0f : v;
    byte |= k << (2 * e);
  }
  S_re += (double)q_re;
  S_im += (double)q_im;
  return byte;
}

// ---------------------------------------------------------------- stage kernel
// One block per tile; the block's partial goes to the tile's workspace slot.
template <int PREV>
__global__ void __launch_bounds__(kQThreads) quant_stage_kernel(const __grid_constant__ QParams p) {
  pdl_trigger();  // the reduction of this stage may launch and wait for this grid
  // Find this block's tensor (at most IFQ_MAX_GROUP entries, uniform per block).
  int ti = 0;
  while (ti + 1 < p.count && (int64_t)blockIdx.x >= p.t[ti + 1].block_begin) ++ti;
  const QTensorArg& T = p.t[ti];
  const int64_t blk = (int64_t)blockIdx.x - T.block_begin;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t quad0 = blk * kQuadsPerBlock + (int64_t)warp * (32 * kQuadsPerThread) + lane;

  // The weights are inputs of the call, never written by its earlier launches: their
  // loads (8 x 128 bits per thread) go out before waiting for the previous launch.
  float wr[kQuadsPerThread][4], wi[kQuadsPerThread][4];
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
    const bool ok = quad < T.nquads;
    const float4 vr = ok ? __ldcs(reinterpret_cast<const float4*>(T.w_re) + quad) : make_float4(0, 0, 0, 0);
    const float4 vi = ok ? __ldcs(reinterpret_cast<const float4*>(T.w_im) + quad) : make_float4(0, 0, 0, 0);
    wr[q][0] = vr.x; wr[q][1] = vr.y; wr[q][2] = vr.z; wr[q][3] = vr.w;
    wi[q][0] = vi.x; wi[q][1] = vi.y; wi[q][2] = vi.z; wi[q][3] = vi.w;
  }
  pdl_wait();  // the earlier stages' codes and scales are complete from here on
  // They are read through L2 (ld.global.cg), not the read-only or L1 path: this grid starts
  // while the previous stage still runs on the same SMs, and a line of the scales or codes
  // cached there before the previous launches wrote it would be stale.
  double sr[8], si[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    sr[u] = u < PREV ? (double)__ldcg(T.scales + 2 * u) : 0.0;
    si[u] = u < PREV ? (double)__ldcg(T.scales + 2 * u + 1) : 0.0;
  }
  uint32_t prev[kQuadsPerThread][8];
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      prev[q][u] = (u < PREV && quad < T.nquads) ? __ldcg(T.codes + (int64_t)u * T.nquads + quad) : 0u;
  }

  // Non-finite weights are rare: one check for all 16 entries, exact handling only then.
  float z = 0.0f;
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e) z += wr[q][e] * 0.0f + wi[q][e] * 0.0f;
  const bool bad = z != 0.0f;  // NaN iff some entry is NaN or infinite

  double S_re = 0.0, S_im = 0.0;
  unsigned long long C_re = 0;
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
    if (quad >= T.nquads) break;
    const uint32_t byte = bad ? quad_code<PREV, true>(wr[q], wi[q], prev[q], sr, si, S_re, S_im)
                              : quad_code<PREV, false>(wr[q], wi[q], prev[q], sr, si, S_re, S_im);
    C_re += 4u - (uint32_t)__popc(byte & 0x55u);
    T.codes[(int64_t)PREV * T.nquads + quad] = (uint8_t)byte;
  }

  if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(p.status, IFQ_DEV_NONFINITE);

  block_sum3(S_re, S_im, C_re);
  if (threadIdx.x == 0) {
    QPartial part;
    part.s_re = S_re;
    part.s_im = S_im;
    part.c_re = C_re;
    part.pad = 0;
    T.partials[blk] = part;
  }
}

// ---------------------------------------------------------------- scale reduction
// One block per tensor: thread i adds the partials of tiles i, i + 256, ... in
// order, then the block adds the threads' sums in a fixed tree.
__global__ void __launch_bounds__(kQThreads) quant_reduce_kernel(const __grid_constant__ QParams p) {
  pdl_trigger();  // the next stage may launch and start streaming its weights
  pdl_wait();     // every tile partial of this stage is written
  const QTensorArg& T = p.t[blockIdx.x];
  double a = 0.0, b = 0.0;
  unsigned long long c = 0;
  for (int64_t i = threadIdx.x; i < T.nblocks; i += kQThreads) {
    const QPartial* pp = T.partials + i;
    a += __ldcg(&pp->s_re);  // through L2: written by the grid this one overlapped
    b += __ldcg(&pp->s_im);
    c += __ldcg(&pp->c_re);
  }
  block_sum3(a, b, c);
  if (threadIdx.x == 0) {
    const unsigned long long total = (unsigned long long)T.nquads * 4ull;
    const unsigned long long c_im = total - c;
    T.scales[2 * p.stage] = c > 0 ? (float)(a / (double)c) : 0.0f;
    T.scales[2 * p.stage + 1] = c_im > 0 ? (float)(b / (double)c_im) : 0.0f;
  }
}

// ---------------------------------------------------------------- conversion fused with stage 1
// ("Fairy2i write-up" §2.1 then §3.1, §3.2.)  One pass over R per layer: the
// block computes U and W for its quads exactly as widely_linear_vec4_kernel
// does, writes them (later stages read them), and runs stage 1 of both
// tensors exactly as quant_stage_kernel<0> does -- same quads per thread,
// same per-quad sums, same tile partials, then the same reduction kernel -- so
// codes, scales and planes equal those of the two-pass path bit for bit.  HBM
// traffic per complex position: 16 B of R read, 16 B of U, W and 0.5 B of
// codes written (the two-pass path also reads U, W back: 48.5 B).
struct FLayer {
  const float* R;      // [2n][2m]
  int64_t n, m;        // U, W are [n][m]
  int64_t fblock_begin;
  QTensorArg u, w;     // w_re / w_im of these are the planes this kernel writes
};

struct FParams {
  FLayer L[IFQ_MAX_GROUP / 2];
  int count;
  uint32_t* status;
};

__device__ __forceinline__ float half_sum(float a, float b) { return __fmul_rn(0.5f, __fadd_rn(a, b)); }
__device__ __forceinline__ float half_diff(float a, float b) { return __fmul_rn(0.5f, __fsub_rn(a, b)); }

__global__ void __launch_bounds__(kQThreads) widely_linear_quant1_kernel(const __grid_constant__ FParams p) {
  int li = 0;
  while (li + 1 < p.count && (int64_t)blockIdx.x >= p.L[li + 1].fblock_begin) ++li;
  const FLayer& L = p.L[li];
  const int64_t blk = (int64_t)blockIdx.x - L.fblock_begin;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t quad0 = blk * kQuadsPerBlock + (int64_t)warp * (32 * kQuadsPerThread) + lane;
  const int64_t m4 = L.m >> 2, half_row = L.m >> 1;  // float4s per output row; per R row = 2 m4
  const int64_t nq = L.u.nquads;
  const float4* R4 = reinterpret_cast<const float4*>(L.R);

  // All loads first (16 x 128-bit per thread), then quad by quad: U and W, their
  // stores, and stage-1 codes in the same quad order as quant_stage_kernel<0>.
  float4 r11[kQuadsPerThread], r12[kQuadsPerThread], r21[kQuadsPerThread], r22[kQuadsPerThread];
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
    r11[q] = r12[q] = r21[q] = r22[q] = make_float4(0, 0, 0, 0);
    if (quad < nq) {
      // output row i, float4 column j4 of U / W (32-bit division when the operands fit)
      const int64_t i = (quad | m4) < ((int64_t)1 << 32) ? (int64_t)((uint32_t)quad / (uint32_t)m4) : quad / m4;
      const int64_t j4 = quad - i * m4;
      const int64_t top = i * half_row + j4, bot = (i + L.n) * half_row + j4;
      r11[q] = __ldcs(R4 + top);
      r12[q] = __ldcs(R4 + top + m4);
      r21[q] = __ldcs(R4 + bot);
      r22[q] = __ldcs(R4 + bot + m4);
    }
  }

  const uint32_t none[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const double zero8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  double Su_re = 0.0, Su_im = 0.0, Sw_re = 0.0, Sw_im = 0.0;
  unsigned long long Cu = 0, Cw = 0;
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kQuadsPerThread; ++q) {
    const int64_t quad = quad0 + 32 * q;
    if (quad >= nq) break;
    const float a11[4] = {r11[q].x, r11[q].y, r11[q].z, r11[q].w}, a12[4] = {r12[q].x, r12[q].y, r12[q].z, r12[q].w};
    const float a21[4] = {r21[q].x, r21[q].y, r21[q].z, r21[q].w}, a22[4] = {r22[q].x, r22[q].y, r22[q].z, r22[q].w};
    float ur[4], ui[4], wr[4], wi[4];
    float z = 0.0f;  // NaN iff some entry of this quad's U or W is NaN or infinite
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ur[e] = half_sum(a11[e], a22[e]);
      ui[e] = half_diff(a21[e], a12[e]);
      wr[e] = half_diff(a11[e], a22[e]);
      wi[e] = half_sum(a12[e], a21[e]);
      z += (ur[e] * 0.0f + ui[e] * 0.0f) + (wr[e] * 0.0f + wi[e] * 0.0f);
    }
    reinterpret_cast<float4*>(const_cast<float*>(L.u.w_re))[quad] = make_float4(ur[0], ur[1], ur[2], ur[3]);
    reinterpret_cast<float4*>(const_cast<float*>(L.u.w_im))[quad] = make_float4(ui[0], ui[1], ui[2], ui[3]);
    reinterpret_cast<float4*>(const_cast<float*>(L.w.w_re))[quad] = make_float4(wr[0], wr[1], wr[2], wr[3]);
    reinterpret_cast<float4*>(const_cast<float*>(L.w.w_im))[quad] = make_float4(wi[0], wi[1], wi[2], wi[3]);
    // The checked form differs from the plain one only on non-finite entries.
    const bool bq = z != 0.0f;
    bad |= bq;
    const uint32_t bu = bq ? quad_code<0, true>(ur, ui, none, zero8, zero8, Su_re, Su_im)
                           : quad_code<0, false>(ur, ui, none, zero8, zero8, Su_re, Su_im);
    const uint32_t bw = bq ? quad_code<0, true>(wr, wi, none, zero8, zero8, Sw_re, Sw_im)
                           : quad_code<0, false>(wr, wi, none, zero8, zero8, Sw_re, Sw_im);
    Cu += 4u - (uint32_t)__popc(bu & 0x55u);
    Cw += 4u - (uint32_t)__popc(bw & 0x55u);
    L.u.codes[quad] = (uint8_t)bu;
    L.w.codes[quad] = (uint8_t)bw;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(p.status, IFQ_DEV_NONFINITE);

  block_sum3(Su_re, Su_im, Cu);
  block_sum3(Sw_re, Sw_im, Cw);
  if (threadIdx.x == 0) {
    QPartial pu, pw;
    pu.s_re = Su_re;
    pu.s_im = Su_im;
    pu.c_re = Cu;
    pu.pad = 0;
    pw.s_re = Sw_re;
    pw.s_im = Sw_im;
    pw.c_re = Cw;
    pw.pad = 0;
    L.u.partials[blk] = pu;
    L.w.partials[blk] = pw;
  }
}

// Fills p for `count` tensors over the workspace (the tile partials) and
// returns the number of tiles of one stage.
int64_t fill_qparams(const ifq_qtensor* t, int count, void* ws, QParams& p) {
  memset(&p, 0, sizeof(p));
  p.count = count;
  char* part = static_cast<char*>(ws);
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    QTensorArg& a = p.t[i];
    a.w_re = t[i].w_re;
    a.w_im = t[i].w_im;
    a.codes = t[i].codes;
    a.scales = t[i].scales;
    a.nquads = t[i].N * t[i].K / 4;
    a.nblocks = quant_blocks_for(t[i].N, t[i].K);
    a.block_begin = tiles;
    a.partials = reinterpret_cast<QPartial*>(part);
    part += (size_t)a.nblocks * sizeof(QPartial);
    tiles += a.nblocks;
  }
  p.tiles = tiles;
  return tiles;
}

// Launch with programmatic stream serialization (the kernel's pdl_wait orders
// it after the previous launch) or, for the first launch of a call, plainly.
template <class Kern>
cudaError_t launch(Kern kern, unsigned grid, int smem, bool chained, const QParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int PREV>
cudaError_t launch_stage(const QParams& p, bool chained, cudaStream_t s) {
  return launch(quant_stage_kernel<PREV>, (unsigned)p.tiles, 0, chained, p, s);
}

// Stages st_begin .. T-1 over every tensor of p: a stage kernel and its reduction each.
// chained: the first stage kernel follows a launch of this call (not the caller's work).
cudaError_t launch_stages(QParams& p, int st_begin, int T, bool chained, cudaStream_t s) {
  for (int st = st_begin; st < T; ++st) {
    p.stage = st;
    const bool ch = chained || st > st_begin;
    cudaError_t e;
    switch (st) {
      case 0: e = launch_stage<0>(p, ch, s); break;
      case 1: e = launch_stage<1>(p, ch, s); break;
      case 2: e = launch_stage<2>(p, ch, s); break;
      case 3: e = launch_stage<3>(p, ch, s); break;
      case 4: e = launch_stage<4>(p, ch, s); break;
      case 5: e = launch_stage<5>(p, ch, s); break;
      case 6: e = launch_stage<6>(p, ch, s); break;
      default: e = launch_stage<7>(p, ch, s); break;
    }
    if (e != cudaSuccess) return e;
    e = launch(quant_reduce_kernel, (unsigned)p.count, 0, true, p, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The 2 count tensors (U_0, W_0, U_1, W_1, ...) of a fused call.
void fused_tensors(const ifq_wl_layer* Ls, int count, ifq_qtensor* t) {
  for (int i = 0; i < count; ++i) {
    const int64_t n = Ls[i].rows / 2, m = Ls[i].cols / 2;
    t[2 * i] = ifq_qtensor{Ls[i].U_re, Ls[i].U_im, n, m, Ls[i].codes_u, Ls[i].scales_u};
    t[2 * i + 1] = ifq_qtensor{Ls[i].W_re, Ls[i].W_im, n, m, Ls[i].codes_w, Ls[i].scales_w};
  }
}

}  // namespace

int64_t quant_blocks_for(int64_t N, int64_t K) {
  const int64_t nquads = N * K / 4;
  return (nquads + kQuadsPerBlock - 1) / kQuadsPerBlock;
}

// Workspace: the tile partials of tensor 0, then of tensor 1, ...
size_t quant_workspace_bytes(const ifq_qtensor* t, int count) {
  size_t bytes = 0;
  for (int i = 0; i < count; ++i) bytes += (size_t)quant_blocks_for(t[i].N, t[i].K) * sizeof(QPartial);
  return bytes;
}

cudaError_t launch_quantize(const ifq_qtensor* t, int count, int T, void* ws, uint32_t* dev_status, cudaStream_t s) {
  QParams p;
  const int64_t tiles = fill_qparams(t, count, ws, p);
  p.status = dev_status;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  return launch_stages(p, 0, T, false, s);
}

// One stage of the quantizer on row shards of the tensors (a tensor's rows split across GPUs): the
// stage kernel writes the shard's codes of `stage` and one partial per tile of the shard into
// `partials`, without the reduction.
cudaError_t launch_quantize_stage(const ifq_qtensor* t, int count, int stage, void* partials, uint32_t* dev_status,
                                  cudaStream_t s) {
  QParams p;
  const int64_t tiles = fill_qparams(t, count, partials, p);
  p.status = dev_status;
  p.stage = stage;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  switch (stage) {
    case 0: return launch_stage<0>(p, false, s);
    case 1: return launch_stage<1>(p, false, s);
    case 2: return launch_stage<2>(p, false, s);
    case 3: return launch_stage<3>(p, false, s);
    case 4: return launch_stage<4>(p, false, s);
    case 5: return launch_stage<5>(p, false, s);
    case 6: return launch_stage<6>(p, false, s);
    default: return launch_stage<7>(p, false, s);
  }
}

// The stage's scales of whole tensors from the tile partials of all their shards, gathered in row order:
// the same reduction kernel, over the same tiles in the same order, as ifq_quantize_pack.
cudaError_t launch_quantize_finish(const ifq_qpartials* q, int count, int stage, cudaStream_t s) {
  QParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.stage = stage;
  for (int i = 0; i < count; ++i) {
    QTensorArg& a = p.t[i];
    a.partials = reinterpret_cast<QPartial*>(const_cast<void*>(q[i].partials));
    a.scales = q[i].scales;
    a.nquads = q[i].N * q[i].K / 4;
    a.nblocks = quant_blocks_for(q[i].N, q[i].K);
  }
  return launch(quant_reduce_kernel, (unsigned)count, 0, false, p, s);
}

size_t widely_linear_quant_workspace_bytes(const ifq_wl_layer* Ls, int count) {
  ifq_qtensor t[IFQ_MAX_GROUP];
  fused_tensors(Ls, count, t);
  return quant_workspace_bytes(t, 2 * count);
}

cudaError_t launch_widely_linear_quantize(const ifq_wl_layer* Ls, int count, int T, void* ws, uint32_t* dev_status,
                                          cudaStream_t s) {
  ifq_qtensor t[IFQ_MAX_GROUP];
  fused_tensors(Ls, count, t);
  QParams p;
  const int64_t tiles = fill_qparams(t, 2 * count, ws, p);
  p.status = dev_status;
  FParams f;
  memset(&f, 0, sizeof(f));
  f.count = count;
  f.status = dev_status;
  int64_t fblocks = 0;
  for (int i = 0; i < count; ++i) {
    FLayer& a = f.L[i];
    a.R = Ls[i].R;
    a.n = Ls[i].rows / 2;
    a.m = Ls[i].cols / 2;
    a.fblock_begin = fblocks;
    a.u = p.t[2 * i];
    a.w = p.t[2 * i + 1];
    fblocks += a.u.nblocks;
  }
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  widely_linear_quant1_kernel<<<(unsigned)fblocks, kQThreads, 0, s>>>(f);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  p.stage = 0;
  e = launch(quant_reduce_kernel, (unsigned)p.count, 0, true, p, s);
  if (e != cudaSuccess) return e;
  return launch_stages(p, 1, T, true, s);
}

// Scratch of ifq_quantize_pack_static, for callers that cannot hand over device
// memory (a C loader without a device allocator, a server whose caches hold
// the rest of the device).  Same layout as the caller workspace above.
static __device__ __align__(256) unsigned char g_quant_scratch[IFQ_QUANT_STATIC_SCRATCH_BYTES];

// The current driver context, through the runtime's driver entry point (no libcuda link); null if
// the entry point is unavailable.
static void* current_context() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  static GetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

cudaError_t launch_quantize_static(const ifq_qtensor* t, int count, int T, uint32_t* dev_status, cudaStream_t s) {
  constexpr int kCachedDevices = 64;
  static std::mutex mu;
  static void* addr[kCachedDevices] = {};
  static void* ctx_of[kCachedDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // The address is cached per device together with the context it was looked up in: after a
  // device reset, or when the caller runs in a context other than the one cached, the array lives
  // at a new address and is looked up again.
  void* ctx = current_context();
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    const bool cacheable = dev >= 0 && dev < kCachedDevices && ctx != nullptr;
    if (cacheable && ctx_of[dev] == ctx) scratch = addr[dev];
    if (!scratch) {
      // With the device current: the array's address in the current context.
      e = cudaGetSymbolAddress(&scratch, g_quant_scratch);
      if (e != cudaSuccess) return e;
      if (cacheable) {
        addr[dev] = scratch;
        ctx_of[dev] = ctx;
      }
    }
  }
  return launch_quantize(t, count, T, scratch, dev_status, s);
}

}  // namespace ifq
