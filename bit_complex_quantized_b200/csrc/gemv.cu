// Decode product y = sum_t (U_hat_t x + W_hat_t conj(x)) for up to 16 tokens (the C ABI
// sends B >= 3 here; one and two tokens take the integer path)
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2; "iFairy talk notes" §2.3.1).
//
// Work split: one CTA of 4 warps per (64-row block, K segment) of one layer
// (warp w: rows 16w..16w+15).  Layers longer than kKSeg positions are cut into
// segments of at most kKSeg, so that the CTAs carry similar work and one long
// layer does not set the kernel's length; a segmented layer's CTAs write partial
// sums to the workspace, which gemv_segment_sum_kernel adds in segment order.
// Blocks of longer layers are numbered first so they start first.
// The CTA walks K in chunks of 256 positions: the chunk of x for all B tokens
// (both planes, bf16) is staged once in shared memory, and every warp uses it
// for its 16 rows and every (stage, branch) code matrix.
//
// Per code, no multiplication by a weight happens: the 2-bit code is turned
// into a pair of exact bf16 operands for the two axis classes,
//     Br = sign * [class == 0] * 2,   Bi = sign * [class == 1] * 2,
// by one shift that drops the code's (class, sign) bits onto bf16 bits (14, 15)
// -- the bf16 pattern with only bit 14 set is 2.0 -- one AND that yields Bi,
// and one XOR with 2.0 that yields Br (a zero may come out as -0, which adds
// nothing).  A shifted 32-bit word carries codes j and j+8 of a 16-code word in
// its two halves, so the K order inside each 16-code group is permuted; the
// activation fragments are permuted identically with two byte-permutes.
// Tensor-core mma.sync m16n8k16 then forms the per-class signed sums
//     P_rr = sum Br x_re, P_ri = sum Br x_im, P_ir = sum Bi x_re, P_ii = sum Bi x_im
// with exact products (+-2 times bf16) and float32 accumulation.  Columns of
// the MMA are (token, plane) pairs: column 2b = x_re of token b, 2b+1 = x_im.
// After each chunk the scales of each (stage, branch) are applied:
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
// (times 1/2 for the operand encoding).  All sums run in a fixed order, so
// results are bit-reproducible.
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerBlock = 16 * kWarps;
constexpr int kChunkCodes = 256;  // codes per row per chunk: 4 threads x 16 bytes
// A staged (token, plane) row holds the chunk's 256 positions as 4 segments of 64 (one per
// lane group tq), each followed by 8 bf16 of padding: 288 bf16 = 576 bytes.  The four
// segments of a row, and the two planes, then fall on distinct banks.
constexpr int kSeg = 64 + 8;
constexpr int kXRow = 4 * kSeg;
constexpr int kKSeg = 2048;  // K positions per CTA at most (a multiple of the 256-position chunk)

struct GemvLayerArg {
  const uint8_t* codes[2];
  const float* scales[2];
  const uint16_t* x[2];  // re, im
  float* y[2];           // re, im
  const float* rot[2];   // optional epilogue rotation [B][N] (re, im), or null
  float* part;           // nseg > 1: partial sums [nseg][B][N][2], else null
  int64_t N;
  int64_t K;
  int64_t block_begin;
  int nbranch;
  int nseg;              // K segments (CTAs per 64-row block)
};

struct GemvParams {
  GemvLayerArg L[IFQ_MAX_GROUP];
  int order[IFQ_MAX_GROUP];  // layers by decreasing K: block numbering order
  int count;
  int T;
  int B;
  int pad;
  int64_t total_blocks;
  uint32_t* status;
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Output element idx = tok * N + n, times the optional rotation rot[idx] (complex RoPE).
__device__ __forceinline__ void store_y(const GemvLayerArg& L, int64_t idx, float yr, float yi) {
  if (L.rot[0]) {
    const float cr = __ldg(L.rot[0] + idx), ci = __ldg(L.rot[1] + idx);
    const float r = cr * yr - ci * yi, i = cr * yi + ci * yr;
    yr = r;
    yi = i;
  }
  L.y[0][idx] = yr;
  L.y[1][idx] = yi;
}

// NT: MMA n-tiles (8 columns = 4 tokens each); MI: code matrices per pass over a chunk.
template <int NT, int MI>
__global__ void __launch_bounds__(32 * kWarps) gemv_kernel(const __grid_constant__ GemvParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the segment sums may launch
  __shared__ __align__(16) uint16_t xs[4 * NT][2][kXRow];  // [token][plane][position in chunk]
  const int64_t blk = blockIdx.x;
  int oi = 0;
  while (oi + 1 < p.count && blk >= p.L[p.order[oi + 1]].block_begin) ++oi;
  const GemvLayerArg& L = p.L[p.order[oi]];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int64_t lb = blk - L.block_begin;                 // (row block, segment), segment fastest
  const int seg = (int)(lb % L.nseg);
  const int64_t row0 = (lb / L.nseg) * kRowsPerBlock + 16 * warp;
  const int64_t rowA = row0 + g, rowB = row0 + g + 8;
  const bool okA = rowA < L.N, okB = rowB < L.N;
  const int64_t K = L.K;
  const int64_t rb = K >> 2;  // bytes per code row
  const int nmat = p.T * L.nbranch;
  const int c_begin = seg * (kKSeg / kChunkCodes);  // this CTA's chunks of the row
  const int nchunks_row = (int)((K + kChunkCodes - 1) / kChunkCodes);
  const int nchunks = min(nchunks_row, c_begin + kKSeg / kChunkCodes);
  const int ntok = 4 * NT;

  float yr[NT][2], yi[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) yr[nt][0] = yr[nt][1] = yi[nt][0] = yi[nt][1] = 0.0f;

  for (int c = c_begin; c < nchunks; ++c) {
    const int64_t kc = (int64_t)c * kChunkCodes;
    const int klen = (int)(K - kc < kChunkCodes ? K - kc : kChunkCodes);  // multiple of 64
    // ---- stage x of the chunk: [token][plane][256] bf16; tokens past B and positions past K are 0
    __syncthreads();  // the previous chunk's fragments are no longer read
    for (int e = threadIdx.x; e < ntok * 2 * (kChunkCodes / 8); e += 32 * kWarps) {
      const int seg = e % (kChunkCodes / 8), pl = (e / (kChunkCodes / 8)) & 1, tok = e / (2 * (kChunkCodes / 8));
      uint4 v = make_uint4(0, 0, 0, 0);
      if (tok < p.B && seg * 8 < klen) v = __ldg(reinterpret_cast<const uint4*>(L.x[pl] + (int64_t)tok * K + kc) + seg);
      *reinterpret_cast<uint4*>(&xs[tok][pl][(seg >> 3) * kSeg + (seg & 7) * 8]) = v;
    }
    __syncthreads();

    // B-operand column of this thread in n-tile nt: token nt*4 + g/2, plane g&1.
    const int p0 = tq * 64;  // this thread's 64 positions of the chunk
    const bool kok = p0 < klen;
    for (int m0 = 0; m0 < nmat; m0 += MI) {
      float acc[MI][NT][2][4];
#pragma unroll
      for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int cl = 0; cl < 2; ++cl) acc[i][nt][cl][0] = acc[i][nt][cl][1] = acc[i][nt][cl][2] = acc[i][nt][cl][3] = 0.f;
      uint4 wa[MI], wb[MI];
#pragma unroll
      for (int i = 0; i < MI; ++i) {
        const int m = m0 + i < nmat ? m0 + i : nmat - 1;
        const int t = m / L.nbranch, br = m % L.nbranch;
        const uint8_t* base = L.codes[br] + (int64_t)t * L.N * rb + ((kc + p0) >> 2);
        wa[i] = (kok && okA && m0 + i < nmat) ? ld_nc_v4(base + rowA * rb) : make_uint4(0, 0, 0, 0);
        wb[i] = (kok && okB && m0 + i < nmat) ? ld_nc_v4(base + rowB * rb) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t X[NT][8];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint16_t* xp = &xs[nt * 4 + (g >> 1)][g & 1][tq * kSeg + 16 * w];
          const uint4 lo = *reinterpret_cast<const uint4*>(xp);
          const uint4 hi = *reinterpret_cast<const uint4*>(xp + 8);
          X[nt][0] = lo.x; X[nt][1] = lo.y; X[nt][2] = lo.z; X[nt][3] = lo.w;
          X[nt][4] = hi.x; X[nt][5] = hi.y; X[nt][6] = hi.z; X[nt][7] = hi.w;
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t b0[NT], b1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            b0[nt] = __byte_perm(X[nt][h], X[nt][h + 4], 0x5410);  // x[p+2h],   x[p+2h+8]
            b1[nt] = __byte_perm(X[nt][h], X[nt][h + 4], 0x7632);  // x[p+2h+1], x[p+2h+9]
          }
#pragma unroll
          for (int i = 0; i < MI; ++i) {
            const uint32_t va = (w == 0) ? wa[i].x : (w == 1) ? wa[i].y : (w == 2) ? wa[i].z : wa[i].w;
            const uint32_t vb = (w == 0) ? wb[i].x : (w == 1) ? wb[i].y : (w == 2) ? wb[i].z : wb[i].w;
            // codes (2h, 2h+8) -> k = 2tq, 2tq+1 ; codes (2h+1, 2h+9) -> k = 2tq+8, 2tq+9
            const uint32_t biA0 = (va << (14 - 4 * h)) & 0xC000C000u;
            const uint32_t biA2 = (va << (12 - 4 * h)) & 0xC000C000u;
            const uint32_t biB0 = (vb << (14 - 4 * h)) & 0xC000C000u;
            const uint32_t biB2 = (vb << (12 - 4 * h)) & 0xC000C000u;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_bf16_16816(acc[i][nt][0], biA0 ^ 0x40004000u, biB0 ^ 0x40004000u, biA2 ^ 0x40004000u,
                             biB2 ^ 0x40004000u, b0[nt], b1[nt]);
              mma_bf16_16816(acc[i][nt][1], biA0, biB0, biA2, biB2, b0[nt], b1[nt]);
            }
          }
        }
      }

      // Apply the scales of each matrix (halved: operands carry a factor 2).
#pragma unroll
      for (int i = 0; i < MI; ++i) {
        const int m = m0 + i;
        if (m >= nmat) break;
        const int t = m / L.nbranch, br = m % L.nbranch;
        const float hr = 0.5f * __ldg(L.scales[br] + 2 * t);
        const float hi = 0.5f * __ldg(L.scales[br] + 2 * t + 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float* Pr = acc[i][nt][0];  // {P_rr g, P_ri g, P_rr g+8, P_ri g+8}
          const float* Pi = acc[i][nt][1];  // {P_ir g, P_ii g, P_ir g+8, P_ii g+8}
          if (br == 0) {
            yr[nt][0] += hr * Pr[0] - hi * Pi[1];
            yi[nt][0] += hr * Pr[1] + hi * Pi[0];
            yr[nt][1] += hr * Pr[2] - hi * Pi[3];
            yi[nt][1] += hr * Pr[3] + hi * Pi[2];
          } else {
            yr[nt][0] += hr * Pr[0] + hi * Pi[1];
            yi[nt][0] += hi * Pi[0] - hr * Pr[1];
            yr[nt][1] += hr * Pr[2] + hi * Pi[3];
            yi[nt][1] += hi * Pi[2] - hr * Pr[3];
          }
        }
      }
    }
  }

  // Columns 2tq, 2tq+1 of n-tile nt are token nt*4 + tq, planes re / im: rows g, g+8.
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = nt * 4 + tq;
    if (tok < p.B) {
      if (L.nseg == 1) {
        if (okA) store_y(L, (int64_t)tok * L.N + rowA, yr[nt][0], yi[nt][0]);
        if (okB) store_y(L, (int64_t)tok * L.N + rowB, yr[nt][1], yi[nt][1]);
      } else {  // partial of this segment: [seg][tok][row][re, im]
        float* pp = L.part + (((int64_t)seg * p.B + tok) * L.N) * 2;
        if (okA) reinterpret_cast<float2*>(pp)[rowA] = make_float2(yr[nt][0], yi[nt][0]);
        if (okB) reinterpret_cast<float2*>(pp)[rowB] = make_float2(yr[nt][1], yi[nt][1]);
      }
    }
  }
}

// Segmented layers: y[tok][n] = sum over segments in order of the partials, times the
// optional rotation.  One thread per (layer, token, output); runs after the product
// kernel (programmatic dependent launch).
__global__ void __launch_bounds__(256) gemv_segment_sum_kernel(const __grid_constant__ GemvParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int64_t idx = (int64_t)blockIdx.x * 256 + threadIdx.x;
  for (int i = 0; i < p.count; ++i) {
    const GemvLayerArg& L = p.L[i];
    if (L.nseg == 1) continue;
    const int64_t n_out = (int64_t)p.B * L.N;
    if (idx < n_out) {
      float ar = 0.0f, ai = 0.0f;
      for (int sg = 0; sg < L.nseg; ++sg) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(L.part) + (int64_t)sg * n_out + idx);
        ar += v.x;
        ai += v.y;
      }
      store_y(L, idx, ar, ai);
      return;
    }
    idx -= n_out;
  }
}

template <int NT, int MI>
cudaError_t launch_nt_mi(const GemvParams& p, cudaStream_t s) {
  gemv_kernel<NT, MI><<<(unsigned)p.total_blocks, 32 * kWarps, 0, s>>>(p);
  return cudaGetLastError();
}

int segments_of(int64_t K) { return (int)((K + kKSeg - 1) / kKSeg); }

}  // namespace

// Partial sums of the segmented layers: [nseg][B][N][2] floats each, 256-byte aligned.
size_t gemv_bf16_workspace_bytes(const ifq_layer* Ls, int count, int B) {
  size_t off = 0;
  for (int i = 0; i < count; ++i) {
    const int nseg = segments_of(Ls[i].K);
    if (nseg > 1) off += ((size_t)nseg * B * Ls[i].N * 8 + 255) / 256 * 256;
  }
  return off;
}

cudaError_t launch_gemv(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status,
                        cudaStream_t s) {
  GemvParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.B = B;
  p.status = dev_status;
  for (int i = 0; i < count; ++i) {
    GemvLayerArg& a = p.L[i];
    a.codes[0] = Ls[i].codes_u;
    a.scales[0] = Ls[i].scales_u;
    a.codes[1] = Ls[i].codes_w;
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
    a.nseg = segments_of(a.K);
    p.order[i] = i;
  }
  int64_t sum_outputs = 0;
  {
    char* base = static_cast<char*>(ws);
    size_t off = 0;
    for (int i = 0; i < count; ++i) {
      GemvLayerArg& a = p.L[i];
      if (a.nseg == 1) continue;
      a.part = reinterpret_cast<float*>(base + off);
      off += ((size_t)a.nseg * B * a.N * 8 + 255) / 256 * 256;
      sum_outputs += (int64_t)B * a.N;
    }
  }
  // Longest rows first (stable): their blocks are launched first.
  for (int i = 1; i < count; ++i)
    for (int j = i; j > 0 && p.L[p.order[j]].K > p.L[p.order[j - 1]].K; --j) {
      const int t = p.order[j];
      p.order[j] = p.order[j - 1];
      p.order[j - 1] = t;
    }
  int64_t blocks = 0;
  for (int i = 0; i < count; ++i) {
    GemvLayerArg& a = p.L[p.order[i]];
    a.block_begin = blocks;
    blocks += (a.N + kRowsPerBlock - 1) / kRowsPerBlock * a.nseg;
  }
  p.total_blocks = blocks;
  if (blocks > 0x7fffffffLL || sum_outputs > ((int64_t)1 << 38)) return cudaErrorInvalidConfiguration;
  const int NT = (2 * B + 7) / 8;
  cudaError_t e;
  switch (NT) {
    case 1: e = launch_nt_mi<1, 4>(p, s); break;
    case 2: e = launch_nt_mi<2, 2>(p, s); break;
    case 3: e = launch_nt_mi<3, 2>(p, s); break;
    default: e = launch_nt_mi<4, 2>(p, s); break;
  }
  if (e != cudaSuccess || sum_outputs == 0) return e;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)((sum_outputs + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_segment_sum_kernel, p);
}

}  // namespace ifq
