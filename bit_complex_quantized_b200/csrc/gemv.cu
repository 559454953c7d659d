// Decode product y = sum_t (U_hat_t x + W_hat_t conj(x)) for B = 1..16 tokens
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2; "iFairy talk notes" §2.3.1).
//
// Work split: one CTA of 4 warps per 16-row tile of one layer; warp w takes the
// 256-code K-chunks c = w, w+4, ... of every (stage, branch) code matrix, and
// the four warps' partial outputs are summed in a fixed order through shared
// memory, so results are bit-reproducible.
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
// The epilogue applies the scales once per (stage, branch):
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
// (times 1/2 for the operand encoding).
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kWarpsPerTile = 4;
constexpr int kChunkCodes = 256;  // codes per row per chunk: 4 threads x 16 bytes

struct GemvLayerArg {
  const uint8_t* codes[2];
  const float* scales[2];
  const uint16_t* x[2];  // re, im
  float* y[2];           // re, im
  int64_t N;
  int64_t K;
  int64_t tile_begin;
  int nbranch;
  int pad;
};

struct GemvParams {
  GemvLayerArg L[IFQ_MAX_GROUP];
  int count;
  int T;
  int B;
  int pad;
  int64_t total_tiles;
  uint32_t* status;
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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

// NT: MMA n-tiles (8 columns = 4 tokens each); MI: code matrices handled per pass.
template <int NT, int MI>
__global__ void __launch_bounds__(32 * kWarpsPerTile) gemv_kernel(const __grid_constant__ GemvParams p) {
  const int64_t tile = blockIdx.x;
  int li = 0;
  while (li + 1 < p.count && tile >= p.L[li + 1].tile_begin) ++li;
  const GemvLayerArg& L = p.L[li];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int64_t row0 = (tile - L.tile_begin) * 16;
  const int64_t rowA = row0 + g, rowB = row0 + g + 8;
  const bool okA = rowA < L.N, okB = rowB < L.N;
  const int64_t K = L.K;
  const int64_t rb = K >> 2;  // bytes per code row
  const int nmat = p.T * L.nbranch;
  const int nchunks = (int)((K + kChunkCodes - 1) / kChunkCodes);

  // B-operand column owned by this thread in n-tile nt: token nt*4 + g/2, plane g&1.
  const uint16_t* xcol[NT];
  bool xok[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = nt * 4 + (g >> 1);
    xok[nt] = tok < p.B;
    xcol[nt] = L.x[g & 1] + (int64_t)(xok[nt] ? tok : 0) * K;
  }

  float yr[NT][2], yi[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) yr[nt][0] = yr[nt][1] = yi[nt][0] = yi[nt][1] = 0.0f;

  for (int m0 = 0; m0 < nmat; m0 += MI) {
    float acc[MI][NT][2][4];
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) acc[i][nt][c][0] = acc[i][nt][c][1] = acc[i][nt][c][2] = acc[i][nt][c][3] = 0.f;

    const uint8_t* mrowA[MI];
    const uint8_t* mrowB[MI];
#pragma unroll
    for (int i = 0; i < MI; ++i) {
      const int m = m0 + i;
      const int t = m / L.nbranch, br = m % L.nbranch;
      const uint8_t* base = L.codes[br] + (int64_t)t * L.N * rb;
      mrowA[i] = base + (okA ? rowA : 0) * rb;
      mrowB[i] = base + (okB ? rowB : 0) * rb;
    }

    for (int c = warp; c < nchunks; c += kWarpsPerTile) {
      const int64_t pos0 = (int64_t)c * kChunkCodes + tq * 64;  // this thread's 64 K positions
      const bool kok = pos0 < K;                                // K % 64 == 0: all-or-nothing
      uint4 wa[MI], wb[MI];
#pragma unroll
      for (int i = 0; i < MI; ++i) {
        wa[i] = (kok && okA) ? ld_nc_v4(mrowA[i] + (pos0 >> 2)) : make_uint4(0, 0, 0, 0);
        wb[i] = (kok && okB) ? ld_nc_v4(mrowB[i] + (pos0 >> 2)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t X[NT][8];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (kok && xok[nt]) {
            const uint4 lo = __ldg(reinterpret_cast<const uint4*>(xcol[nt] + pos0 + 16 * w));
            const uint4 hi = __ldg(reinterpret_cast<const uint4*>(xcol[nt] + pos0 + 16 * w + 8));
            X[nt][0] = lo.x; X[nt][1] = lo.y; X[nt][2] = lo.z; X[nt][3] = lo.w;
            X[nt][4] = hi.x; X[nt][5] = hi.y; X[nt][6] = hi.z; X[nt][7] = hi.w;
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) X[nt][q] = 0u;
          }
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
    }

    // Apply the scales of each matrix (halved: operands carry a factor 2).
#pragma unroll
    for (int i = 0; i < MI; ++i) {
      const int m = m0 + i;
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

  // Sum the warps' K-slices in a fixed order and store.
  __shared__ float red[kWarpsPerTile][NT * 4][32];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    red[warp][nt * 4 + 0][lane] = yr[nt][0];
    red[warp][nt * 4 + 1][lane] = yi[nt][0];
    red[warp][nt * 4 + 2][lane] = yr[nt][1];
    red[warp][nt * 4 + 3][lane] = yi[nt][1];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float s = red[0][nt * 4 + q][lane];
#pragma unroll
        for (int w = 1; w < kWarpsPerTile; ++w) s += red[w][nt * 4 + q][lane];
        v[q] = s;
      }
      const int tok = nt * 4 + tq;
      if (tok < p.B) {
        if (okA) {
          L.y[0][(int64_t)tok * L.N + rowA] = v[0];
          L.y[1][(int64_t)tok * L.N + rowA] = v[1];
        }
        if (okB) {
          L.y[0][(int64_t)tok * L.N + rowB] = v[2];
          L.y[1][(int64_t)tok * L.N + rowB] = v[3];
        }
      }
    }
  }
}

template <int NT, int MI>
cudaError_t launch_nt_mi(const GemvParams& p, cudaStream_t s) {
  gemv_kernel<NT, MI><<<(unsigned)p.total_tiles, 32 * kWarpsPerTile, 0, s>>>(p);
  return cudaGetLastError();
}

// Several matrices per pass only pay off with one n-tile (B <= 4); with more
// n-tiles the accumulators already fill the register file.
cudaError_t launch_nt1(const GemvParams& p, int mi, cudaStream_t s) {
  switch (mi) {
    case 4: return launch_nt_mi<1, 4>(p, s);
    case 3: return launch_nt_mi<1, 3>(p, s);
    case 2: return launch_nt_mi<1, 2>(p, s);
    default: return launch_nt_mi<1, 1>(p, s);
  }
}

}  // namespace

cudaError_t launch_gemv(const ifq_layer* Ls, int count, int T, int B, uint32_t* dev_status, cudaStream_t s) {
  GemvParams p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.B = B;
  p.status = dev_status;
  int64_t tiles = 0;
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
    a.N = Ls[i].N;
    a.K = Ls[i].K;
    a.tile_begin = tiles;
    tiles += (Ls[i].N + 15) / 16;
  }
  p.total_tiles = tiles;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int NT = (2 * B + 7) / 8;
  // Matrices per pass: the largest of 4, 3, 2 that divides every layer's
  // (stage, branch) matrix count, so that one activation-fragment load serves them all.
  int mi = 1;
  if (NT == 1) {
    for (int c : {4, 3, 2}) {
      bool ok = true;
      for (int i = 0; i < count; ++i) ok &= (T * p.L[i].nbranch) % c == 0;
      if (ok) {
        mi = c;
        break;
      }
    }
  }
  switch (NT) {
    case 1: return launch_nt1(p, mi, s);
    case 2: return launch_nt_mi<2, 1>(p, s);
    case 3: return launch_nt_mi<3, 1>(p, s);
    default: return launch_nt_mi<4, 1>(p, s);
  }
}

}  // namespace ifq
