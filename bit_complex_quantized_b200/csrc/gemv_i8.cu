// Decode product for one or two tokens (B = 1, 2) on the integer tensor cores, exactly
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2; "iFairy talk notes" §2.3.1).
// The description below is the one-token case; two tokens share each operand's extraction
// (half_chunk_mma) and keep one int32 sum per (plane, token).
//
// Re-coding the 2-bit code.  With k = 2 s + c (c: axis bit, s: sign bit), the
// real and imaginary parts of the codeword [1, i, -1, -i][k] are
//     Br = (1-c)(1-2s),   Bi = c(1-2s),
// which mix c and s.  In the Gray code g1 = s, g0 = c XOR s they become affine:
//     Br = 1 - g0 - g1,   Bi = g0 - g1,
// so two 0/1 bit-planes per code suffice:
//     sum_j Br_j x_j = sum_j x_j - G0 - G1,   sum_j Bi_j x_j = G0 - G1,   G_b = sum_j g_b,j x_j.
// In registers both planes are read at bit 2q+1 of each byte (q: position of
// the code in its byte): g1 = s is that bit of the code word w, g0 = c XOR s is
// that bit of w ^ (w << 1).  One logic op per (plane, q) -- (w ^ 2w) & m or
// w & m -- selects 4 codes, one per byte, as int8 operands 2*4^q g (-128 g at
// q = 3).  Each (plane, q) has its own int32 accumulator, so no shift is
// needed; the weights are undone exactly when the accumulators are combined.
//
// Activations.  ifq_gemv first runs gemv_prep_kernel: per block of up to 2048
// K positions, x (bf16, both planes) is scaled by 2^E with the block maximum in
// [2^29, 2^30) and rounded to an integer v, whose four balanced base-256 digits
// are the bytes of (v + 0x80808080) ^ 0x80808080.  The rounding error is at
// most 2^-E per position, so sum_j(|e_re,j| + |e_im,j|) <= 2048 * 2^-E, below
// 4e-6 of the block's largest |x| -- inside the 1e-5 tolerance for any x.
// The digits are stored in MMA-fragment order with the exact block sums of v.
//
// Main kernel (programmatic dependent launch after the prep kernel): the codes
// are cut into 1 KB chunks (16 rows x 256 K positions of one (stage, branch)
// matrix), ordered tile by tile, and every warp of a persistent grid takes an
// equal contiguous range of chunks (stream-K), so the load is balanced to one
// chunk.  A warp walks its range in pieces (one tile, one matrix, one K block
// at most), streams each piece into a double-buffered shared slot (completion
// on an mbarrier), and runs mma.sync m16n8k32 s8 (columns = plane x digit, exact int32
// accumulation).  Per tile it keeps the float64 output sums in registers; a
// tile split between warps leaves one partial per warp in the workspace, and
// the last of them to arrive (atomic ticket) adds the partials in warp order
// and writes y -- results do not depend on timing.
#include "ifq_common.cuh"
#include "ifq_internal.h"

#include <mutex>

namespace ifq {
namespace {

constexpr int kKBlock = 2048;                  // K positions per exponent block
constexpr int kWarps = 4;                      // warps per CTA in the main kernel
constexpr int kPieceChunks = 8;                // at most 8 chunks (256 K positions each) per piece: one K block
constexpr int kSlotBytes = 8192;               // one slot: 16 rows x 8 chunks x 64 bytes
constexpr int kMainSmem = kWarps * 2 * kSlotBytes + kWarps * 2 * 8;
constexpr int kPrepThreads = 128;                // one item (plane, position, 16-group) per thread of a chunk
// Resident CTAs per SM: three, or two for four tokens (their sums and fragments need more registers).
constexpr int ctas_per_sm(int nb) { return nb >= 4 ? 2 : 3; }
static_assert(kPieceChunks * 256 == kKBlock, "a piece is at most one K block, and one run of the int32 sums");

// Slot layouts.  Pieces inside a full K block arrive by one 4-D tensor copy as
// [chunk][row][64 B] (lanes of a quarter warp read two adjacent 64-byte rows:
// conflict-free).  Pieces of a row's last, partial block arrive by one bulk copy
// per row as [row][512 B].
// The scalars first and the tensor maps (read by the copy engine only) last, so the
// fields a warp reads sit in few constant-cache lines.
struct I8Layer {
  const uint8_t* codes[2];
  const float* scales[2];
  const uint16_t* x[2];
  float* y[2];
  const float* rot[2];    // optional epilogue rotation [N] (re, im), or null
  uint4* frag;            // [blocks][8 chunks][NB][32 lanes][4]: a lane's 8 k-step fragments of a chunk, contiguous
  double* bsum;           // [blocks][NB][9][2]: exact sums of v over the block's first c chunks, per plane
  int* bexp;              // [blocks][NB]
  float* partials;        // [tiles][chunks per tile][NB][16][2] (one slot per warp touching the tile)
  int* next;              // [tiles][chunks per tile]: end of the portion that starts at this chunk
  unsigned int* tickets;  // [tiles]: finished chunks of the tile
  int64_t N, K;
  int64_t chunk_begin;    // first global chunk
  int64_t prep_begin;     // first prep CTA
  int32_t tiles;          // 16-row tiles
  int32_t blocks;         // K blocks
  int32_t nbranch;
  int32_t nch;            // 256-wide K chunks per row
  int32_t nbf;            // full 2048-wide K blocks (streamed by tensor copies)
  CUtensorMap tmap[2];    // per branch: (64 B, row of [T][N], chunk in block, full block), box 64 x 16 x 8 x 1
};

// Capacity kCap >= count: calls of up to 8 layers pass a small parameter block.
// The call-wide scalars and the layer-begin tables lead, in the first constant-cache lines.
template <int kCap>
struct I8Params {
  int64_t total_chunks;
  int count;
  int T;
  int B;    // tokens; the kernels are built for NB >= B and treat tokens B..NB-1 as zero
  int sms;  // > 0: CTA b works as CTA (b % sms) * (gridDim / sms) + b / sms
  uint32_t* status;
  int64_t chunk_begin[kCap];  // copies of the layers' first chunk and first prep CTA, packed so that
  int64_t prep_begin[kCap];   // the search for a layer touches one or two constant-cache lines
  I8Layer L[kCap];
};

__device__ __forceinline__ void imma_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                           uint32_t b1) {
  // Not volatile: a pure function of its registers, so the compiler may interleave it with loads.
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

template <class P>
__device__ __forceinline__ int find_layer_by(const P& p, int64_t idx, bool prep) {
  int li = 0;
  while (li + 1 < p.count && idx >= (prep ? p.prep_begin[li + 1] : p.chunk_begin[li + 1])) ++li;
  return li;
}

// ---------------------------------------------------------------- prep kernel
// One CTA per (layer, K block, 256-wide chunk): every CTA of a block finds the
// block's exponent, then writes the digit fragments of its own chunk and the
// exact sum of v up to its chunk's end (prefix sums at chunk boundaries).  The
// first CTA of a layer also zeroes the layer's tile tickets.
template <class P, int NB>
__global__ void __launch_bounds__(kPrepThreads) gemv_prep_kernel(const __grid_constant__ P p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ __align__(16) uint16_t xs[2][kKBlock];
  __shared__ unsigned int smax[kPrepThreads / 32];
  __shared__ long long ssum[2][kPrepThreads / 32];

  const int li = find_layer_by(p, blockIdx.x, true);
  const I8Layer& L = p.L[li];
  const int bc = (int)(blockIdx.x - L.prep_begin);
  const int b = bc >> 3, c = bc & 7;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (bc == 0)
    for (int t = tid; t < L.tiles; t += kPrepThreads) L.tickets[t] = 0u;

  const int64_t k0 = (int64_t)b * kKBlock;
  const int klen = (int)(L.K - k0 < kKBlock ? L.K - k0 : kKBlock);  // multiple of 64
  if (c * 256 >= klen) return;  // the block's last chunk lies before this one

  for (int tok = 0; tok < NB; ++tok) {
    if (tok > 0) __syncthreads();  // the previous token's use of xs, smax and ssum is over
    const bool live = tok < p.B;   // tokens past the batch are zero
    unsigned int mx = 0;
#pragma unroll
    for (int r = 0; r < kKBlock / (8 * kPrepThreads); ++r) {
#pragma unroll
      for (int pl = 0; pl < 2; ++pl) {
        const int idx = (r * kPrepThreads + tid) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (idx < klen && live) v = __ldg(reinterpret_cast<const uint4*>(L.x[pl] + (int64_t)tok * L.K + k0 + idx));
        *reinterpret_cast<uint4*>(&xs[pl][idx]) = v;
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mx = max(mx, wv[q] & 0x7FFFu);
          mx = max(mx, (wv[q] >> 16) & 0x7FFFu);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) smax[warp] = mx;
    __syncthreads();
    mx = 0;
#pragma unroll
    for (int w = 0; w < kPrepThreads / 32; ++w) mx = max(mx, smax[w]);
    const bool nonfinite = mx >= 0x7F80u;
    int E = 0;  // max |x| * 2^E in [2^29, 2^30)
    if (mx != 0 && !nonfinite) {
      const uint32_t f = mx << 16;
      const int e = (f >> 23) ? (int)(f >> 23) - 127 : (31 - __clz(f)) - 149;
      E = 29 - e;
    }
    if (nonfinite && tid == 0 && c == 0) set_status(p.status, IFQ_DEV_NONFINITE);
    const int E1 = min(E, 127);
    const float f1 = __int_as_float((E1 + 127) << 23);
    const float f2 = __int_as_float((E - E1 + 127) << 23);

    // Exact sum of v over positions [0, 256 (c + 1)) of the block, per plane (prefix sums
    // at chunk boundaries): thread t adds positions t, t + 128, ... below the bound.
    long long vsum = 0;
    {
      const int pl = tid & 1;
      const int bound = (c + 1) * 256 < klen ? (c + 1) * 256 : klen;
#pragma unroll
      for (int r = 0; r < kKBlock / (kPrepThreads / 2); ++r) {  // independent terms: unrolled for latency
        const int j = (tid >> 1) + r * (kPrepThreads / 2);
        if (j < bound && !nonfinite) {
          const float xf = __uint_as_float((uint32_t)xs[pl][j] << 16);
          vsum += __float2int_rn((xf * f1) * f2);
        }
      }
    }
    // Item (plane pl, in-byte position q, 16-position group grp = (chunk c, slice tq, word w))
    // covers positions grp*16 + 4i + q, i = 0..3: bytes i of the code word w at position q.
    // One item per thread: the chunk's 128 items.
    {
      const int it = tid;
      const int pl = it & 1, q = (it >> 1) & 3, grp = c * 16 + (it >> 3);
      uint32_t D[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = grp * 16 + 4 * i + q;
        int v = 0;
        if (j < klen && !nonfinite) {
          const float xf = __uint_as_float((uint32_t)xs[pl][j] << 16);
          v = __float2int_rn((xf * f1) * f2);
        }
        D[i] = ((uint32_t)v + 0x80808080u) ^ 0x80808080u;
      }
      const uint32_t lo01 = __byte_perm(D[0], D[1], 0x5140), lo23 = __byte_perm(D[2], D[3], 0x5140);
      const uint32_t hi01 = __byte_perm(D[0], D[1], 0x7362), hi23 = __byte_perm(D[2], D[3], 0x7362);
      const uint32_t dig[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                               __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
      const int tqs = (grp >> 2) & 3, w = grp & 3;
      const int ks = (w >> 1) * 4 + q;  // k-step within the chunk: (word pair, position)
      // a lane's fragments for chunk c: 8 k-steps x (b0, b1) = 64 contiguous bytes
      uint32_t* fr =
          reinterpret_cast<uint32_t*>(L.frag + (((int64_t)b * 8 + c) * NB + tok) * 32 * 4) + ks * 2 + (w & 1);
#pragma unroll
      for (int d = 0; d < 4; ++d) fr[((pl * 4 + d) * 4 + tqs) * 16] = dig[d];
    }
#pragma unroll
    for (int o = 16; o > 1; o >>= 1) vsum += __shfl_xor_sync(0xffffffffu, vsum, o);  // even / odd lanes
    if (lane < 2) ssum[lane][warp] = vsum;
    __syncthreads();
    if (tid < 2) {
      long long s = 0;
#pragma unroll
      for (int w = 0; w < kPrepThreads / 32; ++w) s += ssum[tid][w];
      // prefix[c + 1]; the block's first CTA also writes prefix[0] = 0
      double* pre = L.bsum + ((int64_t)b * NB + tok) * 18;
      pre[(c + 1) * 2 + tid] = nonfinite ? __longlong_as_double(0x7FF8000000000000LL) : (double)s;
      if (c == 0) pre[tid] = 0.0;
      if (tid == 0 && c == 0) L.bexp[(int64_t)b * NB + tok] = E;
    }
  }  // tokens
}

// ---------------------------------------------------------------- main kernel
// Output n of the token, times the optional rotation rot[n] (complex RoPE).
__device__ __forceinline__ void store_y(const I8Layer& L, int64_t n, float yr, float yi) {
  if (L.rot[0]) {
    const float cr = __ldg(L.rot[0] + n), ci = __ldg(L.rot[1] + n);
    const float r = cr * yr - ci * yi, i = cr * yi + ci * yr;
    yr = r;
    yi = i;
  }
  L.y[0][n] = yr;
  L.y[1][n] = yi;
}

// A piece: chunks [ch, ch + len) of one (tile, matrix) row block, inside one K block.
struct Piece {
  int li;
  int mat;
  int ch;
  int len;
  int64_t tile;
  int64_t gbegin;  // global index of its first chunk
};

__device__ __forceinline__ int piece_len(const I8Layer& L, int ch, int64_t gbegin, int64_t c_hi) {
  const int block_end = min(L.nch, (ch / 8 + 1) * 8);
  int64_t len = min(block_end - ch, kPieceChunks);
  if (gbegin + len > c_hi) len = c_hi - gbegin;
  return (int)len;
}

// The piece that starts at global chunk c (one division chain per warp, at its start).
template <class P>
__device__ __forceinline__ Piece make_piece(const P& p, int64_t c, int64_t c_hi) {
  Piece pc;
  pc.li = find_layer_by(p, c, false);
  const I8Layer& L = p.L[pc.li];
  const int64_t tc = (int64_t)p.T * L.nbranch * L.nch;  // chunks per tile
  const int64_t local = c - p.chunk_begin[pc.li];
  // 32-bit division when the operands fit (the usual case): far shorter than the 64-bit routine
  pc.tile = (local | tc) < ((int64_t)1 << 32) ? (int64_t)((uint32_t)local / (uint32_t)tc) : local / tc;
  const int r = (int)(local - pc.tile * tc);
  pc.mat = r / L.nch;
  pc.ch = r - pc.mat * L.nch;
  pc.gbegin = c;
  pc.len = piece_len(L, pc.ch, c, c_hi);
  return pc;
}

// The piece after `pc` in chunk order (chunks, then matrices, then tiles, then layers).
template <class P>
__device__ __forceinline__ Piece next_piece(const P& p, const Piece& pc, int64_t c_hi) {
  Piece n = pc;
  n.gbegin = pc.gbegin + pc.len;
  n.ch = pc.ch + pc.len;
  const I8Layer* L = &p.L[n.li];
  if (n.ch >= L->nch) {
    n.ch = 0;
    if (++n.mat >= p.T * L->nbranch) {
      n.mat = 0;
      if (++n.tile >= L->tiles) {
        n.tile = 0;
        ++n.li;
        L = &p.L[n.li];
      }
    }
  }
  n.len = piece_len(*L, n.ch, n.gbegin, c_hi);
  return n;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* addr, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

// Warp w < W owns chunks [lo(w), lo(w+1)) with lo(w) = floor(w C / W); W <= C, so no range is empty.
__device__ __forceinline__ int64_t range_lo(int64_t w, int64_t C, int64_t W) {
  const int64_t num = w * C;  // 32-bit division when the operands fit (the usual case)
  return (num | W) < ((int64_t)1 << 32) ? (int64_t)((uint32_t)num / (uint32_t)W) : num / W;
}


// As imma_16832 with a zero accumulator input: starts a fresh sum without zeroing registers.
__device__ __forceinline__ void imma_16832_first(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ uint32_t xor_and(uint32_t a, uint32_t b, uint32_t c) {  // (a ^ b) & c in one op
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x28;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// One chunk (16 rows x 256 positions) against this lane's 8 k-step fragments:
// 16 MMAs, one per (in-byte position q, Gray plane), over the chunk's two word pairs.
// Both Gray planes are taken at bit 2q+1 of each byte: g1 = s is that bit of w,
// and g0 = c XOR s is that bit of w ^ (w << 1), so no separate Gray step is needed.
// kFirst: the piece's first chunk, whose first MMAs start the sums.
template <bool kFirst>
__device__ __forceinline__ void chunk_mma(int (&acc0)[4][4], int (&acc1)[4][4], const uint4* rowa, const uint4* rowb,
                                          const uint4 (&F)[4]) {
  const uint4 va = *rowa, vb = *rowb;
#pragma unroll
  for (int wp = 0; wp < 2; ++wp) {
    const uint32_t a0 = wp ? va.z : va.x, a1 = wp ? va.w : va.y;
    const uint32_t b0 = wp ? vb.z : vb.x, b1 = wp ? vb.w : vb.y;
    const uint32_t a0s = a0 * 2u, a1s = a1 * 2u, b0s = b0 * 2u, b1s = b1 * 2u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int ks = wp * 4 + q;
      const uint32_t fx = (ks & 1) ? F[ks >> 1].z : F[ks >> 1].x;
      const uint32_t fy = (ks & 1) ? F[ks >> 1].w : F[ks >> 1].y;
      const uint32_t m = 0x02020202u << (2 * q);
      if (kFirst && wp == 0) {
        imma_16832_first(acc0[q], xor_and(a0, a0s, m), xor_and(b0, b0s, m), xor_and(a1, a1s, m), xor_and(b1, b1s, m),
                         fx, fy);
        imma_16832_first(acc1[q], a0 & m, b0 & m, a1 & m, b1 & m, fx, fy);
      } else {
        imma_16832(acc0[q], xor_and(a0, a0s, m), xor_and(b0, b0s, m), xor_and(a1, a1s, m), xor_and(b1, b1s, m), fx,
                   fy);
        imma_16832(acc1[q], a0 & m, b0 & m, a1 & m, b1 & m, fx, fy);
      }
    }
  }
}

// Several tokens (NB >= 2): half a chunk -- one word pair per row, 4 positions x 2 planes
// -- against every token's fragments of those 4 k-steps.  Each operand is shifted down so
// that its bit sits at bit 1 of each byte (weight 2 for every position): one int32 sum
// per (plane, token) instead of one per (plane, position), at the price of a shift per
// operand, which the NB MMAs per operand pay for.  kFirst: the first MMA of each sum.
template <int NB, bool kFirst>
__device__ __forceinline__ void half_chunk_mma(int (&acc0)[NB][4], int (&acc1)[NB][4], uint32_t a0, uint32_t a1,
                                               uint32_t b0, uint32_t b1, const uint4 (&F)[NB][2]) {
  const uint32_t ua0 = a0 ^ (a0 << 1), ua1 = a1 ^ (a1 << 1), ub0 = b0 ^ (b0 << 1), ub1 = b1 ^ (b1 << 1);
  const uint32_t m = 0x02020202u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t g0a0 = (ua0 >> (2 * q)) & m, g0b0 = (ub0 >> (2 * q)) & m;
    const uint32_t g0a1 = (ua1 >> (2 * q)) & m, g0b1 = (ub1 >> (2 * q)) & m;
    const uint32_t g1a0 = (a0 >> (2 * q)) & m, g1b0 = (b0 >> (2 * q)) & m;
    const uint32_t g1a1 = (a1 >> (2 * q)) & m, g1b1 = (b1 >> (2 * q)) & m;
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const uint32_t fx = (q & 1) ? F[t][q >> 1].z : F[t][q >> 1].x;
      const uint32_t fy = (q & 1) ? F[t][q >> 1].w : F[t][q >> 1].y;
      if (kFirst && q == 0) {
        imma_16832_first(acc0[t], g0a0, g0b0, g0a1, g0b1, fx, fy);
        imma_16832_first(acc1[t], g1a0, g1b0, g1a1, g1b1, fx, fy);
      } else {
        imma_16832(acc0[t], g0a0, g0b0, g0a1, g0b1, fx, fy);
        imma_16832(acc1[t], g1a0, g1b0, g1a1, g1b1, fx, fy);
      }
    }
  }
}

// A lane's fragments of half h (word pair) of a chunk for every token; fr0 points at token 0's.
template <int NB>
__device__ __forceinline__ void load_half_frags(uint4 (&F)[NB][2], const uint4* fr0, int h) {
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    F[t][0] = fr0[t * 128 + 2 * h];
    F[t][1] = fr0[t * 128 + 2 * h + 1];
  }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Where a piece's chunks sit in its slot.  In a full K block one tensor copy
// brings chunks [ch, ch + 8) of the block, or, for a piece that starts at the
// block start and stops early, chunks [ch + len - 8, ch + len): the coordinates
// outside the block are zero-filled, not read.  So the piece's first chunk is
// at chunk position p0 = 8 - len in that case, else 0.
__device__ __forceinline__ bool piece_by_tensor(const I8Layer& L, const Piece& pc) { return (pc.ch >> 3) < L.nbf; }
__device__ __forceinline__ int piece_p0(const Piece& pc) {
  return ((pc.ch & 7) == 0 && pc.len < kPieceChunks) ? kPieceChunks - pc.len : 0;
}

// Put the piece's codes in flight into the slot.
template <class P>
__device__ __forceinline__ void issue_piece(const P& p, const Piece& pc, uint32_t slot, uint64_t* bar,
                                            int lane) {
  const I8Layer& L = p.L[pc.li];
  const int64_t row0 = pc.tile * 16;
  const int t = L.nbranch == 2 ? pc.mat >> 1 : pc.mat, br = L.nbranch == 2 ? pc.mat & 1 : 0;
  if (piece_by_tensor(L, pc)) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, kSlotBytes);  // the whole box, zero-filled parts included
      const int cib = piece_p0(pc) ? pc.len - kPieceChunks : (pc.ch & 7);
      tma_load_4d(slot, &L.tmap[br], 0, (int)((int64_t)t * L.N + row0), cib, pc.ch >> 3, bar);
    }
    return;
  }
  // Last, partial K block of the rows: lanes 0..15 each copy one code row.
  const int rows = (int)(L.N - row0 < 16 ? L.N - row0 : 16);
  const int64_t kend = (int64_t)(pc.ch + pc.len) * 256 < L.K ? (int64_t)(pc.ch + pc.len) * 256 : L.K;
  const uint32_t bytes = (uint32_t)((kend - (int64_t)pc.ch * 256) >> 2);
  if (lane == 0) mbar_arrive_expect_tx(bar, bytes * (uint32_t)rows);
  __syncwarp();
  if (lane < rows) {
    const int64_t rb = L.K >> 2;
    const uint8_t* src = L.codes[br] + ((int64_t)t * L.N + row0 + lane) * rb + (int64_t)pc.ch * 64;
    bulk_g2s(slot + lane * 512, src, bytes, bar);
  }
}

template <class P, int NB>
__global__ void __launch_bounds__(kWarps * 32, ctas_per_sm(NB)) gemv_i8_kernel(const __grid_constant__ P p) {
  constexpr int AQ = NB == 1 ? 4 : NB;  // int32 sums per plane: per position q (one token) or per token
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * 2 * kSlotBytes) + warp * 2;
  const uint32_t slots = smem_u32(smem + warp * 2 * kSlotBytes);
  const uint32_t slots0 = smem_u32(smem);
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // W <= C warps take part, so every range is non-empty and the warps owning a
  // tile's chunks are consecutive.
  const int64_t C = p.total_chunks;
  const int64_t W = (int64_t)gridDim.x * kWarps < C ? (int64_t)gridDim.x * kWarps : C;
  // CTAs b, b + sms, ... usually share an SM; giving them adjacent ranges lets
  // them share activation fragments in L1.
  const int64_t lb = p.sms > 0 ? (int64_t)(blockIdx.x % p.sms) * (gridDim.x / p.sms) + blockIdx.x / p.sms
                               : (int64_t)blockIdx.x;
  const int64_t gw = lb * kWarps + warp;
  if (gw >= W) return;
  const int64_t c_lo = range_lo(gw, C, W), c_hi = range_lo(gw + 1, C, W);

  // warm the TMA descriptor cache with this call's code maps, once per CTA
  if (warp == 0 && lane < 2 * p.count && p.L[lane >> 1].nbf > 0 && (lane & 1) < p.L[lane >> 1].nbranch)
    asm volatile("prefetch.tensormap [%0];" ::"l"(&p.L[lane >> 1].tmap[lane & 1]) : "memory");
  int abort_flag = 0;
  uint32_t phases = 0u;  // bit s: parity of the next completion of slot s
  int s = 0;
  // The code bytes do not depend on the prep kernel: the first two pieces are
  // put in flight before waiting for the prep kernel's activation digits.
  Piece cur = make_piece(p, c_lo, c_hi);
  issue_piece(p, cur, slots, &bars[0], lane);
  bool prep_done = false;
  double yr[NB][2], yi[NB][2];  // per token, rows g, g+8 of the current tile (tq == 0)
#pragma unroll
  for (int t = 0; t < NB; ++t) yr[t][0] = yr[t][1] = yi[t][0] = yi[t][1] = 0.0;

  for (;;) {
    const int64_t nc = cur.gbegin + cur.len;
    const bool has_next = nc < c_hi;
    Piece nxt;
    if (has_next) {
      nxt = next_piece(p, cur, c_hi);
      issue_piece(p, nxt, slots + (s ^ 1) * kSlotBytes, &bars[s ^ 1], lane);
    }
    if (!prep_done) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      prep_done = true;
    }
    // While the codes are in flight: this lane's fragments of the piece's first
    // chunk and the inputs of its combine step.
    const I8Layer& L = p.L[cur.li];
    const int blk = cur.ch >> 3;
    // lane's fragments of the piece's first chunk, token 0 (tokens follow at 128 uint4, chunks at NB * 128).
    // The prep kernel writes them while this grid runs (programmatic launch), so they are read with
    // ordinary loads, not through the read-only path.
    const uint4* fr = L.frag + ((((int64_t)blk * 8 + (cur.ch & 7)) * NB) * 32 + lane) * 4;
    constexpr int kF0 = NB == 1 ? 4 : 2;  // one token: the whole first chunk; several: its first half
    uint4 F0[NB][kF0];
#pragma unroll
    for (int tk = 0; tk < NB; ++tk)
#pragma unroll
      for (int k = 0; k < kF0; ++k) F0[tk][k] = fr[tk * 128 + k];
    const int t = L.nbranch == 2 ? cur.mat >> 1 : cur.mat, br = L.nbranch == 2 ? cur.mat & 1 : 0;
    float sr = 0.0f, si = 0.0f;
    int bexp[NB];
    double bs_re[NB], bs_im[NB];
#pragma unroll
    for (int tk = 0; tk < NB; ++tk) {
      bexp[tk] = 0;
      bs_re[tk] = bs_im[tk] = 0.0;
    }
    if (tq == 0) {
      sr = __ldg(L.scales[br] + 2 * t);
      si = __ldg(L.scales[br] + 2 * t + 1);
#pragma unroll
      for (int tk = 0; tk < NB; ++tk) {
        bexp[tk] = L.bexp[(int64_t)blk * NB + tk];
        // exact sums of v over the piece's chunks, from the prefix sums
        const double* pre = L.bsum + ((int64_t)blk * NB + tk) * 18 + (cur.ch & 7) * 2;
        bs_re[tk] = pre[2 * cur.len] - pre[0];
        bs_im[tk] = pre[2 * cur.len + 1] - pre[1];
      }
    }

    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded_sleep(&bars[s], (phases >> s) & 1u, &abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();  // orders every lane's slot reads after lane 0's completed wait
    phases ^= 1u << s;
    if (!ok) {
      if (lane == 0) set_status(p.status, IFQ_DEV_TIMEOUT);
      if (has_next) {  // let the other slot's copies land before leaving
        volatile int never = 0;
        if (lane == 0) mbar_wait_bounded(&bars[s ^ 1], (phases >> (s ^ 1)) & 1u, &never);
      }
      return;
    }

    const uint32_t slot = slots + s * kSlotBytes;  // shared-window address of this slot
    // Plain shared loads (ordered after the barrier wait above by its memory clobber).
    const uint8_t* sbase = smem + (slot - slots0) + tq * 16;

    int acc0[AQ][4], acc1[AQ][4];  // the piece's int32 sums, started by chunk 0: [q or token][fragment reg]
    // Positions past K carry zero activation digits, so code bytes there (stale or not) add nothing.
    const bool whole = cur.len == kPieceChunks && piece_by_tensor(L, cur);  // a whole K block
    // tensor layout: chunk c at c * 1024 from chunk position p0, rows at 64; row layout: chunks at 64, rows at 512
    const bool tens = piece_by_tensor(L, cur);
    const int cstride = tens ? 1024 / 16 : 64 / 16, rstride = tens ? 64 : 512;
    const uint4* rowa = reinterpret_cast<const uint4*>(sbase + (tens ? piece_p0(cur) * 1024 : 0) + g * rstride);
    const uint4* rowb = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(rowa) + 8 * rstride);
    if constexpr (NB == 1) {
      const uint4(&F00)[4] = F0[0];
      if (whole) {
        uint4 Fc[4] = {F00[0], F00[1], F00[2], F00[3]};
#pragma unroll
        for (int c = 0; c < kPieceChunks; ++c) {
          uint4 Fn[4];
          if (c + 1 < kPieceChunks) {
#pragma unroll
            for (int k = 0; k < 4; ++k) Fn[k] = fr[(c + 1) * 128 + k];
          }
          if (c == 0)
            chunk_mma<true>(acc0, acc1, rowa, rowb, Fc);
          else
            chunk_mma<false>(acc0, acc1, rowa + c * 64, rowb + c * 64, Fc);
          if (c + 1 < kPieceChunks) {
#pragma unroll
            for (int k = 0; k < 4; ++k) Fc[k] = Fn[k];
          }
        }
      } else {
        chunk_mma<true>(acc0, acc1, rowa, rowb, F00);
#pragma unroll 1
        for (int c = 1; c < cur.len; ++c) {
          uint4 F[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) F[k] = fr[c * 128 + k];
          chunk_mma<false>(acc0, acc1, rowa + c * cstride, rowb + c * cstride, F);
        }
      }
    } else {
      // half-chunks h = 2 c + word pair; each token's fragments of the next half load during this one
      uint4 Fh[NB][2];
#pragma unroll
      for (int tk = 0; tk < NB; ++tk) Fh[tk][0] = F0[tk][0], Fh[tk][1] = F0[tk][1];
      const int nh = 2 * cur.len;
#pragma unroll 2
      for (int h = 0; h < nh; ++h) {
        const int c = h >> 1, wp = h & 1;
        uint4 Fn[NB][2];
        if (h + 1 < nh) load_half_frags<NB>(Fn, fr + ((h + 1) >> 1) * NB * 128, (h + 1) & 1);
        const uint4 va = rowa[c * cstride], vb = rowb[c * cstride];
        const uint32_t a0 = wp ? va.z : va.x, a1 = wp ? va.w : va.y;
        const uint32_t b0 = wp ? vb.z : vb.x, b1 = wp ? vb.w : vb.y;
        if (h == 0)
          half_chunk_mma<NB, true>(acc0, acc1, a0, a1, b0, b1, Fh);
        else
          half_chunk_mma<NB, false>(acc0, acc1, a0, a1, b0, b1, Fh);
        if (h + 1 < nh) {
#pragma unroll
          for (int tk = 0; tk < NB; ++tk) Fh[tk][0] = Fn[tk][0], Fh[tk][1] = Fn[tk][1];
        }
      }
    }
    __syncwarp();  // every lane is done with this slot before it is refilled

    // ---- combine, per token.  One token: the planes carry weights 2*4^q (-128 at q = 3),
    // so 64 a_0 + 16 a_1 + 4 a_2 - a_3 = 128 G; several tokens: weight 2 everywhere, so
    // 64 a = 128 G.  Both exact in int32.  The digit columns are then merged in float32:
    // its rounding (2^-24 of at most 3 sum_j |v_j| per piece) stays far inside the
    // product tolerance.
#pragma unroll
    for (int tk = 0; tk < NB; ++tk) {
      float qa[2], qb[2];  // rows g, g+8: this thread's two digit columns, merged
      {
        int G0[4], G1[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if constexpr (NB == 1) {
            G0[r] = 64 * acc0[0][r] + 16 * acc0[1][r] + 4 * acc0[2][r] - acc0[3][r];
            G1[r] = 64 * acc1[0][r] + 16 * acc1[1][r] + 4 * acc1[2][r] - acc1[3][r];
          } else {
            G0[r] = 64 * acc0[tk][r];
            G1[r] = 64 * acc1[tk][r];
          }
        }
        const float dscale = (tq & 1) ? 65536.0f : 1.0f;  // columns 2tq, 2tq+1 hold digits 2(tq&1), +1
        qa[0] = dscale * fmaf(256.0f, (float)G0[1], (float)G0[0]);
        qa[1] = dscale * fmaf(256.0f, (float)G0[3], (float)G0[2]);
        qb[0] = dscale * fmaf(256.0f, (float)G1[1], (float)G1[0]);
        qb[1] = dscale * fmaf(256.0f, (float)G1[3], (float)G1[2]);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        qa[r] += __shfl_xor_sync(0xffffffffu, qa[r], 1);
        qb[r] += __shfl_xor_sync(0xffffffffu, qb[r], 1);
      }
      float oa[2], ob[2];  // threads tq 0,1 hold plane re, 2,3 plane im: fetch the other plane
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        oa[r] = __shfl_xor_sync(0xffffffffu, qa[r], 2);
        ob[r] = __shfl_xor_sync(0xffffffffu, qb[r], 2);
      }
      if (tq == 0) {
        const double inv = __longlong_as_double((long long)(1023 - bexp[tk]) << 52);  // 2^-E (outside float range)
        const float fre = (float)bs_re[tk], fim = (float)bs_im[tk];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          // G0 = QA / 128, G1 = QB / 128;  P_r = S - G0 - G1,  P_i = G0 - G1 (S: the piece's sums of v)
          const float Prr = fre - (qa[r] + qb[r]) * 0.0078125f;
          const float Pir = (qa[r] - qb[r]) * 0.0078125f;
          const float Pri = fim - (oa[r] + ob[r]) * 0.0078125f;
          const float Pii = (oa[r] - ob[r]) * 0.0078125f;
          float vr, vi;
          if (br == 0) {
            vr = sr * Prr - si * Pii;
            vi = sr * Pri + si * Pir;
          } else {
            vr = sr * Prr + si * Pii;
            vi = si * Pir - sr * Pri;
          }
          yr[tk][r] += (double)vr * inv;
          yi[tk][r] += (double)vi * inv;
        }
      }
    }

    // ---- tile finished for this warp: write y, or a partial and possibly reduce.
    // The tile's chunks [0, tc) are split into contiguous portions, one per warp
    // that touched it.  A portion starting at local chunk c0 leaves its partial in
    // slot c0 and the start of the next portion in next[c0]; the ticket counts
    // finished chunks, and the warp that completes it adds the partials in chunk
    // order, so the result does not depend on timing.
    const bool tile_done = !has_next || nxt.li != cur.li || nxt.tile != cur.tile;
    if (tile_done) {
      const int64_t tc = (int64_t)p.T * L.nbranch * L.nch;
      const int64_t tb = L.chunk_begin + cur.tile * tc;
      const int64_t c0 = (c_lo > tb ? c_lo : tb) - tb, c1 = nc - tb;  // this warp's portion of the tile
      const int64_t row0 = cur.tile * 16;
      if (c0 == 0 && c1 == tc) {
        if (tq == 0) {
#pragma unroll
          for (int tk = 0; tk < NB; ++tk)
#pragma unroll
            for (int r = 0; r < 2; ++r)
              if (tk < p.B && row0 + g + 8 * r < L.N)
                store_y(L, tk * L.N + row0 + g + 8 * r, (float)yr[tk][r], (float)yi[tk][r]);
        }
      } else {
        const int64_t slot0 = cur.tile * tc;
        float* part = L.partials + (slot0 + c0) * 32 * NB;  // [token][row][re, im]
        if (tq == 0) {
#pragma unroll
          for (int tk = 0; tk < NB; ++tk)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              part[tk * 32 + 2 * (g + 8 * r)] = (float)yr[tk][r];
              part[tk * 32 + 2 * (g + 8 * r) + 1] = (float)yi[tk][r];
            }
        }
        if (lane == 0) L.next[slot0 + c0] = (int)c1;
        __syncwarp();
        unsigned prev = 0;
        // acq_rel at gpu scope: the partial stores of the whole warp (ordered before
        // lane 0 by the warp barrier above) are visible before the ticket moves, and
        // the last arriver sees every other portion's stores after its own atomic.
        if (lane == 0) prev = atom_add_acq_rel_gpu(L.tickets + cur.tile, (unsigned)(c1 - c0));
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if ((int64_t)prev + (c1 - c0) == tc) {
          __syncwarp();
          if (lane < 16 && row0 + lane < L.N) {
            float ar[NB], ai[NB];
#pragma unroll
            for (int tk = 0; tk < NB; ++tk) ar[tk] = ai[tk] = 0.0f;
            int64_t c = 0;
            for (int64_t guard = 0; c < tc && guard < tc; ++guard) {
              const float* pt = L.partials + (slot0 + c) * 32 * NB + 2 * lane;
#pragma unroll
              for (int tk = 0; tk < NB; ++tk) {
                ar[tk] += __ldcg(pt + tk * 32);
                ai[tk] += __ldcg(pt + tk * 32 + 1);
              }
              const int64_t cn = __ldcg(L.next + slot0 + c);
              if (cn <= c) break;  // cannot happen: portions are non-empty and ordered
              c = cn;
            }
#pragma unroll
            for (int tk = 0; tk < NB; ++tk)
              if (tk < p.B) store_y(L, tk * L.N + row0 + lane, ar[tk], ai[tk]);
          }
          if (lane == 0) L.tickets[cur.tile] = 0u;
        }
      }
#pragma unroll
      for (int tk = 0; tk < NB; ++tk) yr[tk][0] = yr[tk][1] = yi[tk][0] = yi[tk][1] = 0.0;
    }
    if (!has_next) break;
    cur = nxt;
    s ^= 1;
  }
}

// Workspace layout: 256 B header (unused), then per layer, each region
// 256-byte aligned: fragments, chunk sums, block exponents, partials, portion
// links, tickets.
struct WsLayout {
  size_t frag, bsum, bexp, part, next, tick;
};

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// nb: tokens the kernels are built for (1, 2 or 4).
size_t layout_layers(const ifq_layer* Ls, int count, int T, int nb, WsLayout* out) {
  size_t off = 256;
  for (int i = 0; i < count; ++i) {
    const int64_t tiles = (Ls[i].N + 15) / 16;
    const int64_t blocks = (Ls[i].K + kKBlock - 1) / kKBlock;
    const int64_t nmat = (int64_t)T * (Ls[i].codes_w ? 2 : 1);
    WsLayout w;
    w.frag = off;
    off = align256(off + (size_t)blocks * 8 * nb * 32 * 64);
    w.bsum = off;
    off = align256(off + (size_t)blocks * nb * 18 * 8);
    w.bexp = off;
    off = align256(off + (size_t)blocks * nb * 4);
    const int64_t nch = (Ls[i].K + 255) / 256;
    w.part = off;
    off = align256(off + (size_t)tiles * nmat * nch * nb * 32 * 4);
    w.next = off;
    off = align256(off + (size_t)tiles * nmat * nch * 4);
    w.tick = off;
    off = align256(off + (size_t)tiles * 4);
    if (out) out[i] = w;
  }
  return off;
}

}  // namespace

// Tokens per launch the integer path is built for: B = 1 or 2.  (The template also builds
// for four tokens, B = 3..4 padded; the bf16 path with K segments measured faster there.)
int gemv_i8_tokens(int B) { return B <= 1 ? 1 : 2; }

size_t gemv_i8_workspace_bytes(const ifq_layer* Ls, int count, int T, int B) {
  return layout_layers(Ls, count, T, gemv_i8_tokens(B), nullptr);
}

namespace {

template <int kCap, int NB>
cudaError_t kernel_attr() {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemv_i8_kernel<I8Params<kCap>, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kMainSmem);
  });
  return attr_err;
}

// The launch parameters of one call: the layers' descriptors and workspace slices, the tensor maps
// of the codes, the prep grid and the main grid.
template <int kCap, int NB>
cudaError_t build_params(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status,
                         I8Params<kCap>& p, int64_t& preps, int64_t& ctas) {
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.B = B;
  p.status = dev_status;
  WsLayout lay[IFQ_MAX_GROUP];
  layout_layers(Ls, count, T, NB, lay);
  char* base = static_cast<char*>(ws);
  int64_t chunks = 0;
  preps = 0;
  for (int i = 0; i < count; ++i) {
    I8Layer& a = p.L[i];
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
    a.tiles = (int32_t)((a.N + 15) / 16);
    a.blocks = (int32_t)((a.K + kKBlock - 1) / kKBlock);
    a.frag = reinterpret_cast<uint4*>(base + lay[i].frag);
    a.bsum = reinterpret_cast<double*>(base + lay[i].bsum);
    a.bexp = reinterpret_cast<int*>(base + lay[i].bexp);
    a.partials = reinterpret_cast<float*>(base + lay[i].part);
    a.next = reinterpret_cast<int*>(base + lay[i].next);
    a.tickets = reinterpret_cast<unsigned int*>(base + lay[i].tick);
    a.nch = (int32_t)((a.K + 255) / 256);
    a.nbf = (int32_t)(a.K / kKBlock);
    if ((int64_t)T * a.N >= ((int64_t)1 << 31)) a.nbf = 0;  // rows beyond a tensor coordinate: row copies only
    for (int b = 0; b < a.nbranch && a.nbf > 0; ++b) {
      // (byte in chunk, row of [T][N], chunk in block, block): strides K/4, 64, 512 bytes
      const uint64_t dims[4] = {64, (uint64_t)T * (uint64_t)a.N, 8, (uint64_t)a.nbf};
      const uint64_t strides[3] = {(uint64_t)a.K / 4, 64, 512};
      const uint32_t box[4] = {64, 16, 8, 1};
      if (!encode_tiled_map(&a.tmap[b], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.codes[b], dims, strides, box,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    }
    a.chunk_begin = p.chunk_begin[i] = chunks;
    a.prep_begin = p.prep_begin[i] = preps;
    chunks += (int64_t)a.tiles * T * a.nbranch * a.nch;
    preps += (int64_t)a.blocks * 8;
  }
  p.total_chunks = chunks;
  if (chunks >= ((int64_t)1 << 40) || preps > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ctas = (int64_t)sms * ctas_per_sm(NB);
  const int64_t need = (chunks + kWarps - 1) / kWarps;  // at least one chunk per warp
  if (ctas > need) ctas = need;
  p.sms = ctas == (int64_t)sms * ctas_per_sm(NB) ? sms : 0;
  return cudaSuccess;
}

// The prep kernel, then the main kernel as its programmatic dependent.
template <int kCap, int NB>
cudaError_t launch_params(const I8Params<kCap>& p, int64_t preps, int64_t ctas, cudaStream_t s) {
  cudaError_t e = kernel_attr<kCap, NB>();
  if (e != cudaSuccess) return e;
  gemv_prep_kernel<I8Params<kCap>, NB><<<(unsigned)preps, kPrepThreads, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = kMainSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<I8Params<kCap>, NB>, p);
}

template <int kCap, int NB>
cudaError_t launch_cap(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, cudaStream_t s) {
  I8Params<kCap> p;
  int64_t preps = 0, ctas = 0;
  const cudaError_t e = build_params<kCap, NB>(Ls, count, T, B, ws, dev_status, p, preps, ctas);
  if (e != cudaSuccess) return e;
  return launch_params<kCap, NB>(p, preps, ctas, s);
}

// A prepared call: the finished parameters of the largest group, reused by every run.
struct alignas(64) I8Plan {
  int32_t nb, cap;
  int64_t preps, ctas;
  alignas(64) unsigned char params[sizeof(I8Params<IFQ_MAX_GROUP>)];
};

template <int NB>
cudaError_t plan_nb(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* st, I8Plan& pl) {
  pl.nb = NB;
  pl.cap = count <= 8 ? 8 : IFQ_MAX_GROUP;
  if (pl.cap == 8)
    return build_params<8, NB>(Ls, count, T, B, ws, st, *reinterpret_cast<I8Params<8>*>(pl.params), pl.preps, pl.ctas);
  return build_params<IFQ_MAX_GROUP, NB>(Ls, count, T, B, ws, st,
                                         *reinterpret_cast<I8Params<IFQ_MAX_GROUP>*>(pl.params), pl.preps, pl.ctas);
}

template <int NB>
cudaError_t run_nb(const I8Plan& pl, cudaStream_t s) {
  if (pl.cap == 8) return launch_params<8, NB>(*reinterpret_cast<const I8Params<8>*>(pl.params), pl.preps, pl.ctas, s);
  return launch_params<IFQ_MAX_GROUP, NB>(*reinterpret_cast<const I8Params<IFQ_MAX_GROUP>*>(pl.params), pl.preps,
                                          pl.ctas, s);
}

}  // namespace

template <int NB>
cudaError_t launch_nb(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, cudaStream_t s) {
  return count <= 8 ? launch_cap<8, NB>(Ls, count, T, B, ws, dev_status, s)
                    : launch_cap<IFQ_MAX_GROUP, NB>(Ls, count, T, B, ws, dev_status, s);
}

cudaError_t launch_gemv_i8(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status,
                           cudaStream_t s) {
  return gemv_i8_tokens(B) == 1 ? launch_nb<1>(Ls, count, T, B, ws, dev_status, s)
                                : launch_nb<2>(Ls, count, T, B, ws, dev_status, s);
}

size_t gemv_i8_plan_bytes() { return sizeof(I8Plan); }

cudaError_t plan_gemv_i8(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, void* dst) {
  I8Plan& pl = *static_cast<I8Plan*>(dst);
  return gemv_i8_tokens(B) == 1 ? plan_nb<1>(Ls, count, T, B, ws, dev_status, pl)
                                : plan_nb<2>(Ls, count, T, B, ws, dev_status, pl);
}

cudaError_t run_gemv_i8_plan(const void* src, cudaStream_t s) {
  const I8Plan& pl = *static_cast<const I8Plan*>(src);
  switch (pl.nb) {
    case 1: return run_nb<1>(pl, s);
    case 2: return run_nb<2>(pl, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ifq
