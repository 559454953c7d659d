// Prefill product on the 5th-generation tensor cores (tcgen05 / TMEM)
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2 -- the GEMM rebuilt
// from additions, subtractions and swaps).
//
// For each (stage t, branch) code matrix the per-class signed sums of one tile
// are one real MMA with exact operands:
//     D = [Br; Bi] [X_re; X_im]^T
// Br, Bi in {-2, 0, +2} are the code's real / imaginary parts (times 2),
// expanded from the packed codes straight into TMEM, where they are the MMA's
// A operand (M = 128: Br and Bi rows of 64 outputs).  X_* are the bf16
// activation planes [M][K], brought in by TMA; the two 128-token tiles of a K
// block form the B operand (N = 256: real plane, then imaginary plane).
// Products are exact and accumulate in float32 in TMEM; each lane holds one
// (output, class) row and the columns hold (plane, token), so the four
// quadrants are
//     P_rr = Br x_re,  P_ri = Br x_im,  P_ir = Bi x_re,  P_ii = Bi x_im
// and their scales are applied in the epilogue:
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
// Keeping the expanded codes out of shared memory halves its traffic per MMA
// (activations in by TMA and out to the tensor core, 16 KB per K16 step), so
// the MMA is not starved by shared-memory bandwidth.
//
// One persistent launch per call: one CTA per SM walks a static list of the call's tiles (all
// layers, longest K first), so the tail of one layer's tiles is filled by the next layer's, and the
// copy / expansion / MMA pipeline and the TMEM allocation carry over from tile to tile; while the
// epilogue stores one tile's y, the MMAs of the next tile run.
// CTA tile: 128 tokens x 64 outputs; K in blocks of 64.  Warp roles (15 warps):
//   0-3   expanders: code tile -> A rows in TMEM (warp w writes lanes 32w..32w+31;
//         lane 32w + j holds output 16w + (j & 15), class Br for j < 16, Bi else)
//   4-11  epilogue: tcgen05.ld of the finished (stage, branch) accumulator, the
//         Br/Bi exchange between lanes j and j ^ 16, scales, and y accumulated
//         in shared memory (the first pass of a tile overwrites it); y stored to
//         global at the tile's end.  Each warp releases the accumulator right
//         after its last TMEM read of the pass, before that chunk's arithmetic.
//   12    TMA producer of the activations: X_re, X_im tiles (128 B swizzle), 4 stages
//   13    TMEM allocator and single-thread MMA issuer (M=128, N=256, K=16 per instruction)
//   14    TMA producer of the codes: 64 x 16-byte tiles in a ring of 16 stages of their own, so
//         that an expander finds its codes in place as soon as its A stage is free
// TMEM: the accumulator (256 columns) and 8 stages of A (32 columns each), twice the activation
// stages, so that the expanders run up to 8 stages ahead of the MMAs.
// Every mbarrier wait is bounded; a lost wait sets IFQ_DEV_TIMEOUT, the CTA
// drains its outstanding copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int BM = 128;      // tokens per tile; the MMA's N is 2 BM (both planes)
constexpr int BN = 64;       // outputs per tile; the MMA's M is 2 BN (Br and Bi rows)
constexpr int BK = 64;       // K per stage (one 128-byte swizzle row of bf16)
constexpr int STAGES = 4;                    // activation stages in shared memory
constexpr int ASTAGES = 8;                   // stages of the expanded codes (A) in TMEM
constexpr int CSTAGES = 16;                  // code stages: a ring of its own, filled far ahead
constexpr int kExpWarps = 4;
constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter, each half the tokens
constexpr int kProducerWarp = kExpWarps + kEpiWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kCodeWarp = kMmaWarp + 1;
constexpr int kThreads = (kCodeWarp + 1) * 32;
constexpr uint32_t kTileX = BM * BK * 2;        // 16 KB per activation plane
constexpr uint32_t kTileC = BN * (BK / 4);      // 1 KB of codes
constexpr uint32_t kStageBytes = 2 * kTileX;    // 32 KB: X_re, X_im
constexpr uint32_t kTmaBytes = 2 * kTileX;
constexpr uint32_t kCodeOff = STAGES * kStageBytes;
constexpr uint32_t kYOff = kCodeOff + CSTAGES * kTileC;
constexpr uint32_t kYFloats = 2 * BM * BN;      // y accumulators of the tile: [plane][token][output]
constexpr uint32_t kSmemBytes = kYOff + kYFloats * 4 + 1024 /*align*/ + 512 /*barriers*/;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol = 2 * BM;              // A stage a at columns kAcol + 32 a
constexpr uint32_t kIdesc = umma_idesc_bf16(2 * BN, 2 * BM);
static_assert(kAcol + ASTAGES * (BK / 2) <= kTmemCols, "TMEM budget");

// One layer of a grouped call.  Its output tiles are numbered from tile_begin: token tile
// (128 tokens) major, output tile (64 outputs) minor, so that the tiles running at the same time
// share their activation tiles in L2.
struct __align__(64) GemmLayer {
  CUtensorMap tmap_x[2];      // bf16 [M][K]: box {64, 128}, 128 B swizzle
  CUtensorMap tmap_codes[2];  // u8 [T*N][K/4]: box {16, 64}
  const float* scales[2];
  float* y[2];
  const float* rot[2];        // optional epilogue rotation [M][N] (re, im), or null
  int64_t N, K;
  int64_t tile_begin;
  int32_t nbranch, tiles_n;
};

// Capacity kCap >= count.  The layers are stored heaviest first (most K steps per tile), so that the
// CTAs take the long tiles before the short ones.
template <int kCap>
struct __align__(64) GemmParams {
  int64_t tile_begin[kCap];   // copies of the layers' first tiles, for the tile -> layer search
  int64_t tiles;              // all tiles of the call
  int64_t M;
  int count, T;
  uint64_t wait_ns;           // limit of each pipeline wait (drains after a lost wait keep IFQ_WAIT_LIMIT_NS)
  uint32_t* status;
  GemmLayer L[kCap];
};

static_assert(sizeof(GemmParams<IFQ_MAX_GROUP>) <= 32764, "kernel parameter block limit");

struct Smem {
  uint64_t full_tma[STAGES];
  uint64_t empty[STAGES];
  uint64_t full_a[ASTAGES];
  uint64_t empty_a[ASTAGES];
  uint64_t full_c[CSTAGES];
  uint64_t empty_c[CSTAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int epi_stop;
};

static_assert(sizeof(Smem) <= 512, "barrier block");

struct Tile {
  int li;
  int64_t n0, m0;
};

template <int kCap>
__device__ __forceinline__ Tile decode_tile(const GemmParams<kCap>& p, int64_t t) {
  int li = 0;
  while (li + 1 < p.count && t >= p.tile_begin[li + 1]) ++li;
  const int64_t local = t - p.tile_begin[li];
  const int64_t tn = p.L[li].tiles_n;
  Tile r;
  r.li = li;
  r.n0 = (local % tn) * BN;
  r.m0 = (local / tn) * BM;
  return r;
}

// Two codes (bits 0..3 of `nib`) -> one 32-bit column of A: the bf16 pair (Br or Bi of the
// lower code in the low half).  The multiply places code 0's axis bit on bit 14 (the exponent
// bit of 2.0) and its sign on bit 15, code 1's on bits 30 and 31.  Bi is then +-2 where the
// axis bit is set and +-0 where it is not; Br flips the axis bit.  A signed zero adds nothing
// to the float32 sums, so no further masking is needed.
__device__ __forceinline__ uint32_t expand_pair(uint32_t nib, bool imag) {
  const uint32_t spread = (nib * 0x10004000u) & 0xC000C000u;
  return imag ? spread : spread ^ 0x40004000u;
}

// Store a finished tile's y from shared memory ([plane][token][output]), rows of 64 outputs as float4,
// with the optional rotation.  e: the calling thread's index among the 256 epilogue threads.
__device__ __forceinline__ void store_tile_y(const GemmLayer& L, int64_t M, const Tile& tl, const float* ys, int e) {
  const bool vec = (L.N & 3) == 0 && tl.n0 + BN <= L.N;
  for (int idx = e; idx < BM * (BN / 4); idx += kEpiWarps * 32) {
    const int tok = idx / (BN / 4), c4 = idx - tok * (BN / 4);
    const int64_t m = tl.m0 + tok;
    if (m >= M) continue;
    const float4 r4 = *reinterpret_cast<const float4*>(ys + tok * BN + 4 * c4);
    const float4 i4 = *reinterpret_cast<const float4*>(ys + BM * BN + tok * BN + 4 * c4);
    float vr[4] = {r4.x, r4.y, r4.z, r4.w}, vi[4] = {i4.x, i4.y, i4.z, i4.w};
    const int64_t o = m * L.N + tl.n0 + 4 * c4;
    const int nv = vec ? 4 : (int)(L.N - (tl.n0 + 4 * c4) < 4 ? L.N - (tl.n0 + 4 * c4) : 4);  // valid outputs
    if (L.rot[0]) {  // complex RoPE: times rot[m][n]
      float cr[4] = {1.f, 1.f, 1.f, 1.f}, ci[4] = {0.f, 0.f, 0.f, 0.f};
      if (vec) {
        const float4 c = __ldg(reinterpret_cast<const float4*>(L.rot[0] + o));
        const float4 d = __ldg(reinterpret_cast<const float4*>(L.rot[1] + o));
        cr[0] = c.x; cr[1] = c.y; cr[2] = c.z; cr[3] = c.w;
        ci[0] = d.x; ci[1] = d.y; ci[2] = d.z; ci[3] = d.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nv) {
            cr[j] = __ldg(L.rot[0] + o + j);
            ci[j] = __ldg(L.rot[1] + o + j);
          }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float r = cr[j] * vr[j] - ci[j] * vi[j], im = cr[j] * vi[j] + ci[j] * vr[j];
        vr[j] = r;
        vi[j] = im;
      }
    }
    if (vec) {
      *reinterpret_cast<float4*>(L.y[0] + o) = make_float4(vr[0], vr[1], vr[2], vr[3]);
      *reinterpret_cast<float4*>(L.y[1] + o) = make_float4(vi[0], vi[1], vi[2], vi[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < nv) {
          L.y[0][o + j] = vr[j];
          L.y[1][o + j] = vi[j];
        }
    }
  }
}

template <int kCap>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmParams<kCap> p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ys = reinterpret_cast<float*>(smem + kYOff);
  Smem* S = reinterpret_cast<Smem*>(smem + kYOff + kYFloats * 4);
  volatile int* abort = &S->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = p.T;  // passes per tile: T stages x the layer's branches (times nbranch below)
  const int64_t t_first = blockIdx.x, t_step = gridDim.x;

  auto xtile = [&](int s) { return smem + s * kStageBytes; };  // X_re, then X_im 16 KB later
  auto ctile = [&](int c) { return smem + kCodeOff + c * kTileC; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full_tma[s], 1);
      mbar_init(&S->empty[s], 1);
    }
    for (int a = 0; a < ASTAGES; ++a) {
      mbar_init(&S->full_a[a], kExpWarps);
      mbar_init(&S->empty_a[a], 1);
    }
    for (int c = 0; c < CSTAGES; ++c) {
      mbar_init(&S->full_c[c], 1);
      mbar_init(&S->empty_c[c], kExpWarps);
    }
    mbar_init(&S->acc_full, 1);
    mbar_init(&S->acc_empty, kEpiWarps);
    mbar_init(&S->drain, 1);
    S->abort = 0;
    S->epi_stop = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane < p.count) {
    const GemmLayer& L = p.L[lane];
    prefetch_tmap(&L.tmap_x[0]);
    prefetch_tmap(&L.tmap_x[1]);
    prefetch_tmap(&L.tmap_codes[0]);
    if (L.nbranch > 1) prefetch_tmap(&L.tmap_codes[1]);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      int it = 0;  // stage fills of this CTA, across its tiles
      for (int64_t tt = t_first; tt < p.tiles && !*abort; tt += t_step) {
        const Tile tl = decode_tile(p, tt);
        const GemmLayer& L = p.L[tl.li];
        const int KB = (int)(L.K / BK), np = P * L.nbranch;
        bool ok = true;
        for (int q = 0; q < np && ok; ++q) {
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
            if (!mbar_wait_bounded_ns(&S->empty[s], ph ^ 1u, abort, p.wait_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&S->full_tma[s], kTmaBytes);
            tma_load_2d(xtile(s), &L.tmap_x[0], kb * BK, (int32_t)tl.m0, &S->full_tma[s]);
            tma_load_2d(xtile(s) + kTileX, &L.tmap_x[1], kb * BK, (int32_t)tl.m0, &S->full_tma[s]);
            ++issued[s];
          }
        }
        if (!ok) break;
      }
      if (*abort) {
        // Let every issued copy land before the CTA's shared memory is released.
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued[s] > 0) mbar_wait_bounded(&S->full_tma[s], (uint32_t)(issued[s] - 1) & 1u, &never);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
    const uint64_t xdesc0 = umma_desc_sw128(smem_u32(xtile(0)));
    int it = 0, gp = 0;  // stage uses and (stage, branch) passes of this CTA, across its tiles
    bool ok = true;
    for (int64_t tt = t_first; tt < p.tiles && ok; tt += t_step) {
      const Tile tl = decode_tile(p, tt);
      const GemmLayer& L = p.L[tl.li];
      const int KB = (int)(L.K / BK), np = P * L.nbranch;
      for (int q = 0; q < np && ok; ++q, ++gp) {
        // the epilogue has read the previous pass's accumulator
        int w_ok = 1;
        if (lane == 0) w_ok = !*abort && mbar_wait_bounded_ns(&S->acc_empty, ((uint32_t)gp & 1u) ^ 1u, abort, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;  // every lane takes lane 0's result: the warp stays converged
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, sa = it % ASTAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u, pha = (uint32_t)(it / ASTAGES) & 1u;
          if (lane == 0)
            w_ok = mbar_wait_bounded_ns(&S->full_tma[s], ph, abort, p.wait_ns) &&
                   mbar_wait_bounded_ns(&S->full_a[sa], pha, abort, p.wait_ns);
          ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
          if (!ok) break;
          tc_fence_after();
          // the four K16 steps of the stage: B advances 32 bytes (2 descriptor units) per step inside the
          // 128-byte swizzle row, A 8 TMEM columns
          umma_bf16_ta_x4(tmem, tmem + kAcol + 32 * sa, xdesc0 + (uint64_t)((uint32_t)s * (kStageBytes >> 4)), kIdesc,
                          kb != 0);
          umma_commit_elect(&S->empty[s]);     // the activation stage may be refilled
          umma_commit_elect(&S->empty_a[sa]);  // the A stage may be rewritten
        }
        if (!ok) break;
        umma_commit_elect(&S->acc_full);
      }
    }
    if (lane == 0 && *abort) {
      volatile int never = 0;
      umma_commit(&S->drain);
      mbar_wait_bounded(&S->drain, 0u, &never);
    }
  } else if (warp == kCodeWarp) {
    // ------------------------------------------------------------ code producer: the 1 KB code tiles, up
    // to CSTAGES stages ahead of the expanders (the activation stages are far fewer)
    if (lane == 0) {
      int issued[CSTAGES];
      for (int c = 0; c < CSTAGES; ++c) issued[c] = 0;
      int it = 0;
      bool ok = true;
      for (int64_t tt = t_first; tt < p.tiles && ok && !*abort; tt += t_step) {
        const Tile tl = decode_tile(p, tt);
        const GemmLayer& L = p.L[tl.li];
        const int KB = (int)(L.K / BK), np = P * L.nbranch;
        for (int q = 0; q < np && ok; ++q) {
          const int t = q / L.nbranch, br = q % L.nbranch;
          const int32_t crow = (int32_t)((int64_t)t * L.N + tl.n0);
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int c = it % CSTAGES;
            const uint32_t ph = (uint32_t)(it / CSTAGES) & 1u;
            if (!mbar_wait_bounded_ns(&S->empty_c[c], ph ^ 1u, abort, p.wait_ns)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&S->full_c[c], kTileC);
            tma_load_2d(ctile(c), &L.tmap_codes[br], kb * (BK / 4), crow, &S->full_c[c]);
            ++issued[c];
          }
        }
      }
      if (*abort) {
        volatile int never = 0;
        for (int c = 0; c < CSTAGES; ++c)
          if (issued[c] > 0) mbar_wait_bounded(&S->full_c[c], (uint32_t)(issued[c] - 1) & 1u, &never);
      }
    }
  } else if (warp < kExpWarps) {
    // ------------------------------------------------------------ expanders
    const bool imag = lane >= 16;
    const int o = 16 * warp + (lane & 15);   // this lane's output row within the tile
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + kAcol;
    int it = 0;
    bool ok = true;
    for (int64_t tt = t_first; tt < p.tiles && ok; tt += t_step) {
      const Tile tl = decode_tile(p, tt);
      const GemmLayer& L = p.L[tl.li];
      const int KB = (int)(L.K / BK), np = P * L.nbranch;
      for (int q = 0; q < np && ok; ++q) {
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int sa = it % ASTAGES, cs = it % CSTAGES;
          const uint32_t pha = (uint32_t)(it / ASTAGES) & 1u, cph = (uint32_t)(it / CSTAGES) & 1u;
          int w_ok = 1;
          // the A stage is free once the MMAs that read it are done; the codes were loaded far ahead
          if (lane == 0)
            w_ok = mbar_wait_bounded_ns(&S->full_c[cs], cph, abort, p.wait_ns) &&
                   mbar_wait_bounded_ns(&S->empty_a[sa], pha ^ 1u, abort, p.wait_ns);
          ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
          if (!ok) break;
          // Rows past N carry other stages' or no codes; their outputs are never stored.
          const uint4 cw = *reinterpret_cast<const uint4*>(ctile(cs) + o * 16);
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
          uint32_t col[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) col[c] = expand_pair((w[c >> 3] >> (4 * (c & 7))) & 0xFu, imag);
          __syncwarp();
          if (lane == 0) mbar_arrive(&S->empty_c[cs]);  // every lane has its code word in registers
          tmem_st_32x32b_x32(trow + 32 * sa, col);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S->full_a[sa]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;                   // TMEM lane quarter
    const int half = (warp - kExpWarps) >> 2;  // token chunks c with c % 2 == half
    const bool imag = lane >= 16;
    const int o = 16 * qd + (lane & 15);
    const uint32_t trow = tmem + ((uint32_t)(qd * 32) << 16);
    const int e = threadIdx.x - kExpWarps * 32;  // 0..255
    int gp = 0;
    for (int64_t tt = t_first; tt < p.tiles; tt += t_step) {
      const Tile tl = decode_tile(p, tt);
      const GemmLayer& L = p.L[tl.li];
      const int np = P * L.nbranch;
      bool ok = true;
      for (int q = 0; q < np; ++q, ++gp) {
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait_bounded_ns(&S->acc_full, (uint32_t)gp & 1u, abort, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
        if (!ok) break;
        tc_fence_after();
        const int t = q / L.nbranch, br = q % L.nbranch;
        const float hr = 0.5f * __ldg(L.scales[br] + 2 * t);
        const float hi = 0.5f * __ldg(L.scales[br] + 2 * t + 1);
        const float sgn = br == 0 ? -1.0f : 1.0f;
#pragma unroll 1
        for (int c = half; c < BM / 32; c += 2) {
          uint32_t u[32], v[32];
          tmem_ld_32x32b_x32(trow + 32 * c, u);         // this lane's class, real plane, tokens 32c..
          tmem_ld_32x32b_x32(trow + BM + 32 * c, v);    // imaginary plane
          tmem_wait_ld();
          if (c + 2 >= BM / 32) {
            // this warp's last read of the accumulator: the next pass may overwrite it while the
            // values in registers are applied
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->acc_empty);
          }
          // lane j < 16 (Br) takes tokens 32c + 0..15, lane j >= 16 (Bi) tokens 32c + 16..31;
          // each gets the other class's values of its tokens from lane j ^ 16.  The first pass of a
          // tile writes this lane's y entries, the later ones read, update and write them back.
          const int tok0 = 32 * c + (imag ? 16 : 0);
          float* yre = ys + tok0 * BN + o;
          float* yim = ys + BM * BN + tok0 * BN + o;
          float cre[16], cim[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            cre[i] = q == 0 ? 0.0f : yre[i * BN];
            cim[i] = q == 0 ? 0.0f : yim[i * BN];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float mu_lo = __uint_as_float(u[i]), mv_lo = __uint_as_float(v[i]);
            const float mu_hi = __uint_as_float(u[16 + i]), mv_hi = __uint_as_float(v[16 + i]);
            // send the partner the values of the partner's tokens, receive those of mine
            const float pu = __shfl_xor_sync(0xffffffffu, imag ? mu_lo : mu_hi, 16);
            const float pv = __shfl_xor_sync(0xffffffffu, imag ? mv_lo : mv_hi, 16);
            const float mu = imag ? mu_hi : mu_lo, mv = imag ? mv_hi : mv_lo;
            const float P_rr = imag ? pu : mu, P_ri = imag ? pv : mv;
            const float P_ir = imag ? mu : pu, P_ii = imag ? mv : pv;
            cre[i] += hr * P_rr + sgn * hi * P_ii;
            cim[i] += hi * P_ir - sgn * hr * P_ri;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            yre[i * BN] = cre[i];
            yim[i * BN] = cim[i];
          }
        }
      }
      // The tile's y is complete in shared memory.  Every epilogue warp takes the same decision to go
      // on (a lost wait anywhere stops them all at this point), then they store y together.
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      if (e == 0) S->epi_stop = *abort;
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      if (S->epi_stop) break;
      store_tile_y(L, p.M, tl, ys, e);
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");  // ys is free for the next tile
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S->abort) set_status(p.status, IFQ_DEV_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {row_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_tiled_map(m, dt, 2, base, dims, strides, box, sw);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_tiled_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                      const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int kCap>
cudaError_t launch_cap(const ifq_layer* Ls, int count, int T, int64_t M, uint64_t wait_ns, uint32_t* dev_status,
                       cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel<kCap>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  GemmParams<kCap> p;
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.M = M;
  p.wait_ns = wait_ns;
  p.status = dev_status;
  // heaviest layers first: K steps per tile times (stage, branch) passes
  int order[IFQ_MAX_GROUP];
  for (int i = 0; i < count; ++i) order[i] = i;
  for (int i = 1; i < count; ++i)
    for (int j = i; j > 0; --j) {
      const ifq_layer &a = Ls[order[j - 1]], &b = Ls[order[j]];
      const int64_t wa = a.K * (a.codes_w ? 2 : 1), wb = b.K * (b.codes_w ? 2 : 1);
      if (wa >= wb) break;
      const int t = order[j - 1];
      order[j - 1] = order[j];
      order[j] = t;
    }
  const int64_t tiles_m = (M + BM - 1) / BM;
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    const ifq_layer& L = Ls[order[i]];
    GemmLayer& g = p.L[i];
    g.nbranch = L.codes_w ? 2 : 1;
    g.N = L.N;
    g.K = L.K;
    g.scales[0] = L.scales_u;
    g.scales[1] = L.scales_w;
    g.y[0] = L.y_re;
    g.y[1] = L.y_im;
    g.rot[0] = L.rot_re;
    g.rot[1] = L.rot_im;
    g.tiles_n = (int32_t)((L.N + BN - 1) / BN);
    g.tile_begin = p.tile_begin[i] = tiles;
    tiles += (int64_t)g.tiles_n * tiles_m;
    bool ok = make_map_2d(&g.tmap_x[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.x_re, (uint64_t)L.K, (uint64_t)M,
                          (uint64_t)L.K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map_2d(&g.tmap_x[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.x_im, (uint64_t)L.K, (uint64_t)M,
                          (uint64_t)L.K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    for (int b = 0; b < g.nbranch && ok; ++b)
      ok = make_map_2d(&g.tmap_codes[b], CU_TENSOR_MAP_DATA_TYPE_UINT8, b == 0 ? L.codes_u : L.codes_w,
                       (uint64_t)L.K / 4, (uint64_t)T * L.N, (uint64_t)L.K / 4, BK / 4, BN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
  }
  p.tiles = tiles;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = tiles < sms ? tiles : sms;  // one persistent CTA per SM
  gemm_kernel<kCap><<<(unsigned)grid, kThreads, kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const ifq_layer* Ls, int count, int T, int64_t M, uint64_t wait_ns, uint32_t* dev_status,
                        cudaStream_t s) {
  return count <= 8 ? launch_cap<8>(Ls, count, T, M, wait_ns, dev_status, s)
                    : launch_cap<IFQ_MAX_GROUP>(Ls, count, T, M, wait_ns, dev_status, s);
}

}  // namespace ifq
