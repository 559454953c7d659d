// Decode product y = sum_t (U_hat_t x + W_hat_t conj(x)) for 1..4 tokens on the 5th-generation tensor
// cores with 4-bit block-scaled operands (tcgen05 kind::mxf4) ("Fairy2i write-up" §2.1, §4.2;
// "iFairy article" §二.2 -- the product rebuilt from signed additions).
//
// Each code contributes Re b = Br and Im b = Bi in {-1, 0, +1} (exactly one is non-zero).  Both are
// e2m1 values, so per (stage, branch) code matrix and 64-output block one MMA step computes
//     D[(class, output)][(token, plane, digit)] += sum over 64 positions of B_class * digit
// with A = [Br; Bi] (M = 128 rows, expanded from the 2-bit codes in shared memory, 4 bits per code and
// class) and B = the activations split into eight signed base-8 digits in {-4..3} (also e2m1 values)
// whose UE8M0 block scale 2^(3j - E) restores digit j's weight for each 32-position block.  The
// tensor core multiplies exactly and accumulates in float32; the epilogue adds the eight digit
// columns of each (token, plane), pairs the Br and Bi rows of an output and applies the scales:
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
//
// Activation digits: per (token, plane, 32-position block) x is scaled by 2^E so that the block's
// largest |x| lies in [2^21, 2^22), rounded to an integer v and written as v = sum_j d_j 8^j.  The
// rounding error is at most 2^-22 of the block's largest |x| per position, so for any input the
// error of a product is below 2^-22 * 32 * sum |x| -- far inside the 1e-5 acceptance bound.
//
// Work: units of (layer, K segment, 64-output block, (stage, branch) matrix), split evenly over one
// persistent CTA per SM in that order, so consecutive units of a CTA share the segment's digits and
// the units of one output block follow each other.  Each unit writes its contribution to its own
// workspace slot; after a run of consecutive units of one output block a CTA counts the run on the
// block's ticket, and the CTA that completes a block adds its slots in unit order and writes y.  An
// output therefore depends only on its own row's codes and the activations -- not on how rows or
// units are split across CTAs (or across GPUs of a row-split) -- and results are bit-reproducible.
//
// Codes reach shared memory by one 2-D tensor copy per code stage (64 rows x 128 B, 128-byte swizzle,
// so that the expanders' 16-byte reads of 32 rows are free of bank conflicts), with many stages in
// flight.  (Measured on a 70B-shaped matrix with no compute: tensor copies of any box shape stream
// near 4.5 TB/s with 96 KB in flight per SM; one bulk copy per row piece only 1.2 TB/s.)
//
// Warp roles (14 warps):
//   0-7  expanders: code stage (64 rows x 128 B) -> A tiles in shared memory, one MMA step of 32 rows
//        per warp and A stage; at a segment change warps 0-3 also write the digits' scale factors
//        into TMEM (lane quarter = warp)
//   8-11 epilogue: TMEM accumulator -> slot; last unit of a block -> y
//   12   producer: code stages (tensor copies) and the segment's digit tiles and factor words (bulk
//        copies)
//   13   TMEM allocation and the MMA issuer (the whole warp runs the loop; one elected lane issues,
//        four MMAs of an A stage at a time)
// TMEM: two accumulators of N = 16 NB columns, the A factors (4 columns), two segment buffers of B
// factors (a 4-column slot per MMA step).  Every mbarrier wait is bounded: a lost wait sets
// IFQ_DEV_TIMEOUT, the CTA drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int kStepK = 64;                        // positions per MMA step (K of one mxf4 MMA)
constexpr int kASteps = 4;                        // MMA steps per A stage
constexpr int kCSteps = 8;                        // MMA steps per code stage: 512 positions, 128 B per row
constexpr int kRowsU = 64;                        // outputs per unit
constexpr int kMaxAStages = 6;
constexpr uint32_t kCRowBytes = 128;              // code bytes per row and code stage
constexpr uint32_t kStageC = kRowsU * kCRowBytes;  // 8 KB
constexpr uint32_t kStepA = 2 * kRowsU * 32;      // A of one step: 128 rows x 32 B
constexpr uint32_t kStageA = kASteps * kStepA;    // 16 KB
constexpr int kDig = 8;                           // base-8 digits per activation
constexpr int kExpWarps = 8, kEpiWarps = 4;
constexpr int kProducerWarp = 12, kMmaWarp = 13;
constexpr int kThreads = 448;
constexpr int kPrepThreads = 256;
constexpr uint32_t kLBO = 128, kSBO = 256;        // core matrices: K-adjacent 128 B apart, 8-row groups 256 B apart

template <int NB>
struct Fp4Cfg {
  static constexpr int N = 16 * NB;                       // MMA N: (token, plane, digit)
  static constexpr int G = (N + 31) / 32;                 // factor word columns per step
  static constexpr int kSegK = NB <= 2 ? 2048 : 1024;     // positions per unit
  static constexpr int kSegSteps = kSegK / kStepK;
  static constexpr uint32_t kStepX = N * 32;              // B tile per step
  static constexpr uint32_t kXBuf = kSegSteps * kStepX;
  static constexpr uint32_t kSfBuf = kSegSteps * N * 4;   // factor words [step][row]
  // The factor operands of an MMA start on a 4-column boundary: each step's B factors take a 4-column
  // slot (G <= 2 columns used), the A factors 4 columns.
  static constexpr uint32_t kSfStride = 4;
  static_assert(G <= (int)kSfStride, "factor slot");
  static constexpr uint32_t kSfaCol = 2 * N;              // accumulators at columns 0 and N
  static constexpr uint32_t kSfbCol = kSfaCol + 4;        // 2 buffers x kSegSteps slots
  static constexpr uint32_t kCols = kSfbCol + 2 * kSegSteps * kSfStride;
  static constexpr uint32_t kTmemCols = kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(kCols <= 512, "TMEM budget");
  // A and B e2m1 (mxf4 format 1), K-major, N / 8, UE8M0 factors, M = 128, factor ids 0
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | (8u << 24);
  static constexpr uint32_t kOffX = 0;
  static constexpr uint32_t kOffSf = 2 * kXBuf;
  static constexpr int kCodeStages = NB == 1 ? 10 : 8;
  static constexpr int kAStages = NB == 1 ? 6 : 5;
  static constexpr uint32_t kOffC = (kOffSf + 2 * kSfBuf + 1023) & ~1023u;
  static constexpr uint32_t kOffA = (kOffC + kCodeStages * kStageC + 1023) & ~1023u;
  static constexpr uint32_t kOffBar = kOffA + kAStages * kStageA;
  static constexpr uint32_t kSmem = kOffBar + 512 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

struct __align__(64) Fp4Layer {
  CUtensorMap tmap[2];      // codes of U, W: u8 [T*N][K/4], box {128 B, 64 rows}, 128-byte swizzle
  const float* scales[2];
  const uint16_t* x[2];     // bf16 [B][K]
  float* y[2];
  const float* rot[2];      // optional [B][N] rotation, or null
  const uint8_t* dig;       // workspace: digit tiles [K/64 steps][N rows x 32 B]
  uint8_t* sfw;             // workspace: factor words [K/64 steps][N] (bytes 0, 1: the step's two blocks)
  unsigned int* tickets;    // workspace: one per 64-output block
  int64_t N, K;
  int64_t unit_begin;
  int nbranch, P, nblk, nseg, nsteps;
  int pad;
};

template <int kCap>
struct __align__(64) Fp4Params {
  int64_t unit_begin[kCap];  // copy of the layers' first units, for the unit search
  Fp4Layer L[kCap];
  float* slots;             // workspace: [unit][NB tokens][64 outputs] float2
  int64_t units;
  int64_t prep_warps;
  int64_t tickets;          // total tickets (zeroed by the prep kernel)
  unsigned int* ticket_base;
  uint32_t* status;
  int count, T, B, pad;
};

constexpr int kMaxCodeStages = 16;

struct Smem {
  uint64_t x_full[2], x_empty[2];
  uint64_t c_full[kMaxCodeStages], c_empty[kMaxCodeStages];
  uint64_t a_full[kMaxAStages], a_empty[kMaxAStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int last_flag;
};

struct Unit {
  int l, seg, blk, p;
};

template <int kCap>
__device__ __forceinline__ Unit decode_unit(const Fp4Params<kCap>& p, int64_t u) {
  int l = 0;
  while (l + 1 < p.count && u >= p.unit_begin[l + 1]) ++l;
  const Fp4Layer& L = p.L[l];
  int64_t v = u - p.unit_begin[l];
  Unit r;
  r.l = l;
  r.p = (int)(v % L.P);
  v /= L.P;
  r.blk = (int)(v % L.nblk);
  r.seg = (int)(v / L.nblk);
  return r;
}

__device__ __forceinline__ uint32_t core_off(int row, int kbyte) {  // byte of (row, kbyte) in a K-major tile
  return (uint32_t)((row >> 3) * kSBO + (kbyte >> 4) * kLBO + (row & 7) * 16 + (kbyte & 15));
}

__device__ __forceinline__ uint64_t desc_noswz(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (uint64_t)(kLBO >> 4) << 16 | (uint64_t)(kSBO >> 4) << 32 |
         (uint64_t)1u << 46;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Up to four MMA steps of one A stage from one elected lane of a converged warp: step c reads A at
// ad + c * 4 KB, B at bd + c * kStepX (both as descriptor start-address increments) and its B factors
// at sf + 4 c; the first accumulates only if `acc`, the others always.
template <uint32_t kStepX>
__device__ __forceinline__ void umma_mxf4_group_t(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                                  uint32_t sf, uint32_t acc, int n) {
  constexpr uint64_t kA = kStepA >> 4, kB = kStepX >> 4;
  if (n == 4) {
    asm volatile(
        "{\n\t.reg .pred e, p, t;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %7, %8, %3, [%5], [%9], t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %10, %11, %3, [%5], [%12], t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %13, %14, %3, [%5], [%15], t;\n\t"
        "}" ::"r"(d), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sf), "l"(ad + kA), "l"(bd + kB),
        "r"(sf + 4u), "l"(ad + 2 * kA), "l"(bd + 2 * kB), "r"(sf + 8u), "l"(ad + 3 * kA), "l"(bd + 3 * kB),
        "r"(sf + 12u)
        : "memory");
  } else {
    for (int c = 0; c < n; ++c) {
      asm volatile(
          "{\n\t.reg .pred e, p;\n\t"
          "elect.sync _|e, 0xffffffff;\n\t"
          "setp.ne.b32 p, %4, 0;\n\t"
          "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
          "}" ::"r"(d), "l"(ad + c * kA), "l"(bd + c * kB), "r"(idesc), "r"(c == 0 ? acc : 1u), "r"(sfa),
          "r"(sf + 4u * c)
          : "memory");
    }
  }
}

__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t a) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(a) : "memory");
}

// e2m1 encoding of a digit in {-4..3}: sign bit 3, magnitudes 0, 1, 2, 3, 4 -> 0, 2, 4, 5, 6
__device__ __forceinline__ uint32_t e2m1_of(int d) {
  const int a = d < 0 ? -d : d;
  const uint32_t mag = a == 0 ? 0u : a == 1 ? 2u : a == 2 ? 4u : a == 3 ? 5u : 6u;
  return d < 0 ? (8u | mag) : mag;
}

__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// Element order inside one 64-position step, shared by the code expansion and the digit tiles:
// element 16 g + 8 h + i is position 16 g + 2 i + h (even positions of each 16-position group
// first), so that a 32-bit code word expands into two words of 8 nibbles by masks and shifts.
__device__ __forceinline__ int element_of(int pos_in_step) {
  const int g = pos_in_step >> 4, i = (pos_in_step & 15) >> 1, h = pos_in_step & 1;
  return 16 * g + 8 * h + i;
}

// ---------------------------------------------------------------- prep: activation digits
// One warp per (layer, 32-position block, token slot, plane); lane = position in the block.
template <int NB, int kCap>
__global__ void __launch_bounds__(kPrepThreads) fp4_prep_kernel(const __grid_constant__ Fp4Params<kCap> p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int N = Fp4Cfg<NB>::N;
  const int64_t gt = (int64_t)blockIdx.x * kPrepThreads + threadIdx.x;
  if (gt < p.tickets) p.ticket_base[gt] = 0u;
  int64_t w = gt >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= p.prep_warps) return;
  int li = 0;
  for (; li < p.count; ++li) {
    const int64_t nw = (p.L[li].K / 32) * NB * 2;
    if (w < nw) break;
    w -= nw;
  }
  const Fp4Layer& L = p.L[li];
  const int pl = (int)(w & 1), tok = (int)((w >> 1) % NB);
  const int64_t blk = (w >> 1) / NB;  // 32-position block
  const int64_t pos = blk * 32 + lane;
  const float x_in = tok < p.B ? bf16f(L.x[pl][(int64_t)tok * L.K + pos]) : 0.0f;
  const bool bad = !isfinite(x_in);
  const bool block_bad = __any_sync(0xffffffffu, bad);
  const float x = bad ? 0.0f : x_in;
  float m = fabsf(x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int E = 0;
  if (m > 0.0f) E = min(21 - ilogbf(m), 127);  // m 2^E in [2^21, 2^22); factors 127 + 3j - E stay in 0..254
  int v = __float2int_rn(ldexpf(x, E));
  uint32_t nib[kDig];
#pragma unroll
  for (int j = 0; j < kDig; ++j) {
    const int d = ((v + 4) & 7) - 4;
    nib[j] = e2m1_of(d);
    v = (v - d) >> 3;
  }
  const int e = element_of((int)(pos & 63));
  uint8_t* tile = const_cast<uint8_t*>(L.dig) + (pos >> 6) * Fp4Cfg<NB>::kStepX;
#pragma unroll
  for (int j = 0; j < kDig; ++j) {
    const uint32_t other = __shfl_xor_sync(0xffffffffu, nib[j], 2);  // element e ^ 1 is position pos ^ 2
    if ((e & 1) == 0) tile[core_off((tok * 2 + pl) * kDig + j, e >> 1)] = (uint8_t)(nib[j] | other << 4);
  }
  if (lane < kDig) {  // factor of digit row j for this block: 2^(3j - E); a non-finite x gives the NaN factor
    const int row = (tok * 2 + pl) * kDig + lane;
    uint8_t* word = L.sfw + ((pos >> 6) * N + row) * 4;
    word[blk & 1] = block_bad ? (uint8_t)0xFF : (uint8_t)(127 + 3 * lane - E);
    if ((blk & 1) == 0) {  // bytes 2 and 3 are not read (factor id 0); keep them defined
      word[2] = 0x7F;
      word[3] = 0x7F;
    }
  }
  if (block_bad && lane == 0) set_status(p.status, IFQ_DEV_NONFINITE);
}

// ---------------------------------------------------------------- main kernel
template <int NB, int kCap>
__global__ void __launch_bounds__(kThreads, 1) fp4_gemv_kernel(const __grid_constant__ Fp4Params<kCap> p) {
  using C = Fp4Cfg<NB>;
  constexpr int N = C::N;
  constexpr int CS = C::kCodeStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem* S = reinterpret_cast<Smem*>(smem + C::kOffBar);
  volatile int* abort = &S->abort;
  auto xbuf = [&](int b) { return smem + C::kOffX + b * C::kXBuf; };
  auto sfbuf = [&](int b) { return reinterpret_cast<uint32_t*>(smem + C::kOffSf + b * C::kSfBuf); };
  auto cstage = [&](int s) { return smem + C::kOffC + s * kStageC; };
  auto astage = [&](int s) { return smem + C::kOffA + s * kStageA; };

  const int64_t ub = (int64_t)blockIdx.x * p.units / gridDim.x;
  const int64_t ue = (int64_t)(blockIdx.x + 1) * p.units / gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S->x_full[b], 1);
      mbar_init(&S->x_empty[b], 1);
      mbar_init(&S->acc_full[b], 1);
      mbar_init(&S->acc_empty[b], kEpiWarps);
    }
    for (int s = 0; s < CS; ++s) {
      mbar_init(&S->c_full[s], 1);
      mbar_init(&S->c_empty[s], kExpWarps);
    }
    for (int s = 0; s < C::kAStages; ++s) {
      mbar_init(&S->a_full[s], kExpWarps);
      mbar_init(&S->a_empty[s], 1);
    }
    mbar_init(&S->drain, 1);
    S->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer (whole warp)
    int issued[kMaxCodeStages];
    for (int s = 0; s < kMaxCodeStages; ++s) issued[s] = 0;
    int x_issued[2] = {0, 0};
    bool waited = false, ok = true;
    int64_t prev_key = -1;
    int xseq = -1, cseq = 0;
    for (int64_t u = ub; u < ue && ok; ++u) {
      const Unit un = decode_unit(p, u);
      const Fp4Layer& L = p.L[un.l];
      const int64_t key = ((int64_t)un.l << 32) | un.seg;
      const int steps = min(C::kSegSteps, L.nsteps - un.seg * C::kSegSteps);
      const int ncs = (steps + kCSteps - 1) / kCSteps;
      bool need_x = key != prev_key;
      if (need_x) {
        ++xseq;
        prev_key = key;
      }
      const int xb = xseq & 1;
      const int t = un.p / L.nbranch, br = un.p % L.nbranch;
      const int64_t n0 = (int64_t)un.blk * kRowsU;
      const int32_t row = (int32_t)((int64_t)t * L.N + n0);
      const int32_t col0 = un.seg * (C::kSegK / 4);
      for (int cs = 0; cs < ncs; ++cs) {
        const int s = cseq % CS;
        int w_ok = 1;
        if (lane == 0) {
          w_ok = mbar_wait_bounded(&S->c_empty[s], ((uint32_t)(cseq / CS) & 1u) ^ 1u, abort);
          if (w_ok) {
            mbar_arrive_expect_tx(&S->c_full[s], kStageC);  // the whole box, zero-filled past the tensor
            tma_load_2d(cstage(s), &L.tmap[br], col0 + cs * (int)kCRowBytes, row, &S->c_full[s]);
          }
        }
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        ++issued[s];
        ++cseq;
        // the segment's digits follow the first code stages (they come from the prep kernel)
        if (need_x && (cs + 1 == ncs || cs + 1 == CS)) {
          need_x = false;
          if (lane == 0) {
            w_ok = mbar_wait_bounded(&S->x_empty[xb], ((uint32_t)(xseq >> 1) & 1u) ^ 1u, abort);
            if (w_ok) {
              if (!waited) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
              }
              const uint32_t xbytes = (uint32_t)steps * C::kStepX, sbytes = (uint32_t)steps * N * 4;
              mbar_arrive_expect_tx(&S->x_full[xb], xbytes + sbytes);
              bulk_g2s(xbuf(xb), L.dig + (int64_t)un.seg * C::kSegSteps * C::kStepX, xbytes, &S->x_full[xb]);
              bulk_g2s(sfbuf(xb), L.sfw + (int64_t)un.seg * C::kSegSteps * N * 4, sbytes, &S->x_full[xb]);
              ++x_issued[xb];
            }
          }
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
            ok = false;
            break;
          }
        }
      }
    }
    if (lane == 0 && *abort) {
      // let every issued copy land before the CTA's shared memory is released
      volatile int never = 0;
      for (int b = 0; b < 2; ++b)
        if (x_issued[b] > 0) mbar_wait_bounded(&S->x_full[b], (uint32_t)(x_issued[b] - 1) & 1u, &never);
      for (int s = 0; s < CS; ++s)
        if (issued[s] > 0) mbar_wait_bounded(&S->c_full[s], (uint32_t)(issued[s] - 1) & 1u, &never);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
    int64_t prev_key = -1;
    int xseq = -1, aseq = 0, useq = 0;
    bool ok = true;
    const uint64_t adesc0 = desc_noswz(smem_u32(astage(0)));
    for (int64_t u = ub; u < ue && ok; ++u) {
      const Unit un = decode_unit(p, u);
      const Fp4Layer& L = p.L[un.l];
      const int64_t key = ((int64_t)un.l << 32) | un.seg;
      if (key != prev_key) {
        ++xseq;
        prev_key = key;
      }
      const int xb = xseq & 1;
      const int steps = min(C::kSegSteps, L.nsteps - un.seg * C::kSegSteps);
      const int ab = useq & 1;
      int w_ok = 1;
      if (lane == 0)
        w_ok = mbar_wait_bounded(&S->x_full[xb], (uint32_t)(xseq >> 1) & 1u, abort) &&
               mbar_wait_bounded(&S->acc_empty[ab], ((uint32_t)(useq >> 1) & 1u) ^ 1u, abort);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(ab * N);
      const uint64_t bdesc0 = desc_noswz(smem_u32(xbuf(xb)));
      const uint32_t sfb0 = tmem + C::kSfbCol + (uint32_t)(xb * C::kSegSteps) * C::kSfStride;
      for (int st0 = 0; st0 < steps; st0 += kASteps) {
        const int sa = aseq % C::kAStages;
        if (lane == 0) w_ok = mbar_wait_bounded(&S->a_full[sa], (uint32_t)(aseq / C::kAStages) & 1u, abort);
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // descriptors advance by adding the byte offset / 16 to the start-address field
        const uint64_t ad = adesc0 + (uint64_t)((uint32_t)sa * (kStageA >> 4));
        const uint64_t bd = bdesc0 + (uint64_t)((uint32_t)st0 * (C::kStepX >> 4));
        const uint32_t sf = sfb0 + (uint32_t)st0 * C::kSfStride;
        const int n = min(kASteps, steps - st0);
        umma_mxf4_group_t<C::kStepX>(d, ad, bd, C::kIdesc, tmem + C::kSfaCol, sf, st0 > 0 ? 1u : 0u, n);
        umma_commit_elect(&S->a_empty[sa]);
        ++aseq;
      }
      if (!ok) break;
      umma_commit_elect(&S->acc_full[ab]);
      ++useq;
      // the last unit of this segment: its digits and factors may be replaced once these MMAs end
      bool seg_end = u + 1 >= ue;
      if (!seg_end) {
        const Unit nx = decode_unit(p, u + 1);
        seg_end = nx.l != un.l || nx.seg != un.seg;
      }
      if (seg_end) umma_commit_elect(&S->x_empty[xb]);
    }
    if (lane == 0 && *abort) {
      volatile int never = 0;
      umma_commit(&S->drain);
      mbar_wait_bounded(&S->drain, 0u, &never);
    }
  } else if (warp < kExpWarps) {
    // ------------------------------------------------------------ expanders
    const bool sf_warp = warp < 4;                   // warps 0-3 own the four TMEM lane quarters
    const uint32_t tq = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    if (sf_warp) tmem_st_x4(tq + C::kSfaCol, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);  // A factors: 1
    const int o = 32 * (warp & 1) + lane;            // this lane's output row in the unit
    const int c = warp >> 1;                         // its MMA step of each A stage
    const int rbr = 32 * (o >> 4) + (o & 15), rbi = rbr + 16;  // its A rows (Br, Bi)
    int64_t prev_key = -1;
    int xseq = -1, cseq = 0, aseq = 0;
    bool ok = true;
    for (int64_t u = ub; u < ue && ok; ++u) {
      const Unit un = decode_unit(p, u);
      const Fp4Layer& L = p.L[un.l];
      const int64_t key = ((int64_t)un.l << 32) | un.seg;
      const int steps = min(C::kSegSteps, L.nsteps - un.seg * C::kSegSteps);
      const int ncs = (steps + kCSteps - 1) / kCSteps;
      if (key != prev_key) {
        ++xseq;
        prev_key = key;
        const int xb = xseq & 1;
        // the segment's B factors into the four lane quarters (the MMA reads every quarter)
        int w_ok = 1;
        if (lane == 0 && sf_warp)
          w_ok = mbar_wait_bounded(&S->x_full[xb], (uint32_t)(xseq >> 1) & 1u, abort) &&
                 mbar_wait_bounded(&S->x_empty[xb], ((uint32_t)(xseq >> 1) & 1u) ^ 1u, abort);
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        if (sf_warp) {
          tc_fence_after();
          const uint32_t* sf = sfbuf(xb);
          const uint32_t col = tq + C::kSfbCol + (uint32_t)(xb * C::kSegSteps) * C::kSfStride;
          for (int kb = 0; kb < steps; ++kb)
#pragma unroll
            for (int g = 0; g < C::G; ++g) {
              const int row = 32 * g + lane;
              tmem_st_x1(col + (uint32_t)kb * C::kSfStride + g, row < N ? sf[kb * N + row] : 0x7F7F7F7Fu);
            }
          tmem_wait_st();
        }
      }
      for (int cs = 0; cs < ncs && ok; ++cs) {
        const int s = cseq % CS;
        const int steps_cs = min(kCSteps, steps - cs * kCSteps);
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait_bounded(&S->c_full[s], (uint32_t)(cseq / CS) & 1u, abort);
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
          ok = false;
          break;
        }
        const uint8_t* rowp = cstage(s) + o * kCRowBytes;
        for (int a0 = 0; a0 < steps_cs; a0 += kASteps) {
          const int sa = aseq % C::kAStages;
          if (lane == 0) w_ok = mbar_wait_bounded(&S->a_empty[sa], ((uint32_t)(aseq / C::kAStages) & 1u) ^ 1u, abort);
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
            ok = false;
            break;
          }
          uint8_t* a_base = astage(sa);
          if (a0 + c < steps_cs) {
            const uint4 cw = *reinterpret_cast<const uint4*>(rowp + 16 * ((a0 + c) ^ (o & 7)));  // 128 B swizzle
            const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
            uint32_t bi[8], br[8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              // nibble i of the even word: code 16g + 2i (axis bit 4i, sign 4i + 1); of the odd word:
              // code 16g + 2i + 1 (axis 4i + 2, sign 4i + 3).  e2m1 +-1 is sign | 0b010, +-0 is sign | 0.
              const uint32_t w = wv[g];
              const uint32_t ev = ((w << 2) & 0x88888888u) | ((w << 1) & 0x22222222u);
              const uint32_t od = (w & 0x88888888u) | ((w >> 1) & 0x22222222u);
              bi[2 * g] = ev;
              bi[2 * g + 1] = od;
              br[2 * g] = ev ^ 0x22222222u;
              br[2 * g + 1] = od ^ 0x22222222u;
            }
            uint8_t* at = a_base + c * kStepA;
            *reinterpret_cast<uint4*>(at + core_off(rbr, 0)) = make_uint4(br[0], br[1], br[2], br[3]);
            *reinterpret_cast<uint4*>(at + core_off(rbr, 16)) = make_uint4(br[4], br[5], br[6], br[7]);
            *reinterpret_cast<uint4*>(at + core_off(rbi, 0)) = make_uint4(bi[0], bi[1], bi[2], bi[3]);
            *reinterpret_cast<uint4*>(at + core_off(rbi, 16)) = make_uint4(bi[4], bi[5], bi[6], bi[7]);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S->a_full[sa]);
          ++aseq;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S->c_empty[s]);
        ++cseq;
      }
    }
  } else if (warp < kExpWarps + kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");  // tickets are zeroed by the prep kernel
    const int q = warp & 3;
    const bool imag = lane >= 16;                   // this lane's class: Bi rows
    const int o = 16 * q + (lane & 15);             // its output row in the unit
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const int et = threadIdx.x - kExpWarps * 32;    // 0..127
    int64_t run_first = -1;
    int useq = 0;
    bool ok = true;
    for (int64_t u = ub; u < ue && ok; ++u) {
      const Unit un = decode_unit(p, u);
      const Fp4Layer& L = p.L[un.l];
      const int ab = useq & 1;
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait_bounded(&S->acc_full[ab], (uint32_t)(useq >> 1) & 1u, abort);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float pre[NB], pim[NB];
      {
        uint32_t d[N];
        if constexpr (N == 16) {
          uint32_t (&r)[16] = *reinterpret_cast<uint32_t(*)[16]>(d);
          tmem_ld_32x32b_x16(trow + (uint32_t)(ab * N), r);
        } else {
#pragma unroll
          for (int h = 0; h < N / 32; ++h) {
            uint32_t (&r)[32] = *reinterpret_cast<uint32_t(*)[32]>(d + 32 * h);
            tmem_ld_32x32b_x32(trow + (uint32_t)(ab * N + 32 * h), r);
          }
        }
        tmem_wait_ld();
#pragma unroll
        for (int tk = 0; tk < NB; ++tk) {
          float a = 0.0f, b = 0.0f;
#pragma unroll
          for (int j = 0; j < kDig; ++j) {
            a += __uint_as_float(d[(2 * tk) * kDig + j]);
            b += __uint_as_float(d[(2 * tk + 1) * kDig + j]);
          }
          pre[tk] = a;
          pim[tk] = b;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->acc_empty[ab]);
      ++useq;
      // pair the Br row (lanes 0..15) with the Bi row (lanes 16..31) of each output: the unit's slot
      const int t = un.p / L.nbranch, brn = un.p % L.nbranch;
      const float s_re = __ldg(L.scales[brn] + 2 * t), s_im = __ldg(L.scales[brn] + 2 * t + 1);
      float2* slot = reinterpret_cast<float2*>(p.slots) + (size_t)u * NB * kRowsU;
#pragma unroll
      for (int tk = 0; tk < NB; ++tk) {
        const float ore = __shfl_xor_sync(0xffffffffu, pre[tk], 16);
        const float oim = __shfl_xor_sync(0xffffffffu, pim[tk], 16);
        const float P_rr = imag ? ore : pre[tk], P_ri = imag ? oim : pim[tk];
        const float P_ir = imag ? pre[tk] : ore, P_ii = imag ? pim[tk] : oim;
        const bool mine = NB == 1 ? !imag : (imag ? tk >= (NB + 1) / 2 : tk < (NB + 1) / 2);
        if (mine) {
          float cre, cim;
          if (brn == 0) {
            cre = s_re * P_rr - s_im * P_ii;
            cim = s_re * P_ri + s_im * P_ir;
          } else {
            cre = s_re * P_rr + s_im * P_ii;
            cim = s_im * P_ir - s_re * P_ri;
          }
          slot[tk * kRowsU + o] = make_float2(cre, cim);
        }
      }
      if (run_first < 0) run_first = u;
      bool run_end = u + 1 >= ue;
      if (!run_end) {
        const Unit nx = decode_unit(p, u + 1);
        run_end = nx.l != un.l || nx.seg != un.seg || nx.blk != un.blk;
      }
      if (!run_end) continue;
      // the run's units are counted at once
      const unsigned run_len = (unsigned)(u - run_first + 1);
      run_first = -1;
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      if (et == 0) {
        const unsigned need = (unsigned)(L.nseg * L.P);
        const unsigned old = atomicAdd(L.tickets + un.blk, run_len);
        S->last_flag = old + run_len == need;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      if (S->last_flag) {
        __threadfence();
        const int64_t n0 = (int64_t)un.blk * kRowsU;
        for (int idx = et; idx < p.B * kRowsU; idx += kEpiWarps * 32) {
          const int tk = idx / kRowsU, oo = idx % kRowsU;
          const int64_t n = n0 + oo;
          if (n >= L.N) continue;
          float yre = 0.0f, yim = 0.0f;
          for (int sg = 0; sg < L.nseg; ++sg)
            for (int pp = 0; pp < L.P; ++pp) {
              const int64_t uu = L.unit_begin + ((int64_t)sg * L.nblk + un.blk) * L.P + pp;
              const float2 v = __ldcg(reinterpret_cast<const float2*>(p.slots) + ((size_t)uu * NB + tk) * kRowsU + oo);
              yre += v.x;
              yim += v.y;
            }
          const int64_t off = (int64_t)tk * L.N + n;
          if (L.rot[0]) {
            const float cr = __ldg(L.rot[0] + off), ci = __ldg(L.rot[1] + off);
            const float r = cr * yre - ci * yim, im = cr * yim + ci * yre;
            yre = r;
            yim = im;
          }
          L.y[0][off] = yre;
          L.y[1][off] = yim;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S->abort) set_status(p.status, IFQ_DEV_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
struct Fp4Layout {
  size_t dig, sfw, tick, slots, total;
};

int fp4_slots_nb(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : 4; }

template <int NB>
size_t layout(const ifq_layer* Ls, int count, int T, size_t* dig, size_t* sfw, size_t* tick, size_t* slots) {
  using C = Fp4Cfg<NB>;
  size_t off = 0;
  int64_t units = 0, tickets = 0;
  for (int i = 0; i < count; ++i) {
    const int64_t steps = Ls[i].K / kStepK;
    dig[i] = off;
    off += (size_t)steps * C::kStepX;
    sfw[i] = off;
    off += (size_t)steps * C::N * 4;
    off = (off + 255) & ~(size_t)255;
    const int64_t nblk = (Ls[i].N + kRowsU - 1) / kRowsU;
    const int64_t nseg = (Ls[i].K + C::kSegK - 1) / C::kSegK;
    units += nblk * nseg * T * (Ls[i].codes_w ? 2 : 1);
    tickets += nblk;
  }
  *tick = off;
  off += (size_t)tickets * 4;
  off = (off + 255) & ~(size_t)255;
  *slots = off;
  off += (size_t)units * NB * kRowsU * 8;
  return off;
}

// The launch parameters of a call (tensor maps, workspace layout, unit counts) and its grid sizes.
template <int kCap, int NB>
cudaError_t build_params(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status,
                         Fp4Params<kCap>& p, int64_t& prep_blocks_out, int64_t& ctas_out) {
  using C = Fp4Cfg<NB>;
  size_t dig[IFQ_MAX_GROUP], sfw[IFQ_MAX_GROUP], tick = 0, slots = 0;
  layout<NB>(Ls, count, T, dig, sfw, &tick, &slots);
  char* base = static_cast<char*>(ws);
  memset(&p, 0, sizeof(p));
  p.count = count;
  p.T = T;
  p.B = B;
  p.status = dev_status;
  p.slots = reinterpret_cast<float*>(base + slots);
  p.ticket_base = reinterpret_cast<unsigned int*>(base + tick);
  int64_t units = 0, tickets = 0, prep_warps = 0;
  for (int i = 0; i < count; ++i) {
    Fp4Layer& a = p.L[i];
    const ifq_layer& l = Ls[i];
    a.nbranch = l.codes_w ? 2 : 1;
    a.P = T * a.nbranch;
    a.scales[0] = l.scales_u;
    a.scales[1] = l.scales_w;
    a.x[0] = l.x_re;
    a.x[1] = l.x_im;
    a.y[0] = l.y_re;
    a.y[1] = l.y_im;
    a.rot[0] = l.rot_re;
    a.rot[1] = l.rot_im;
    a.N = l.N;
    a.K = l.K;
    a.nsteps = (int)(l.K / kStepK);
    a.nblk = (int)((l.N + kRowsU - 1) / kRowsU);
    a.nseg = (int)((l.K + C::kSegK - 1) / C::kSegK);
    a.dig = reinterpret_cast<const uint8_t*>(base + dig[i]);
    a.sfw = reinterpret_cast<uint8_t*>(base + sfw[i]);
    a.tickets = p.ticket_base + tickets;
    a.unit_begin = p.unit_begin[i] = units;
    units += (int64_t)a.nblk * a.nseg * a.P;
    tickets += a.nblk;
    prep_warps += (l.K / 32) * NB * 2;
    for (int b = 0; b < a.nbranch; ++b) {
      const uint64_t dims[2] = {(uint64_t)l.K / 4, (uint64_t)T * (uint64_t)l.N};
      const uint64_t strides[1] = {(uint64_t)l.K / 4};
      const uint32_t box[2] = {kCRowBytes, (uint32_t)kRowsU};
      if (!encode_tiled_map(&a.tmap[b], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b == 0 ? l.codes_u : l.codes_w, dims,
                            strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    }
  }
  p.units = units;
  p.tickets = tickets;
  p.prep_warps = prep_warps;
  const int64_t prep_threads = std::max<int64_t>(prep_warps * 32, tickets);
  const int64_t prep_blocks = (prep_threads + kPrepThreads - 1) / kPrepThreads;
  if (prep_blocks > 0x7fffffffLL || units >= ((int64_t)1 << 40)) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  prep_blocks_out = prep_blocks;
  ctas_out = std::min<int64_t>(sms, units);
  return cudaSuccess;
}

// Launches the prep kernel and the product for parameters made by build_params.
template <int kCap, int NB>
cudaError_t launch_params(const Fp4Params<kCap>& p, int64_t prep_blocks, int64_t ctas, cudaStream_t s) {
  using C = Fp4Cfg<NB>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(fp4_gemv_kernel<NB, kCap>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)C::kSmem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  fp4_prep_kernel<NB, kCap><<<(unsigned)prep_blocks, kPrepThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fp4_gemv_kernel<NB, kCap>, p);
}


template <int kCap, int NB>
cudaError_t launch_cap(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, cudaStream_t s) {
  Fp4Params<kCap> p;
  int64_t prep_blocks = 0, ctas = 0;
  cudaError_t e = build_params<kCap, NB>(Ls, count, T, B, ws, dev_status, p, prep_blocks, ctas);
  if (e != cudaSuccess) return e;
  return launch_params<kCap, NB>(p, prep_blocks, ctas, s);
}

template <int NB>
cudaError_t launch_nb(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, cudaStream_t s) {
  return count <= 8 ? launch_cap<8, NB>(Ls, count, T, B, ws, dev_status, s)
                    : launch_cap<IFQ_MAX_GROUP, NB>(Ls, count, T, B, ws, dev_status, s);
}

}  // namespace

namespace {
// A prepared call: the parameter block of the widest layer capacity and its grid sizes.
struct alignas(64) Fp4Plan {
  int32_t nb, cap;
  int64_t prep_blocks, ctas;
  alignas(64) unsigned char params[sizeof(Fp4Params<IFQ_MAX_GROUP>)];
};

template <int NB>
cudaError_t plan_nb(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* st, Fp4Plan& pl) {
  pl.nb = NB;
  pl.cap = count <= 8 ? 8 : IFQ_MAX_GROUP;
  if (pl.cap == 8)
    return build_params<8, NB>(Ls, count, T, B, ws, st, *reinterpret_cast<Fp4Params<8>*>(pl.params), pl.prep_blocks,
                               pl.ctas);
  return build_params<IFQ_MAX_GROUP, NB>(Ls, count, T, B, ws, st,
                                         *reinterpret_cast<Fp4Params<IFQ_MAX_GROUP>*>(pl.params), pl.prep_blocks,
                                         pl.ctas);
}

template <int NB>
cudaError_t run_nb(const Fp4Plan& pl, cudaStream_t s) {
  if (pl.cap == 8)
    return launch_params<8, NB>(*reinterpret_cast<const Fp4Params<8>*>(pl.params), pl.prep_blocks, pl.ctas, s);
  return launch_params<IFQ_MAX_GROUP, NB>(*reinterpret_cast<const Fp4Params<IFQ_MAX_GROUP>*>(pl.params),
                                          pl.prep_blocks, pl.ctas, s);
}
}  // namespace

size_t gemv_fp4_plan_bytes() { return sizeof(Fp4Plan); }

cudaError_t plan_gemv_fp4(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status, void* dst) {
  Fp4Plan& pl = *static_cast<Fp4Plan*>(dst);
  switch (fp4_slots_nb(B)) {
    case 1: return plan_nb<1>(Ls, count, T, B, ws, dev_status, pl);
    case 2: return plan_nb<2>(Ls, count, T, B, ws, dev_status, pl);
    default: return plan_nb<4>(Ls, count, T, B, ws, dev_status, pl);
  }
}

cudaError_t run_gemv_fp4_plan(const void* src, cudaStream_t s) {
  const Fp4Plan& pl = *static_cast<const Fp4Plan*>(src);
  switch (pl.nb) {
    case 1: return run_nb<1>(pl, s);
    case 2: return run_nb<2>(pl, s);
    case 4: return run_nb<4>(pl, s);
    default: return cudaErrorInvalidValue;
  }
}

size_t gemv_fp4_workspace_bytes(const ifq_layer* Ls, int count, int T, int B) {
  size_t dig[IFQ_MAX_GROUP], sfw[IFQ_MAX_GROUP], tick, slots;
  switch (fp4_slots_nb(B)) {
    case 1: return layout<1>(Ls, count, T, dig, sfw, &tick, &slots);
    case 2: return layout<2>(Ls, count, T, dig, sfw, &tick, &slots);
    default: return layout<4>(Ls, count, T, dig, sfw, &tick, &slots);
  }
}

cudaError_t launch_gemv_fp4(const ifq_layer* Ls, int count, int T, int B, void* ws, uint32_t* dev_status,
                            cudaStream_t s) {
  switch (fp4_slots_nb(B)) {
    case 1: return launch_nb<1>(Ls, count, T, B, ws, dev_status, s);
    case 2: return launch_nb<2>(Ls, count, T, B, ws, dev_status, s);
    default: return launch_nb<4>(Ls, count, T, B, ws, dev_status, s);
  }
}

}  // namespace ifq
