// Prefill product on the 5th-generation tensor cores (tcgen05 / TMEM)
// ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2 -- the GEMM rebuilt
// from additions, subtractions and swaps).
//
// For each (stage t, branch) code matrix the per-class signed sums are one
// real GEMM with exact operands:
//     D_re = X_re [Br; Bi]^T,   D_im = X_im [Br; Bi]^T
// X_* are the bf16 activation planes [M][K]; Br, Bi in {-2, 0, +2} are the
// code's real / imaginary parts (times 2), expanded from the packed codes in
// shared memory.  Products are exact and accumulate in float32 in TMEM, so the
// +-1 and +-i classes keep separate accumulators (columns 0..63 and 64..127 of
// each D) and their different scales are applied in the epilogue:
//     U:  y_re += s_re P_rr - s_im P_ii,   y_im += s_re P_ri + s_im P_ir
//     W:  y_re += s_re P_rr + s_im P_ii,   y_im += s_im P_ir - s_re P_ri
//
// CTA tile: 128 tokens (TMEM lanes) x 64 outputs; K in blocks of 64.
// Warp roles (14 warps):
//   0      TMA producer: X_re, X_im tiles (128 B swizzle) and the 64 x 16-byte code tile
//   1      TMEM allocator and single-thread MMA issuer (M=128, N=128, K=16 per instruction)
//   2-5    expanders: code tile -> B tile [Br rows 0..63; Bi rows 64..127] in the
//          same 128 B-swizzled K-major layout the TMA uses for X
//   6-13   epilogue: tcgen05.ld of the finished (stage, branch) accumulator,
//          scale, accumulate y in registers; store y at the end
// Accumulators are double-buffered (2 x 256 of the 512 TMEM columns) so the
// epilogue of one (stage, branch) overlaps the main loop of the next.
// Every mbarrier wait is bounded; a lost wait sets IFQ_DEV_TIMEOUT, the CTA
// drains its outstanding copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace ifq {
namespace {

constexpr int BM = 128;      // tokens per tile
constexpr int BN = 64;       // outputs per tile
constexpr int BK = 64;       // K per stage (one 128-byte swizzle row of bf16)
constexpr int STAGES = 4;
constexpr int kThreads = 14 * 32;
constexpr uint32_t kTileX = BM * BK * 2;        // 16 KB per activation plane
constexpr uint32_t kTileB = 2 * BN * BK * 2;    // 16 KB: Br and Bi rows
constexpr uint32_t kTileC = BN * (BK / 4);      // 1 KB of codes
constexpr uint32_t kStageBytes = 2 * kTileX + kTileB + kTileC;  // 49 KB (multiple of 1 KB)
constexpr uint32_t kTmaBytes = 2 * kTileX + kTileC;
constexpr uint32_t kSmemBytes = STAGES * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = umma_idesc_bf16(BM, 2 * BN);

struct __align__(64) GemmArgs {
  CUtensorMap tmap_x[2];      // bf16 [M][K]: box {64, 128}, 128 B swizzle
  CUtensorMap tmap_codes[2];  // u8 [T*N][K/4]: box {16, 64}
  const float* scales[2];
  float* y[2];
  int64_t N, K, M;
  int T, nbranch;
  uint32_t* status;
};

struct Smem {
  uint64_t full_tma[STAGES];
  uint64_t full_b[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Source bits (from, from+1) of w moved to (to, to+1).
__device__ __forceinline__ uint32_t move_bits(uint32_t w, int from, int to) {
  return to >= from ? (w << (to - from)) : (w >> (from - to));
}

// Eight codes (j0..j0+7 of a 16-code word) -> 16 B of bf16 {Bi} and {Br} in K order.
__device__ __forceinline__ void expand8(uint32_t w, int j0, uint4& bi, uint4& br) {
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = j0 + 2 * q;
    const uint32_t lo = move_bits(w, 2 * j, 14);      // code j   -> bits 14,15
    const uint32_t hi = move_bits(w, 2 * j + 2, 30);  // code j+1 -> bits 30,31
    o[q] = __byte_perm(lo, hi, 0x7610) & 0xC000C000u;
  }
  bi = make_uint4(o[0], o[1], o[2], o[3]);
  br = make_uint4(o[0] ^ 0x40004000u, o[1] ^ 0x40004000u, o[2] ^ 0x40004000u, o[3] ^ 0x40004000u);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem* S = reinterpret_cast<Smem*>(smem + STAGES * kStageBytes);
  volatile int* abort = &S->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = (int64_t)blockIdx.x * BN;
  const int64_t m0 = (int64_t)blockIdx.y * BM;
  const int KB = (int)(a.K / BK);
  const int P = a.T * a.nbranch;

  auto xre = [&](int s) { return smem + s * kStageBytes; };
  auto xim = [&](int s) { return smem + s * kStageBytes + kTileX; };
  auto btile = [&](int s) { return smem + s * kStageBytes + 2 * kTileX; };
  auto ctile = [&](int s) { return smem + s * kStageBytes + 2 * kTileX + kTileB; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full_tma[s], 1);
      mbar_init(&S->full_b[s], 4);
      mbar_init(&S->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S->acc_full[b], 1);
      mbar_init(&S->acc_empty[b], 8);
    }
    mbar_init(&S->drain, 1);
    S->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&a.tmap_x[0]);
    prefetch_tmap(&a.tmap_x[1]);
    prefetch_tmap(&a.tmap_codes[0]);
    if (a.nbranch > 1) prefetch_tmap(&a.tmap_codes[1]);
  }
  if (warp == 1) {
    tmem_alloc(&S->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      for (int p = 0; p < P && !*abort; ++p) {
        const int t = p / a.nbranch, br = p % a.nbranch;
        const int32_t crow = (int32_t)((int64_t)t * a.N + n0);
        for (int kb = 0; kb < KB; ++kb) {
          const int it = p * KB + kb, s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&S->empty[s], ph ^ 1u, abort)) break;
          mbar_arrive_expect_tx(&S->full_tma[s], kTmaBytes);
          tma_load_2d(xre(s), &a.tmap_x[0], kb * BK, (int32_t)m0, &S->full_tma[s]);
          tma_load_2d(xim(s), &a.tmap_x[1], kb * BK, (int32_t)m0, &S->full_tma[s]);
          tma_load_2d(ctile(s), &a.tmap_codes[br], kb * (BK / 4), crow, &S->full_tma[s]);
          ++issued[s];
        }
      }
      if (*abort) {
        // Let every issued copy land before the CTA's shared memory is released.
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued[s] > 0) mbar_wait_bounded(&S->full_tma[s], (uint32_t)(issued[s] - 1) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int p = 0; p < P && !*abort; ++p) {
        const int buf = p & 1;
        if (!mbar_wait_bounded(&S->acc_empty[buf], ((uint32_t)(p >> 1) & 1u) ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d_re = tmem + buf * 256, d_im = d_re + 128;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          const int it = p * KB + kb, s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&S->full_tma[s], ph, abort) || !mbar_wait_bounded(&S->full_b[s], ph, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ar = smem_u32(xre(s)), ai = smem_u32(xim(s)), bb = smem_u32(btile(s));
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint32_t acc = (kb | ks) != 0;
            umma_bf16(d_re, umma_desc_sw128(ar + ks * 32), umma_desc_sw128(bb + ks * 32), kIdesc, acc);
            umma_bf16(d_im, umma_desc_sw128(ai + ks * 32), umma_desc_sw128(bb + ks * 32), kIdesc, acc);
          }
          umma_commit(&S->empty[s]);
        }
        if (!ok) break;
        umma_commit(&S->acc_full[buf]);
      }
      if (*abort) {
        volatile int never = 0;
        umma_commit(&S->drain);
        mbar_wait_bounded(&S->drain, 0u, &never);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ expanders
    const int e = threadIdx.x - 64;  // 0..127
    const int r = e >> 1, hf = e & 1;
    const bool row_ok = n0 + r < a.N;
    for (int p = 0; p < P && !__shfl_sync(0xffffffffu, *abort, 0); ++p) {
      for (int kb = 0; kb < KB; ++kb) {
        const int it = p * KB + kb, s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        int ok = 1;
        if (lane == 0)
          ok = mbar_wait_bounded(&S->empty[s], ph ^ 1u, abort) && mbar_wait_bounded(&S->full_tma[s], ph, abort);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        const uint2 cw = row_ok ? *reinterpret_cast<const uint2*>(ctile(s) + r * 16 + hf * 8) : make_uint2(0, 0);
        const uint32_t brow = smem_u32(btile(s)) + r * 128;
        const uint32_t birow = brow + BN * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 bi, brr;
          expand8(c < 2 ? cw.x : cw.y, (c & 1) * 8, bi, brr);
          if (!row_ok) bi = brr = make_uint4(0, 0, 0, 0);
          const int chunk = hf * 4 + c;
          const uint32_t off = (uint32_t)((chunk ^ (r & 7)) * 16);
          st_shared_v4(brow + off, brr);
          st_shared_v4(birow + off, bi);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S->full_b[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 6;             // 0..7
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int hc = e >> 2;              // output half: columns 32*hc .. 32*hc+31
    float yr[32], yi[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) yr[j] = yi[j] = 0.0f;
    for (int p = 0; p < P && !__shfl_sync(0xffffffffu, *abort, 0); ++p) {
      const int buf = p & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&S->acc_full[buf], (uint32_t)(p >> 1) & 1u, abort);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const int t = p / a.nbranch, br = p % a.nbranch;
      const float hr = 0.5f * __ldg(a.scales[br] + 2 * t);
      const float hi = 0.5f * __ldg(a.scales[br] + 2 * t + 1);
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + buf * 256 + hc * 32;
      const float sgn = br == 0 ? -1.0f : 1.0f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t u[16], v[16];
        tmem_ld_32x32b_x16(base + h * 16, u);             // P_rr
        tmem_ld_32x32b_x16(base + 128 + 64 + h * 16, v);  // P_ii
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          yr[h * 16 + j] += hr * __uint_as_float(u[j]) + sgn * hi * __uint_as_float(v[j]);
        tmem_ld_32x32b_x16(base + 128 + h * 16, u);       // P_ri
        tmem_ld_32x32b_x16(base + 64 + h * 16, v);        // P_ir
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          yi[h * 16 + j] += hi * __uint_as_float(v[j]) - sgn * hr * __uint_as_float(u[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->acc_empty[buf]);
    }
    if (!__shfl_sync(0xffffffffu, *abort, 0)) {
      const int64_t m = m0 + q * 32 + lane;
      const int64_t nb = n0 + hc * 32;
      if (m < a.M) {
        float* yre = a.y[0] + m * a.N + nb;
        float* yim = a.y[1] + m * a.N + nb;
        if ((a.N & 3) == 0 && nb + 32 <= a.N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            *reinterpret_cast<float4*>(yre + j) = make_float4(yr[j], yr[j + 1], yr[j + 2], yr[j + 3]);
            *reinterpret_cast<float4*>(yim + j) = make_float4(yi[j], yi[j + 1], yi[j + 2], yi[j + 3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nb + j < a.N) {
              yre[j] = yr[j];
              yim[j] = yi[j];
            }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S->abort) set_status(a.status, IFQ_DEV_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm(const ifq_layer* Ls, int count, int T, int64_t M, uint32_t* dev_status, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  for (int i = 0; i < count; ++i) {
    const ifq_layer& L = Ls[i];
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.nbranch = L.codes_w ? 2 : 1;
    a.N = L.N;
    a.K = L.K;
    a.M = M;
    a.T = T;
    a.status = dev_status;
    a.scales[0] = L.scales_u;
    a.scales[1] = L.scales_w;
    a.y[0] = L.y_re;
    a.y[1] = L.y_im;
    bool ok = make_map_2d(&a.tmap_x[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.x_re, (uint64_t)L.K, (uint64_t)M,
                          (uint64_t)L.K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map_2d(&a.tmap_x[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.x_im, (uint64_t)L.K, (uint64_t)M,
                          (uint64_t)L.K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    for (int b = 0; b < a.nbranch && ok; ++b)
      ok = make_map_2d(&a.tmap_codes[b], CU_TENSOR_MAP_DATA_TYPE_UINT8, b == 0 ? L.codes_u : L.codes_w,
                       (uint64_t)L.K / 4, (uint64_t)T * L.N, (uint64_t)L.K / 4, BK / 4, BN,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    dim3 grid((unsigned)((L.N + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
    gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace ifq
