// Internal launch interfaces between the C-ABI layer (api.cu) and the kernel
// files.  Arguments are validated by the caller; these only enqueue work.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ifq.h"

namespace ifq {

cudaError_t launch_widely_linear(const float* R, int64_t n, int64_t m, float* U_re, float* U_im, float* W_re,
                                 float* W_im, cudaStream_t s);

// Quantizer: per-tensor block counts and workspace layout.
int64_t quant_blocks_for(int64_t N, int64_t K);
size_t quant_workspace_bytes(const ifq_qtensor* t, int count);
cudaError_t launch_quantize(const ifq_qtensor* t, int count, int T, void* ws, uint32_t* dev_status, cudaStream_t s);
// As launch_quantize, with the scratch in a file-scope device array (no allocation).
cudaError_t launch_quantize_static(const ifq_qtensor* t, int count, int T, uint32_t* dev_status, cudaStream_t s);

// One stage on row shards (tile partials, no reduction), and the scales from gathered partials.
cudaError_t launch_quantize_stage(const ifq_qtensor* t, int count, int stage, void* partials, uint32_t* dev_status,
                                  cudaStream_t s);
cudaError_t launch_quantize_finish(const ifq_qpartials* q, int count, int stage, cudaStream_t s);

// Conversion fused with stage 1 of the quantizer, then stages 2..T (quantize.cu).
size_t widely_linear_quant_workspace_bytes(const ifq_wl_layer* L, int count);
cudaError_t launch_widely_linear_quantize(const ifq_wl_layer* L, int count, int T, void* ws, uint32_t* dev_status,
                                          cudaStream_t s);

// Dequantized bf16 weights for training (dequantize.cu).
cudaError_t launch_dequantize(const ifq_dqtensor* t, int count, int T, cudaStream_t s);

// bf16 path for B > IFQ_I8_MAX_BATCH (gemv.cu); its workspace holds the partial sums of
// layers cut into K segments (0 bytes when no layer is).
size_t gemv_bf16_workspace_bytes(const ifq_layer* L, int count, int B);
cudaError_t launch_gemv(const ifq_layer* L, int count, int T, int B, void* ws, uint32_t* dev_status,
                        cudaStream_t s);

// Integer tensor-core path for B <= IFQ_I8_MAX_BATCH tokens (gemv_i8.cu) and its workspace size.
constexpr int IFQ_I8_MAX_BATCH = 2;
size_t gemv_i8_workspace_bytes(const ifq_layer* L, int count, int T, int B);
cudaError_t launch_gemv_i8(const ifq_layer* L, int count, int T, int B, void* ws, uint32_t* dev_status,
                           cudaStream_t s);
// A prepared call of the integer path: its finished launch parameters in a caller buffer (64-byte aligned).
size_t gemv_i8_plan_bytes();
cudaError_t plan_gemv_i8(const ifq_layer* L, int count, int T, int B, void* ws, uint32_t* dev_status, void* dst);
cudaError_t run_gemv_i8_plan(const void* src, cudaStream_t s);

// Layers whose K is a multiple of 4 but not of 64 (product_generic.cu): any number of rows.
cudaError_t launch_product_generic(const ifq_layer* L, int count, int T, int64_t rows, uint32_t* dev_status,
                                   cudaStream_t s);
inline bool any_narrow_k(const ifq_layer* L, int count) {
  for (int i = 0; i < count; ++i)
    if (L[i].K % 64 != 0) return true;
  return false;
}

// Tiled TMA descriptor (cuTensorMapEncodeTiled through the runtime's driver entry point; no
// libcuda link).  strides: rank - 1 byte strides of dimensions 1.. ; zero fill out of bounds.
// False if the entry point is missing or the driver rejects the description.
bool encode_tiled_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                      const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw);

cudaError_t launch_gemm(const ifq_layer* L, int count, int T, int64_t M, uint64_t wait_ns, uint32_t* dev_status,
                        cudaStream_t s);

}  // namespace ifq
