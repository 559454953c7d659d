// C ABI of libifq: argument validation, then one enqueue per entry point.
// Every error is returned before anything is launched.
#include <cuda_runtime.h>
#include <string.h>

#include "../../include/ifq.h"
#include "ifq_common.cuh"
#include "ifq_internal.h"

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(ifq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// The kernels use sm_100a instructions (tcgen05, TMA); refuse other devices.
ifq_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return IFQ_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return IFQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return IFQ_ERR_CUDA;
  if (major != 10 || minor != 0) return IFQ_ERR_UNSUPPORTED;
  return IFQ_OK;
}

ifq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? IFQ_OK : IFQ_ERR_CUDA; }

ifq_status check_layers(const ifq_layer* L, int count, int T) {
  if (!L) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (T < 1 || T > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  for (int i = 0; i < count; ++i) {
    const ifq_layer& l = L[i];
    if (!l.codes_u || !l.scales_u || !l.x_re || !l.x_im || !l.y_re || !l.y_im) return IFQ_ERR_NULL;
    if ((l.codes_w == nullptr) != (l.scales_w == nullptr)) return IFQ_ERR_NULL;
    if ((l.rot_re == nullptr) != (l.rot_im == nullptr)) return IFQ_ERR_NULL;
    if (l.N < 1 || l.K < 4 || (l.K % 4) != 0) return IFQ_ERR_SHAPE;
    if (l.N > (int64_t)1 << 30 || l.K > (int64_t)1 << 30) return IFQ_ERR_SHAPE;
    if (!aligned16(l.codes_u) || (l.codes_w && !aligned16(l.codes_w)) || !aligned16(l.x_re) || !aligned16(l.x_im) ||
        !aligned16(l.y_re) || !aligned16(l.y_im) || (reinterpret_cast<uintptr_t>(l.scales_u) & 3u) ||
        (reinterpret_cast<uintptr_t>(l.scales_w) & 3u) || (l.rot_re && (!aligned16(l.rot_re) || !aligned16(l.rot_im))))
      return IFQ_ERR_ALIGN;
  }
  return IFQ_OK;
}

ifq_status check_qtensors(const ifq_qtensor* tensors, int count) {
  for (int i = 0; i < count; ++i) {
    const ifq_qtensor& t = tensors[i];
    if (!t.w_re || !t.w_im || !t.codes || !t.scales) return IFQ_ERR_NULL;
    if (t.N < 1 || t.K < 4 || (t.K % 4) != 0) return IFQ_ERR_SHAPE;
    if (t.K > (int64_t)1 << 30 || t.N > ((int64_t)1 << 40) / t.K) return IFQ_ERR_SHAPE;
    if (!aligned16(t.w_re) || !aligned16(t.w_im) || !aligned16(t.codes) || (reinterpret_cast<uintptr_t>(t.scales) & 3u))
      return IFQ_ERR_ALIGN;
  }
  return IFQ_OK;
}

// Decode kernel for a call: CUDA cores for layers whose K is not a multiple of 64, else the integer
// tensor-core kernel at one or two tokens and the bf16 kernel above them.
enum class GemvPath : int32_t { kI8 = 0, kBf16 = 1, kGeneric = 2 };

GemvPath gemv_path(const ifq_layer* L, int count, int B) {
  if (ifq::any_narrow_k(L, count)) return GemvPath::kGeneric;
  if (B <= ifq::IFQ_I8_MAX_BATCH) return GemvPath::kI8;
  return GemvPath::kBf16;
}

size_t gemv_workspace(GemvPath path, const ifq_layer* L, int count, int T, int B) {
  switch (path) {
    case GemvPath::kI8: return ifq::gemv_i8_workspace_bytes(L, count, T, B);
    case GemvPath::kBf16: return ifq::gemv_bf16_workspace_bytes(L, count, B);
    default: return 0;
  }
}

cudaError_t launch_path(GemvPath path, const ifq_layer* L, int count, int T, int B, void* ws, uint32_t* dev_status,
                        cudaStream_t s) {
  switch (path) {
    case GemvPath::kI8: return ifq::launch_gemv_i8(L, count, T, B, ws, dev_status, s);
    case GemvPath::kBf16: return ifq::launch_gemv(L, count, T, B, ws, dev_status, s);
    default: return ifq::launch_product_generic(L, count, T, B, dev_status, s);
  }
}

}  // namespace

extern "C" {

const char* ifq_status_string(ifq_status s) {
  switch (s) {
    case IFQ_OK: return "ok";
    case IFQ_ERR_NULL: return "a required pointer is NULL";
    case IFQ_ERR_SHAPE: return "invalid shape";
    case IFQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case IFQ_ERR_STAGES: return "stage count T outside 1..8";
    case IFQ_ERR_BATCH: return "batch outside the supported range";
    case IFQ_ERR_WORKSPACE: return "workspace missing or too small";
    case IFQ_ERR_CUDA: return "CUDA runtime error";
    case IFQ_ERR_UNSUPPORTED: return "device is not sm_100";
    case IFQ_ERR_COUNT: return "descriptor count outside 1..32";
    case IFQ_ERR_STATIC_LIMIT: return "call needs more than the 2 MiB static quantizer scratch";
  }
  return "unknown status";
}

ifq_status ifq_widely_linear_from_real(const float* R, int64_t rows, int64_t cols, float* U_re, float* U_im,
                                       float* W_re, float* W_im, ifq_stream_t stream) {
  if (!R || !U_re || !U_im || !W_re || !W_im) return IFQ_ERR_NULL;
  if (rows < 2 || cols < 2 || (rows & 1) || (cols & 1)) return IFQ_ERR_SHAPE;
  if (!aligned16(R) || !aligned16(U_re) || !aligned16(U_im) || !aligned16(W_re) || !aligned16(W_im))
    return IFQ_ERR_ALIGN;
  ifq_status st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_widely_linear(R, rows / 2, cols / 2, U_re, U_im, W_re, W_im, as_stream(stream)));
}

size_t ifq_quantize_workspace_bytes(const ifq_qtensor* tensors, int count, int T) {
  (void)T;
  if (!tensors || count < 1 || count > IFQ_MAX_GROUP) return 0;
  for (int i = 0; i < count; ++i)
    if (tensors[i].N < 1 || tensors[i].K < 4 || tensors[i].K % 4) return 0;
  return ifq::quant_workspace_bytes(tensors, count);
}

ifq_status ifq_quantize_pack(const ifq_qtensor* tensors, int count, int T, void* workspace, size_t workspace_bytes,
                             uint32_t* dev_status, ifq_stream_t stream) {
  if (!tensors) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (T < 1 || T > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  ifq_status st0 = check_qtensors(tensors, count);
  if (st0 != IFQ_OK) return st0;
  if (!workspace || workspace_bytes < ifq::quant_workspace_bytes(tensors, count)) return IFQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return IFQ_ERR_ALIGN;
  ifq_status st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_quantize(tensors, count, T, workspace, dev_status, as_stream(stream)));
}

ifq_status ifq_quantize_stage(const ifq_qtensor* tensors, int count, int t, void* partials, size_t partials_bytes,
                              uint32_t* dev_status, ifq_stream_t stream) {
  if (!tensors) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (t < 1 || t > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  ifq_status st = check_qtensors(tensors, count);
  if (st != IFQ_OK) return st;
  if (!partials || partials_bytes < ifq::quant_workspace_bytes(tensors, count)) return IFQ_ERR_WORKSPACE;
  if (!aligned16(partials)) return IFQ_ERR_ALIGN;
  st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_quantize_stage(tensors, count, t - 1, partials, dev_status, as_stream(stream)));
}

ifq_status ifq_quantize_finish(const ifq_qpartials* parts, int count, int t, ifq_stream_t stream) {
  if (!parts) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (t < 1 || t > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  for (int i = 0; i < count; ++i) {
    const ifq_qpartials& q = parts[i];
    if (!q.partials || !q.scales) return IFQ_ERR_NULL;
    if (q.N < 1 || q.K < 4 || (q.K % 4) != 0) return IFQ_ERR_SHAPE;
    if (q.K > (int64_t)1 << 30 || q.N > ((int64_t)1 << 40) / q.K) return IFQ_ERR_SHAPE;
    if (!aligned16(q.partials) || (reinterpret_cast<uintptr_t>(q.scales) & 3u)) return IFQ_ERR_ALIGN;
  }
  ifq_status st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_quantize_finish(parts, count, t - 1, as_stream(stream)));
}

ifq_status ifq_quantize_pack_static(const ifq_qtensor* tensors, int count, int T, uint32_t* dev_status,
                                    ifq_stream_t stream) {
  if (!tensors) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (T < 1 || T > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  for (int i = 0; i < count; ++i) {
    const ifq_qtensor& t = tensors[i];
    if (!t.w_re || !t.w_im || !t.codes || !t.scales) return IFQ_ERR_NULL;
    if (t.N < 1 || t.K < 4 || (t.K % 4) != 0) return IFQ_ERR_SHAPE;
    if (t.K > (int64_t)1 << 30 || t.N > ((int64_t)1 << 40) / t.K) return IFQ_ERR_SHAPE;
    if (!aligned16(t.w_re) || !aligned16(t.w_im) || !aligned16(t.codes) || (reinterpret_cast<uintptr_t>(t.scales) & 3u))
      return IFQ_ERR_ALIGN;
  }
  if (ifq::quant_workspace_bytes(tensors, count) > IFQ_QUANT_STATIC_SCRATCH_BYTES) return IFQ_ERR_STATIC_LIMIT;
  ifq_status st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_quantize_static(tensors, count, T, dev_status, as_stream(stream)));
}

static ifq_status check_wl_layers(const ifq_wl_layer* layers, int count, int T) {
  if (!layers) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP / 2) return IFQ_ERR_COUNT;
  if (T < 1 || T > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  for (int i = 0; i < count; ++i) {
    const ifq_wl_layer& l = layers[i];
    if (!l.R || !l.U_re || !l.U_im || !l.W_re || !l.W_im || !l.codes_u || !l.scales_u || !l.codes_w || !l.scales_w)
      return IFQ_ERR_NULL;
    if (l.rows < 2 || (l.rows & 1) || l.cols < 8 || (l.cols % 8) != 0) return IFQ_ERR_SHAPE;
    const int64_t n = l.rows / 2, m = l.cols / 2;
    if (m > (int64_t)1 << 30 || n > ((int64_t)1 << 40) / m) return IFQ_ERR_SHAPE;
    if (!aligned16(l.R) || !aligned16(l.U_re) || !aligned16(l.U_im) || !aligned16(l.W_re) || !aligned16(l.W_im) ||
        !aligned16(l.codes_u) || !aligned16(l.codes_w) || (reinterpret_cast<uintptr_t>(l.scales_u) & 3u) ||
        (reinterpret_cast<uintptr_t>(l.scales_w) & 3u))
      return IFQ_ERR_ALIGN;
  }
  return IFQ_OK;
}

size_t ifq_widely_linear_quantize_workspace_bytes(const ifq_wl_layer* layers, int count, int T) {
  if (!layers || count < 1 || count > IFQ_MAX_GROUP / 2) return 0;
  (void)T;
  for (int i = 0; i < count; ++i)
    if (layers[i].rows < 2 || (layers[i].rows & 1) || layers[i].cols < 8 || (layers[i].cols % 8) != 0) return 0;
  return ifq::widely_linear_quant_workspace_bytes(layers, count);
}

ifq_status ifq_widely_linear_quantize_pack(const ifq_wl_layer* layers, int count, int T, void* workspace,
                                           size_t workspace_bytes, uint32_t* dev_status, ifq_stream_t stream) {
  ifq_status st = check_wl_layers(layers, count, T);
  if (st != IFQ_OK) return st;
  if (!workspace || workspace_bytes < ifq::widely_linear_quant_workspace_bytes(layers, count))
    return IFQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return IFQ_ERR_ALIGN;
  st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_widely_linear_quantize(layers, count, T, workspace, dev_status, as_stream(stream)));
}

ifq_status ifq_dequantize(const ifq_dqtensor* tensors, int count, int T, ifq_stream_t stream) {
  if (!tensors) return IFQ_ERR_NULL;
  if (count < 1 || count > IFQ_MAX_GROUP) return IFQ_ERR_COUNT;
  if (T < 1 || T > IFQ_MAX_STAGES) return IFQ_ERR_STAGES;
  for (int i = 0; i < count; ++i) {
    const ifq_dqtensor& t = tensors[i];
    if (!t.codes || !t.scales || !t.w_re || !t.w_im) return IFQ_ERR_NULL;
    if (t.N < 1 || t.K < 4 || (t.K % 4) != 0) return IFQ_ERR_SHAPE;
    if (t.K > (int64_t)1 << 30 || t.N > ((int64_t)1 << 40) / t.K) return IFQ_ERR_SHAPE;
    if (!aligned16(t.codes) || !aligned16(t.w_re) || !aligned16(t.w_im) ||
        (reinterpret_cast<uintptr_t>(t.scales) & 3u))
      return IFQ_ERR_ALIGN;
  }
  ifq_status st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(ifq::launch_dequantize(tensors, count, T, as_stream(stream)));
}

size_t ifq_gemv_workspace_bytes(const ifq_layer* layers, int count, int T, int B) {
  if (check_layers(layers, count, T) != IFQ_OK || B < 1 || B > IFQ_MAX_GEMV_BATCH) return 0;
  return gemv_workspace(gemv_path(layers, count, B), layers, count, T, B);
}

ifq_status ifq_gemv(const ifq_layer* layers, int count, int T, int B, void* workspace, size_t workspace_bytes,
                    uint32_t* dev_status, ifq_stream_t stream) {
  ifq_status st = check_layers(layers, count, T);
  if (st != IFQ_OK) return st;
  if (B < 1 || B > IFQ_MAX_GEMV_BATCH) return IFQ_ERR_BATCH;
  const GemvPath path = gemv_path(layers, count, B);
  const size_t need = gemv_workspace(path, layers, count, T, B);
  if (need > 0 && (!workspace || workspace_bytes < need)) return IFQ_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return IFQ_ERR_ALIGN;
  st = check_device();
  if (st != IFQ_OK) return st;
  return from_cuda(launch_path(path, layers, count, T, B, workspace, dev_status, as_stream(stream)));
}

// A prepared decode call, in the caller's host buffer: the routing and the descriptors, then (integer
// path) the finished launch parameters at a 64-byte boundary.
namespace {
constexpr uint32_t kPlanMagic = 0x50514649u;
struct alignas(64) GemvPlanHeader {
  uint32_t magic;
  int32_t path;  // a GemvPath
  int32_t count, T, B;
  void* workspace;
  uint32_t* dev_status;
  ifq_layer layers[IFQ_MAX_GROUP];
};
constexpr size_t kPlanParamsOffset = (sizeof(GemvPlanHeader) + 63) & ~(size_t)63;
}  // namespace

size_t ifq_gemv_plan_bytes(void) { return kPlanParamsOffset + ifq::gemv_i8_plan_bytes(); }

ifq_status ifq_gemv_prepare(const ifq_layer* layers, int count, int T, int B, void* workspace,
                            size_t workspace_bytes, uint32_t* dev_status, void* plan, size_t plan_bytes) {
  ifq_status st = check_layers(layers, count, T);
  if (st != IFQ_OK) return st;
  if (B < 1 || B > IFQ_MAX_GEMV_BATCH) return IFQ_ERR_BATCH;
  if (!plan) return IFQ_ERR_NULL;
  if (plan_bytes < ifq_gemv_plan_bytes()) return IFQ_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(plan) & 63u) return IFQ_ERR_ALIGN;
  const GemvPath path = gemv_path(layers, count, B);
  const size_t need = gemv_workspace(path, layers, count, T, B);
  if (need > 0 && (!workspace || workspace_bytes < need)) return IFQ_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return IFQ_ERR_ALIGN;
  st = check_device();
  if (st != IFQ_OK) return st;
  GemvPlanHeader* h = static_cast<GemvPlanHeader*>(plan);
  memset(h, 0, sizeof(GemvPlanHeader));
  h->path = (int32_t)path;
  h->count = count;
  h->T = T;
  h->B = B;
  h->workspace = workspace;
  h->dev_status = dev_status;
  memcpy(h->layers, layers, sizeof(ifq_layer) * count);
  if (path == GemvPath::kI8) {
    const cudaError_t e = ifq::plan_gemv_i8(layers, count, T, B, workspace, dev_status,
                                             static_cast<char*>(plan) + kPlanParamsOffset);
    if (e != cudaSuccess) return IFQ_ERR_CUDA;
  }
  h->magic = kPlanMagic;
  return IFQ_OK;
}

ifq_status ifq_gemv_run(const void* plan, ifq_stream_t stream) {
  if (!plan) return IFQ_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(plan) & 63u) return IFQ_ERR_ALIGN;
  const GemvPlanHeader* h = static_cast<const GemvPlanHeader*>(plan);
  if (h->magic != kPlanMagic) return IFQ_ERR_NULL;
  const GemvPath path = (GemvPath)h->path;
  if (path == GemvPath::kI8)
    return from_cuda(ifq::run_gemv_i8_plan(static_cast<const char*>(plan) + kPlanParamsOffset, as_stream(stream)));
  return from_cuda(launch_path(path, h->layers, h->count, h->T, h->B, h->workspace, h->dev_status, as_stream(stream)));
}

ifq_status ifq_gemm_wait_limit(const ifq_layer* layers, int count, int T, int64_t M, uint64_t wait_limit_ns,
                               uint32_t* dev_status, ifq_stream_t stream) {
  ifq_status st = check_layers(layers, count, T);
  if (st != IFQ_OK) return st;
  if (M < 1 || M > ((int64_t)1 << 31) - 128) return IFQ_ERR_BATCH;
  for (int i = 0; i < count; ++i)
    if ((int64_t)T * layers[i].N > ((int64_t)1 << 31) - 64) return IFQ_ERR_SHAPE;
  if (wait_limit_ns == 0) return IFQ_ERR_SHAPE;
  st = check_device();
  if (st != IFQ_OK) return st;
  if (ifq::any_narrow_k(layers, count))
    return from_cuda(ifq::launch_product_generic(layers, count, T, M, dev_status, as_stream(stream)));
  return from_cuda(ifq::launch_gemm(layers, count, T, M, wait_limit_ns, dev_status, as_stream(stream)));
}

ifq_status ifq_gemm(const ifq_layer* layers, int count, int T, int64_t M, uint32_t* dev_status,
                    ifq_stream_t stream) {
  return ifq_gemm_wait_limit(layers, count, T, M, IFQ_WAIT_LIMIT_NS, dev_status, stream);
}

}  // extern "C"
