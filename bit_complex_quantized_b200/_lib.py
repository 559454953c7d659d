"""ctypes binding of libifq (include/ifq.h): argument marshalling only.

Each function takes torch tensors that already live on the GPU, passes their
device pointers and sizes to the C ABI function of the same name, and raises
IfqError on a non-OK status.  No arithmetic of the method happens here, and
there is no fallback: if libifq.so is missing, loading fails loudly.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libifq.so")

IFQ_MAX_STAGES = 8
IFQ_MAX_GEMV_BATCH = 16
IFQ_MAX_GROUP = 32
IFQ_QUANT_STATIC_SCRATCH_BYTES = 2 << 20
IFQ_DEV_NONFINITE = 0x1
IFQ_DEV_TIMEOUT = 0x2

EXPORTED = (
    "ifq_status_string",
    "ifq_widely_linear_from_real",
    "ifq_quantize_workspace_bytes",
    "ifq_quantize_pack",
    "ifq_quantize_pack_static",
    "ifq_quantize_stage",
    "ifq_quantize_finish",
    "ifq_widely_linear_quantize_workspace_bytes",
    "ifq_widely_linear_quantize_pack",
    "ifq_dequantize",
    "ifq_gemv_workspace_bytes",
    "ifq_gemv",
    "ifq_gemv_plan_bytes",
    "ifq_gemv_prepare",
    "ifq_gemv_run",
    "ifq_gemm",
    "ifq_gemm_wait_limit",
)

STATUS_NAMES = {
    0: "IFQ_OK", 1: "IFQ_ERR_NULL", 2: "IFQ_ERR_SHAPE", 3: "IFQ_ERR_ALIGN", 4: "IFQ_ERR_STAGES",
    5: "IFQ_ERR_BATCH", 6: "IFQ_ERR_WORKSPACE", 7: "IFQ_ERR_CUDA", 8: "IFQ_ERR_UNSUPPORTED", 9: "IFQ_ERR_COUNT",
    10: "IFQ_ERR_STATIC_LIMIT",
}


class IfqError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class QTensor(ctypes.Structure):
    _fields_ = [("w_re", ctypes.c_void_p), ("w_im", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class QPartials(ctypes.Structure):
    _fields_ = [("partials", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("scales", ctypes.c_void_p)]


class DqTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("w_re", ctypes.c_void_p), ("w_im", ctypes.c_void_p)]


class WlLayer(ctypes.Structure):
    _fields_ = [("R", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("U_re", ctypes.c_void_p), ("U_im", ctypes.c_void_p), ("W_re", ctypes.c_void_p),
                ("W_im", ctypes.c_void_p), ("codes_u", ctypes.c_void_p), ("scales_u", ctypes.c_void_p),
                ("codes_w", ctypes.c_void_p), ("scales_w", ctypes.c_void_p)]


class Layer(ctypes.Structure):
    _fields_ = [("codes_u", ctypes.c_void_p), ("scales_u", ctypes.c_void_p), ("codes_w", ctypes.c_void_p),
                ("scales_w", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("x_re", ctypes.c_void_p), ("x_im", ctypes.c_void_p), ("y_re", ctypes.c_void_p),
                ("y_im", ctypes.c_void_p), ("rot_re", ctypes.c_void_p), ("rot_im", ctypes.c_void_p)]


_lib = None


def load():
    """Load libifq.so (built in-tree); raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with python -m bit_complex_quantized_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    lib.ifq_status_string.restype = ctypes.c_char_p
    lib.ifq_status_string.argtypes = [i32]
    lib.ifq_widely_linear_from_real.restype = i32
    lib.ifq_widely_linear_from_real.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
    lib.ifq_quantize_workspace_bytes.restype = sz
    lib.ifq_quantize_workspace_bytes.argtypes = [ctypes.POINTER(QTensor), i32, i32]
    lib.ifq_quantize_pack.restype = i32
    lib.ifq_quantize_pack.argtypes = [ctypes.POINTER(QTensor), i32, i32, vp, sz, vp, vp]
    lib.ifq_quantize_pack_static.restype = i32
    lib.ifq_quantize_pack_static.argtypes = [ctypes.POINTER(QTensor), i32, i32, vp, vp]
    lib.ifq_quantize_stage.restype = i32
    lib.ifq_quantize_stage.argtypes = [ctypes.POINTER(QTensor), i32, i32, vp, sz, vp, vp]
    lib.ifq_quantize_finish.restype = i32
    lib.ifq_quantize_finish.argtypes = [ctypes.POINTER(QPartials), i32, i32, vp]
    lib.ifq_widely_linear_quantize_workspace_bytes.restype = sz
    lib.ifq_widely_linear_quantize_workspace_bytes.argtypes = [ctypes.POINTER(WlLayer), i32, i32]
    lib.ifq_widely_linear_quantize_pack.restype = i32
    lib.ifq_widely_linear_quantize_pack.argtypes = [ctypes.POINTER(WlLayer), i32, i32, vp, sz, vp, vp]
    lib.ifq_dequantize.restype = i32
    lib.ifq_dequantize.argtypes = [ctypes.POINTER(DqTensor), i32, i32, vp]
    lib.ifq_gemv_workspace_bytes.restype = sz
    lib.ifq_gemv_workspace_bytes.argtypes = [ctypes.POINTER(Layer), i32, i32, i32]
    lib.ifq_gemv.restype = i32
    lib.ifq_gemv.argtypes = [ctypes.POINTER(Layer), i32, i32, i32, vp, sz, vp, vp]
    lib.ifq_gemv_plan_bytes.restype = sz
    lib.ifq_gemv_plan_bytes.argtypes = []
    lib.ifq_gemv_prepare.restype = i32
    lib.ifq_gemv_prepare.argtypes = [ctypes.POINTER(Layer), i32, i32, i32, vp, sz, vp, vp, sz]
    lib.ifq_gemv_run.restype = i32
    lib.ifq_gemv_run.argtypes = [vp, vp]
    lib.ifq_gemm.restype = i32
    lib.ifq_gemm.argtypes = [ctypes.POINTER(Layer), i32, i32, i64, vp, vp]
    lib.ifq_gemm_wait_limit.restype = i32
    lib.ifq_gemm_wait_limit.argtypes = [ctypes.POINTER(Layer), i32, i32, i64, ctypes.c_uint64, vp, vp]
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status):
    if status != 0:
        raise IfqError(status, load().ifq_status_string(status).decode())


def ifq_status_string(status):
    return load().ifq_status_string(int(status)).decode()


def ifq_widely_linear_from_real(R, U_re, U_im, W_re, W_im, stream=None):
    """R: float32 [2n][2m]; outputs float32 [n][m] (all on the device)."""
    rows, cols = R.shape
    _check(load().ifq_widely_linear_from_real(_ptr(R), rows, cols, _ptr(U_re), _ptr(U_im), _ptr(W_re), _ptr(W_im),
                                              _stream(stream)))


def _qtensors(tensors):
    arr = (QTensor * len(tensors))()
    for i, t in enumerate(tensors):
        w_re, w_im, codes, scales = t
        arr[i] = QTensor(w_re.data_ptr(), w_im.data_ptr(), w_re.shape[0], w_re.shape[1], codes.data_ptr(),
                         scales.data_ptr())
    return arr


def ifq_quantize_workspace_bytes(tensors, T):
    """tensors: list of (w_re, w_im, codes, scales)."""
    return int(load().ifq_quantize_workspace_bytes(_qtensors(tensors), len(tensors), T))


def ifq_quantize_pack(tensors, T, workspace, dev_status=None, stream=None, workspace_bytes=None):
    """tensors: list of (w_re [N][K] f32, w_im, codes u8 [T][N][K/4], scales f32 [T][2])."""
    arr = _qtensors(tensors)
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().ifq_quantize_pack(arr, len(tensors), T, _ptr(workspace), nbytes, _ptr(dev_status),
                                    _stream(stream)))


def ifq_quantize_pack_static(tensors, T, dev_status=None, stream=None):
    """As ifq_quantize_pack, with the library's fixed device scratch instead of a workspace."""
    arr = _qtensors(tensors)
    _check(load().ifq_quantize_pack_static(arr, len(tensors), T, _ptr(dev_status), _stream(stream)))


def ifq_quantize_stage(tensors, t, partials, dev_status=None, stream=None):
    """Stage t (1-based) of a row shard: codes of the shard and its tile partials in `partials`
    (a device buffer of ifq_quantize_workspace_bytes(tensors, t) bytes)."""
    arr = _qtensors(tensors)
    _check(load().ifq_quantize_stage(arr, len(tensors), t, _ptr(partials),
                                     partials.numel() * partials.element_size(), _ptr(dev_status), _stream(stream)))


def ifq_quantize_finish(parts, t, stream=None):
    """parts: list of (gathered partials of a whole tensor, N, K, scales [T][2]); writes stage t's scales."""
    arr = (QPartials * len(parts))()
    for i, (pt, N, K, sc) in enumerate(parts):
        arr[i] = QPartials(pt.data_ptr(), N, K, sc.data_ptr())
    _check(load().ifq_quantize_finish(arr, len(parts), t, _stream(stream)))


def ifq_dequantize(tensors, T, stream=None):
    """tensors: list of (codes u8 [T][N][K/4], scales f32 [T][2], w_re, w_im) with w_* bf16 [N][K]
    (written): the dequantized weights sum_t (s_re,t Re b_t + i s_im,t Im b_t)."""
    arr = (DqTensor * len(tensors))()
    for i, (codes, scales, w_re, w_im) in enumerate(tensors):
        arr[i] = DqTensor(codes.data_ptr(), scales.data_ptr(), w_re.shape[0], w_re.shape[1], w_re.data_ptr(),
                          w_im.data_ptr())
    _check(load().ifq_dequantize(arr, len(tensors), T, _stream(stream)))


def _wl_layers(layers):
    arr = (WlLayer * len(layers))()
    for i, d in enumerate(layers):
        R = d["R"]
        arr[i] = WlLayer(R.data_ptr(), R.shape[0], R.shape[1], _ptr(d["U_re"]), _ptr(d["U_im"]), _ptr(d["W_re"]),
                         _ptr(d["W_im"]), _ptr(d["codes_u"]), _ptr(d["scales_u"]), _ptr(d["codes_w"]),
                         _ptr(d["scales_w"]))
    return arr


def ifq_widely_linear_quantize_workspace_bytes(layers, T):
    """layers: list of dicts with R [2n][2m] f32, U_re, U_im, W_re, W_im [n][m] f32,
    codes_u, codes_w u8 [T][n][m/4], scales_u, scales_w f32 [T][2] (all on the device)."""
    return int(load().ifq_widely_linear_quantize_workspace_bytes(_wl_layers(layers), len(layers), T))


def ifq_widely_linear_quantize_pack(layers, T, workspace, dev_status=None, stream=None, workspace_bytes=None):
    """Conversion and T-stage quantization of each layer in one call, stage 1 fused with the conversion."""
    arr = _wl_layers(layers)
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().ifq_widely_linear_quantize_pack(arr, len(layers), T, _ptr(workspace), nbytes, _ptr(dev_status),
                                                  _stream(stream)))


def _layers(layers):
    arr = (Layer * len(layers))()
    for i, d in enumerate(layers):
        arr[i] = Layer(d["codes_u"].data_ptr(), d["scales_u"].data_ptr(),
                       None if d.get("codes_w") is None else d["codes_w"].data_ptr(),
                       None if d.get("scales_w") is None else d["scales_w"].data_ptr(),
                       d["N"], d["K"], d["x_re"].data_ptr(), d["x_im"].data_ptr(), d["y_re"].data_ptr(),
                       d["y_im"].data_ptr(),
                       None if d.get("rot_re") is None else d["rot_re"].data_ptr(),
                       None if d.get("rot_im") is None else d["rot_im"].data_ptr())
    return arr


class LayerSet:
    """Layer descriptors marshalled once, for a caller that repeats the same grouped call
    (the tensors must stay alive and in place).  Accepted wherever a list of layer dicts is."""

    def __init__(self, layers):
        self.layers = list(layers)
        self.array = _layers(self.layers)

    def __len__(self):
        return len(self.layers)


def _as_array(layers):
    return (layers.array, len(layers)) if isinstance(layers, LayerSet) else (_layers(layers), len(layers))


def ifq_gemv_workspace_bytes(layers, T, B):
    arr, n = _as_array(layers)
    return int(load().ifq_gemv_workspace_bytes(arr, n, T, B))


def ifq_gemv(layers, T, B, workspace=None, dev_status=None, stream=None, workspace_bytes=None):
    """layers: list of dicts with codes_u, scales_u, codes_w, scales_w (or None), N, K,
    x_re, x_im (bf16 [B][K]), y_re, y_im (float32 [B][N]), and optionally rot_re, rot_im
    (float32 [B][N]: each output is multiplied by rot_re + i rot_im).  workspace: a device
    buffer of ifq_gemv_workspace_bytes() bytes (no initial contents needed)."""
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if workspace_bytes is not None:
        nbytes = workspace_bytes
    arr, n = _as_array(layers)
    _check(load().ifq_gemv(arr, n, T, B, _ptr(workspace), nbytes, _ptr(dev_status), _stream(stream)))


class GemvPlan:
    """A prepared decode call (ifq_gemv_prepare) in a 64-byte aligned host buffer; run() launches it
    (ifq_gemv_run).  The layers' tensors, the workspace and dev_status must stay alive and in place."""

    def __init__(self, layers, T, B, workspace=None, dev_status=None, workspace_bytes=None):
        lib = load()
        n = int(lib.ifq_gemv_plan_bytes())
        self._buf = ctypes.create_string_buffer(n + 64)
        addr = ctypes.addressof(self._buf)
        self.ptr = ctypes.c_void_p((addr + 63) & ~63)
        self._keep = (layers, workspace, dev_status)
        nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        if workspace_bytes is not None:
            nbytes = workspace_bytes
        arr, cnt = _as_array(layers)
        self._arr = arr
        _check(lib.ifq_gemv_prepare(arr, cnt, T, B, _ptr(workspace), nbytes, _ptr(dev_status), self.ptr, n))

    def run(self, stream=None):
        _check(load().ifq_gemv_run(self.ptr, _stream(stream)))


def ifq_gemm(layers, T, M, dev_status=None, stream=None):
    """As ifq_gemv with x [M][K] and y [M][N]."""
    arr, n = _as_array(layers)
    _check(load().ifq_gemm(arr, n, T, M, _ptr(dev_status), _stream(stream)))


def ifq_gemm_wait_limit(layers, T, M, wait_limit_ns, dev_status=None, stream=None):
    """As ifq_gemm with each pipeline wait bounded by wait_limit_ns (IFQ_DEV_TIMEOUT when one runs out)."""
    arr, n = _as_array(layers)
    _check(load().ifq_gemm_wait_limit(arr, n, T, M, int(wait_limit_ns), _ptr(dev_status), _stream(stream)))


# Raw entry point for callers that build ctypes descriptors themselves.
def raw():
    return load()
