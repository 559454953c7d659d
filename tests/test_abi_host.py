"""Host-side checks of libifq (no GPU needed): the shared library loads and
exports every function include/ifq.h declares, and argument errors come back
as status codes before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "ifq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ifq_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_function():
    lib = Q.load()
    names = _declared_functions()
    assert len(names) >= 6
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTED)


def test_status_strings():
    lib = Q.load()
    for s in range(10):
        assert lib.ifq_status_string(s)
    assert Q.ifq_status_string(0) == "ok"


FAKE = 0x10000  # non-null, 16-byte aligned, never dereferenced by validation


def _layer(**kw):
    d = dict(codes_u=FAKE, scales_u=FAKE, codes_w=None, scales_w=None, N=64, K=128,
             x_re=FAKE, x_im=FAKE, y_re=FAKE, y_im=FAKE)
    d.update(kw)
    return L.Layer(d["codes_u"], d["scales_u"], d["codes_w"], d["scales_w"], d["N"], d["K"], d["x_re"],
                   d["x_im"], d["y_re"], d["y_im"])


def _call_gemv(layers, T=1, B=1, ws=FAKE, ws_bytes=1 << 30):
    arr = (L.Layer * max(1, len(layers)))(*layers)
    return Q.load().ifq_gemv(arr if layers else None, len(layers), T, B, ws, ws_bytes, None, None)


def _call_gemm(layers, T=1, M=128):
    arr = (L.Layer * max(1, len(layers)))(*layers)
    return Q.load().ifq_gemm(arr if layers else None, len(layers), T, M, None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(codes_u=None), 1), (dict(x_re=None), 1), (dict(y_im=None), 1),
    (dict(codes_w=FAKE), 1),                       # W codes without W scales
    (dict(K=102), 2), (dict(K=0), 2), (dict(N=0), 2), (dict(K=2), 2),
    (dict(codes_u=FAKE + 4), 3), (dict(x_im=FAKE + 2), 3), (dict(scales_u=FAKE + 1), 3),
])
def test_gemv_gemm_argument_errors(kw, status):
    assert _call_gemv([_layer(**kw)]) == status
    assert _call_gemm([_layer(**kw)]) == status


def test_products_accept_every_width_the_quantizer_accepts():
    """K % 4 == 0 is enough for the products (narrow widths run the CUDA-core kernel): the shape
    checks pass and the call stops only at the batch check, before anything is launched."""
    lib = Q.load()
    for K in (4, 60, 100, 196, 2052):
        assert _call_gemv([_layer(K=K)], B=0) == 5
        assert _call_gemm([_layer(K=K)], M=0) == 5
        assert lib.ifq_gemv_workspace_bytes((L.Layer * 1)(_layer(K=K)), 1, 2, 1) == 0


def test_batch_stage_and_count_errors():
    good = _layer()
    assert _call_gemv([good], T=0) == 4
    assert _call_gemv([good], T=9) == 4
    assert _call_gemv([good], B=0) == 5
    assert _call_gemv([good], B=17) == 5
    assert _call_gemm([good], M=0) == 5
    assert _call_gemv([]) == 1
    many = [good] * 33
    arr = (L.Layer * 33)(*many)
    assert Q.load().ifq_gemv(arr, 33, 1, 1, FAKE, 1 << 30, None, None) == 9


def test_gemv_workspace_errors():
    good = _layer(N=300, K=5504)
    lib = Q.load()
    arr = (L.Layer * 1)(good)
    need = lib.ifq_gemv_workspace_bytes(arr, 1, 2, 1)
    assert need > 0
    assert lib.ifq_gemv_workspace_bytes(arr, 1, 2, 2) > need   # integer path up to B = 2, per token
    assert _call_gemv([good], T=2, B=2, ws=FAKE, ws_bytes=lib.ifq_gemv_workspace_bytes(arr, 1, 2, 2) - 1) == 6
    # B >= 3 (bf16 path): partial sums of the K segments of a layer longer than 2048 positions
    for B in (3, 5, 16):
        assert lib.ifq_gemv_workspace_bytes(arr, 1, 2, B) == (((5504 + 2047) // 2048) * B * 300 * 8 + 255) // 256 * 256
    short = (L.Layer * 1)(_layer(N=300, K=2048))
    assert lib.ifq_gemv_workspace_bytes(short, 1, 2, 5) == 0
    assert _call_gemv([good], T=2, B=5, ws=None, ws_bytes=0) == 6
    assert _call_gemv([good], T=2, B=1, ws=None, ws_bytes=need) == 6
    assert _call_gemv([good], T=2, B=1, ws=FAKE, ws_bytes=need - 1) == 6
    assert _call_gemv([good], T=2, B=1, ws=FAKE + 8, ws_bytes=need) == 3


def test_quantize_argument_errors():
    lib = Q.load()
    qt = L.QTensor(FAKE, FAKE, 64, 128, FAKE, FAKE)
    arr = (L.QTensor * 1)(qt)
    need = lib.ifq_quantize_workspace_bytes(arr, 1, 2)
    assert need > 0
    assert lib.ifq_quantize_pack(arr, 1, 2, None, need, None, None) == 6
    assert lib.ifq_quantize_pack(arr, 1, 2, FAKE, need - 1, None, None) == 6
    assert lib.ifq_quantize_pack(arr, 1, 9, FAKE, need, None, None) == 4
    assert lib.ifq_quantize_pack(arr, 0, 2, FAKE, need, None, None) == 9
    bad = (L.QTensor * 1)(L.QTensor(FAKE, FAKE, 64, 126, FAKE, FAKE))
    assert lib.ifq_quantize_pack(bad, 1, 2, FAKE, need, None, None) == 2
    assert lib.ifq_quantize_workspace_bytes(bad, 1, 2) == 0
    mis = (L.QTensor * 1)(L.QTensor(FAKE + 8, FAKE, 64, 128, FAKE, FAKE))
    assert lib.ifq_quantize_pack(mis, 1, 2, FAKE, need, None, None) == 3
    nul = (L.QTensor * 1)(L.QTensor(FAKE, None, 64, 128, FAKE, FAKE))
    assert lib.ifq_quantize_pack(nul, 1, 2, FAKE, need, None, None) == 1


def test_workspace_grows_with_tensor_size():
    lib = Q.load()
    small = (L.QTensor * 1)(L.QTensor(FAKE, FAKE, 64, 128, FAKE, FAKE))
    big = (L.QTensor * 2)(L.QTensor(FAKE, FAKE, 4096, 4096, FAKE, FAKE), L.QTensor(FAKE, FAKE, 64, 128, FAKE, FAKE))
    assert lib.ifq_quantize_workspace_bytes(big, 2, 3) > lib.ifq_quantize_workspace_bytes(small, 1, 3)


def test_convert_argument_errors():
    lib = Q.load()
    assert lib.ifq_widely_linear_from_real(None, 4, 4, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.ifq_widely_linear_from_real(FAKE, 3, 4, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert lib.ifq_widely_linear_from_real(FAKE, 4, 0, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert lib.ifq_widely_linear_from_real(FAKE, 4, 4, FAKE + 4, FAKE, FAKE, FAKE, None) == 3


def test_layerset_marshals_the_same_descriptors():
    import torch
    t = lambda *s: torch.zeros(*s, dtype=torch.float32)  # noqa: E731
    layers = [dict(codes_u=torch.zeros(2, 8, 16, dtype=torch.uint8), scales_u=t(2, 2), codes_w=None, scales_w=None,
                   N=8, K=64, x_re=t(1, 64), x_im=t(1, 64), y_re=t(1, 8), y_im=t(1, 8)) for _ in range(3)]
    a = L._layers(layers)
    b = Q.LayerSet(layers)
    assert len(b) == 3
    for x, y in zip(a, b.array):
        for f, _ in L.Layer._fields_:
            assert getattr(x, f) == getattr(y, f)


def _wl(**kw):
    d = dict(R=FAKE, rows=8, cols=16, U_re=FAKE, U_im=FAKE, W_re=FAKE, W_im=FAKE, codes_u=FAKE, scales_u=FAKE,
             codes_w=FAKE, scales_w=FAKE)
    d.update(kw)
    return L.WlLayer(d["R"], d["rows"], d["cols"], d["U_re"], d["U_im"], d["W_re"], d["W_im"], d["codes_u"],
                     d["scales_u"], d["codes_w"], d["scales_w"])


def test_fused_convert_quantize_argument_errors():
    lib = Q.load()
    arr = (L.WlLayer * 1)(_wl())
    need = lib.ifq_widely_linear_quantize_workspace_bytes(arr, 1, 2)
    # same workspace as a quantizer call on the two 4 x 8 tensors U and W
    qt = (L.QTensor * 2)(L.QTensor(FAKE, FAKE, 4, 8, FAKE, FAKE), L.QTensor(FAKE, FAKE, 4, 8, FAKE, FAKE))
    assert need == lib.ifq_quantize_workspace_bytes(qt, 2, 2) > 0
    call = lambda a, n=1, T=2, ws=FAKE, nb=need: lib.ifq_widely_linear_quantize_pack(a, n, T, ws, nb, None, None)
    assert call(None) == 1
    assert call(arr, n=0) == 9
    assert call((L.WlLayer * 17)(*([_wl()] * 17)), n=17) == 9   # U and W count twice: at most 16 layers
    assert call(arr, T=0) == 4 and call(arr, T=9) == 4
    assert call((L.WlLayer * 1)(_wl(codes_w=None))) == 1
    assert call((L.WlLayer * 1)(_wl(rows=7))) == 2
    assert call((L.WlLayer * 1)(_wl(cols=12))) == 2            # m = 6 is not a multiple of 4
    assert call((L.WlLayer * 1)(_wl(cols=4))) == 2
    assert call((L.WlLayer * 1)(_wl(U_im=FAKE + 4))) == 3
    assert call((L.WlLayer * 1)(_wl(scales_w=FAKE + 2))) == 3
    assert call(arr, ws=None) == 6 and call(arr, nb=need - 1) == 6
    assert call(arr, ws=FAKE + 8) == 3
    assert lib.ifq_widely_linear_quantize_workspace_bytes((L.WlLayer * 1)(_wl(cols=12)), 1, 2) == 0


def test_rotation_argument_errors():
    lib = Q.load()
    one = lambda **kw: (L.Layer * 1)(_layer(**kw))  # noqa: E731
    base = _layer()
    rot = (L.Layer * 1)(L.Layer(base.codes_u, base.scales_u, None, None, 64, 128, FAKE, FAKE, FAKE, FAKE,
                                FAKE, None))
    assert lib.ifq_gemv(rot, 1, 1, 1, FAKE, 1 << 30, None, None) == 1     # one of the two planes missing
    assert lib.ifq_gemm(rot, 1, 1, 128, None, None) == 1
    mis = (L.Layer * 1)(L.Layer(base.codes_u, base.scales_u, None, None, 64, 128, FAKE, FAKE, FAKE, FAKE,
                                FAKE + 4, FAKE))
    assert lib.ifq_gemv(mis, 1, 1, 1, FAKE, 1 << 30, None, None) == 3
    assert one() is not None


def test_dequantize_argument_errors():
    lib = Q.load()
    ok = (L.DqTensor * 1)(L.DqTensor(FAKE, FAKE, 8, 64, FAKE, FAKE))
    assert lib.ifq_dequantize(None, 1, 1, None) == 1
    assert lib.ifq_dequantize(ok, 0, 1, None) == 9
    assert lib.ifq_dequantize(ok, 1, 9, None) == 4
    assert lib.ifq_dequantize((L.DqTensor * 1)(L.DqTensor(FAKE, FAKE, 8, 66, FAKE, FAKE)), 1, 1, None) == 2
    assert lib.ifq_dequantize((L.DqTensor * 1)(L.DqTensor(FAKE, None, 8, 64, FAKE, FAKE)), 1, 1, None) == 1
    assert lib.ifq_dequantize((L.DqTensor * 1)(L.DqTensor(FAKE, FAKE, 8, 64, FAKE + 2, FAKE)), 1, 1, None) == 3
