"""ctypes wrapper of oracle/phasequant_ref.c (test infrastructure only).

Builds oracle/_build/libphasequant_ref.so with gcc on first use.  The C code
restates the same per-element definitions as oracle/phasequant.py; its pins
are in tests/test_oracle_pins.py (agreement with the NumPy oracle and the
hand-worked fixtures).
"""
import ctypes
import os
import subprocess

import numpy as np

from .phasequant import scales_from_sums

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "phasequant_ref.c")
_LIB = os.path.join(_HERE, "_build", "libphasequant_ref.so")
_lib = None


def build():
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", _SRC, "-o", _LIB,
                    "-lm"], check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        vp = ctypes.c_void_p
        _lib.ref_stage.restype = None
        _lib.ref_stage.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int, vp, vp, vp, vp, vp]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def stage(w_re, w_im, t, prev_codes, prev_scales, want_near=False):
    """Codes (packed, [n/4] flat) and sums of stage t given earlier packed codes [t][n/4] and scales [t][2]."""
    w_re = np.ascontiguousarray(w_re, dtype=np.float32).ravel()
    w_im = np.ascontiguousarray(w_im, dtype=np.float32).ravel()
    n = w_re.size
    prev = np.ascontiguousarray(prev_codes, dtype=np.uint8).reshape(-1) if t > 0 else np.zeros(1, np.uint8)
    ps = np.ascontiguousarray(prev_scales, dtype=np.float32).reshape(-1) if t > 0 else np.zeros(2, np.float32)
    out = np.empty(n // 4, np.uint8)
    sums = np.zeros(4, np.float64)
    near = np.empty(n, np.uint8) if want_near else None
    _load().ref_stage(_p(w_re), _p(w_im), n, t, _p(prev), _p(ps), _p(out), _p(sums), _p(near))
    return out, (float(sums[0]), int(sums[1]), float(sums[2]), int(sums[3])), near


def quantize_tensor(w_re, w_im, T):
    """T stages; returns packed codes [T][N][K/4] and fp32 scales [T][2] (fp64 means rounded)."""
    N, K = np.shape(w_re)
    codes = np.zeros((T, N * K // 4), np.uint8)
    scales = np.zeros((T, 2), np.float32)
    for t in range(T):
        codes[t], sums, _ = stage(w_re, w_im, t, codes[:t], scales[:t])
        scales[t] = scales_from_sums(*sums)
    return codes.reshape(T, N, K // 4), scales
