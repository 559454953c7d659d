"""GPU parity of the product epilogue's complex rotation (complex rotary position
code of the q / k projections) and of the real-part attention score fed by the
planar outputs, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import workloads as W
import oracle as O
from ifq_testlib import DEV, gpu_quantize, layer_desc, run_gemv, status_word, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


def _layer(rng, N, K, T, conj=True):
    ws = [(0.02 * rng.standard_normal((N, K))).astype(np.float32) for _ in range(2)]
    wws = [(0.03 * rng.standard_normal((N, K))).astype(np.float32) for _ in range(2)]
    tens = [(to_dev(ws[0]), to_dev(ws[1]))] + ([(to_dev(wws[0]), to_dev(wws[1]))] if conj else [])
    outs = gpu_quantize(tens, T)
    torch.cuda.synchronize()
    host = [(c.cpu().numpy(), s.cpu().numpy()) for c, s in outs]
    cu, su = outs[0]
    cw, sw = outs[1] if conj else (None, None)
    return (cu, su, cw, sw), host


def _x(rng, rows, K):
    xr = torch.from_numpy(rng.standard_normal((rows, K)).astype(np.float32)).to(torch.bfloat16)
    xi = torch.from_numpy(rng.standard_normal((rows, K)).astype(np.float32)).to(torch.bfloat16)
    return xr, xi, W.bf16_to_f32_numpy(xr), W.bf16_to_f32_numpy(xi)


def _rot(rng, rows, N, unit):
    if unit:  # e^{i theta}, as a rotary code passes
        th = rng.uniform(-np.pi, np.pi, (rows, N))
        return np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    return (rng.standard_normal((rows, N)).astype(np.float32), rng.standard_normal((rows, N)).astype(np.float32))


def check_rotated(d, host, xrn, xin, rr, ri):
    """|y - rot y_ref| <= |rot| (bound + 2^-22 |y_ref|): the product's bound scaled by the rotation,
    plus the float32 rounding of the complex multiply."""
    (cun, sun), rest = host[0], host[1:]
    cwn, swn = rest[0] if rest else (None, None)
    ref = O.product_rows(cun, sun, cwn, swn, xrn, xin)
    want = O.rotate_outputs(ref, rr, ri)
    got = d["y_re"].cpu().numpy().astype(np.float64) + 1j * d["y_im"].cpu().numpy().astype(np.float64)
    mod = np.abs(rr.astype(np.float64) + 1j * ri.astype(np.float64))
    bound = mod * (O.tolerance_bound(sun, swn, xrn, xin)[:, None] + 2.0 ** -22 * np.abs(ref))
    err = np.abs(got - want)
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("N,K,T,unit", [(256, 4096, 2, True), (77, 2048, 2, False), (40, 5504, 3, True)])
def test_gemv_b1_rotation(N, K, T, unit):
    rng = np.random.default_rng(N + K)
    (cu, su, cw, sw), host = _layer(rng, N, K, T)
    xr, xi, xrn, xin = _x(rng, 1, K)
    rr, ri = _rot(rng, 1, N, unit)
    d = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, 1)
    d["rot_re"], d["rot_im"] = to_dev(rr), to_dev(ri)
    st = status_word()
    run_gemv([d], T, 1, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_rotated(d, host, xrn, xin, rr, ri)


@pytest.mark.parametrize("B", [2, 5, 16])
def test_gemv_batched_rotation(B):
    rng = np.random.default_rng(100 + B)
    N, K, T = 131, 1024, 2
    (cu, su, cw, sw), host = _layer(rng, N, K, T)
    xr, xi, xrn, xin = _x(rng, B, K)
    rr, ri = _rot(rng, B, N, B != 5)
    d = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, B)
    d["rot_re"], d["rot_im"] = to_dev(rr), to_dev(ri)
    run_gemv([d], T, B)
    torch.cuda.synchronize()
    check_rotated(d, host, xrn, xin, rr, ri)


@pytest.mark.parametrize("N,M", [(128, 131), (37, 128), (200, 300)])
def test_gemm_rotation(N, M):
    rng = np.random.default_rng(N * M)
    K, T = 1024, 2
    (cu, su, cw, sw), host = _layer(rng, N, K, T)
    xr, xi, xrn, xin = _x(rng, M, K)
    rr, ri = _rot(rng, M, N, N != 37)
    d = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, M)
    d["rot_re"], d["rot_im"] = to_dev(rr), to_dev(ri)
    st = status_word()
    Q.ifq_gemm([d], T, M, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_rotated(d, host, xrn, xin, rr, ri)


def test_rotation_is_identity_when_absent_and_one():
    """rot = 1 gives exactly the unrotated product (the multiply by 1 + 0i is exact)."""
    rng = np.random.default_rng(7)
    N, K, T = 96, 2048, 2
    (cu, su, cw, sw), host = _layer(rng, N, K, T)
    xr, xi, _, _ = _x(rng, 1, K)
    a = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, 1)
    b = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, 1)
    b["rot_re"] = torch.ones((1, N), device=DEV)
    b["rot_im"] = torch.zeros((1, N), device=DEV)
    run_gemv([a, b], T, 1)
    torch.cuda.synchronize()
    assert torch.equal(a["y_re"], b["y_re"]) and torch.equal(a["y_im"], b["y_im"])


def test_real_part_score_from_planar_outputs():
    """q from the decode product (one token, rotated at its position) and k from the prefill
    product (M tokens, each rotated at its own position); the scores Re(q^T conj(k_m)) come from a
    plain real matrix product of the stacked [re, im] planes and match the oracle's."""
    rng = np.random.default_rng(31)
    N, K, T, M = 128, 2048, 2, 150
    (qu, qsu, qw, qsw), qhost = _layer(rng, N, K, T)
    (ku, ksu, kw, ksw), khost = _layer(rng, N, K, T)
    omega = 10000.0 ** (-np.arange(N) / N)
    pos_q, pos_k = M + 3, np.arange(M)
    rq = (np.cos(pos_q * omega)[None, :].astype(np.float32), np.sin(pos_q * omega)[None, :].astype(np.float32))
    rk = (np.cos(pos_k[:, None] * omega[None, :]).astype(np.float32),
          np.sin(pos_k[:, None] * omega[None, :]).astype(np.float32))
    xq_r, xq_i, xq_rn, xq_in = _x(rng, 1, K)
    xk_r, xk_i, xk_rn, xk_in = _x(rng, M, K)
    dq = layer_desc(qu, qsu, qw, qsw, xq_r.to(DEV), xq_i.to(DEV), N, K, 1)
    dq["rot_re"], dq["rot_im"] = to_dev(rq[0]), to_dev(rq[1])
    dk = layer_desc(ku, ksu, kw, ksw, xk_r.to(DEV), xk_i.to(DEV), N, K, M)
    dk["rot_re"], dk["rot_im"] = to_dev(rk[0]), to_dev(rk[1])
    run_gemv([dq], T, 1)
    Q.ifq_gemm([dk], T, M)
    qs = torch.cat([dq["y_re"], dq["y_im"]], dim=1).double()       # [1][2N]
    ks = torch.cat([dk["y_re"], dk["y_im"]], dim=1).double()       # [M][2N]
    s_gpu = (ks @ qs.T)[:, 0].cpu().numpy()
    torch.cuda.synchronize()
    q_ref = O.rotate_outputs(O.product_rows(*qhost[0], *qhost[1], xq_rn, xq_in), *rq)[0]
    k_ref = O.rotate_outputs(O.product_rows(*khost[0], *khost[1], xk_rn, xk_in), *rk)
    s_ref = O.score(q_ref[None, :], k_ref)
    # |d score| <= sum_n |q_n| e_k + |k_n| e_q + e_q e_k, e = the outputs' error bounds
    e_q = O.tolerance_bound(qhost[0][1], qhost[1][1], xq_rn, xq_in)[0] + 2.0 ** -22 * np.abs(q_ref)
    e_k = O.tolerance_bound(khost[0][1], khost[1][1], xk_rn, xk_in)[:, None] + 2.0 ** -22 * np.abs(k_ref)
    bound = np.sum(np.abs(q_ref)[None, :] * e_k + np.abs(k_ref) * e_q[None, :] + e_q[None, :] * e_k, axis=1)
    assert np.all(np.abs(s_gpu - s_ref) <= bound), float(np.max(np.abs(s_gpu - s_ref) / bound))
