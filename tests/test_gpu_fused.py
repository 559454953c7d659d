"""GPU parity of the fused conversion + stage-1 PhaseQuant call
(ifq_widely_linear_quantize_pack): every output equals the two-pass path
(ifq_widely_linear_from_real then ifq_quantize_pack) bit for bit, and the fp64
oracle directly on small layers."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import workloads as W
from ifq_testlib import DEV, check_convert, check_quantized, sample_rows, status_word, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


def _outputs(n, m, T):
    f = lambda: torch.empty((n, m), dtype=torch.float32, device=DEV)
    return dict(U_re=f(), U_im=f(), W_re=f(), W_im=f(),
                codes_u=torch.empty((T, n, m // 4), dtype=torch.uint8, device=DEV),
                scales_u=torch.empty((T, 2), dtype=torch.float32, device=DEV),
                codes_w=torch.empty((T, n, m // 4), dtype=torch.uint8, device=DEV),
                scales_w=torch.empty((T, 2), dtype=torch.float32, device=DEV))


def fused(Rs, T, status=None):
    layers = []
    for R in Rs:
        d = _outputs(R.shape[0] // 2, R.shape[1] // 2, T)
        d["R"] = R
        layers.append(d)
    nbytes = Q.ifq_widely_linear_quantize_workspace_bytes(layers, T)
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)  # no initial contents needed
    Q.ifq_widely_linear_quantize_pack(layers, T, ws, dev_status=status)
    return layers


def two_pass(Rs, T, status=None):
    outs, tensors = [], []
    for R in Rs:
        d = _outputs(R.shape[0] // 2, R.shape[1] // 2, T)
        Q.ifq_widely_linear_from_real(R, d["U_re"], d["U_im"], d["W_re"], d["W_im"])
        tensors += [(d["U_re"], d["U_im"], d["codes_u"], d["scales_u"]),
                    (d["W_re"], d["W_im"], d["codes_w"], d["scales_w"])]
        outs.append(d)
    nbytes = Q.ifq_quantize_workspace_bytes(tensors, T)
    Q.ifq_quantize_pack(tensors, T, torch.empty(nbytes, dtype=torch.uint8, device=DEV), dev_status=status)
    return outs


KEYS = ("U_re", "U_im", "W_re", "W_im", "codes_u", "codes_w", "scales_u", "scales_w")


def assert_same(a, b):
    for k in KEYS:
        x, y = a[k], b[k]
        if x.dtype == torch.float32:
            x, y = x.view(torch.int32), y.view(torch.int32)
        assert torch.equal(x, y), k


@pytest.mark.parametrize("n,m,T", [(1, 4, 1), (37, 100, 2), (129, 256, 3), (300, 1028, 2), (16, 4096, 8)])
def test_fused_equals_two_pass_and_oracle(n, m, T):
    rng = np.random.default_rng(n * 7919 + m)
    R = (0.02 * rng.standard_normal((2 * n, 2 * m))).astype(np.float32)
    Rd = to_dev(R)
    st1, st2 = status_word(), status_word()
    a = fused([Rd], T, st1)[0]
    b = two_pass([Rd], T, st2)[0]
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    assert_same(a, b)
    # and against the fp64 oracle directly
    check_convert(R, [a["U_re"], a["U_im"], a["W_re"], a["W_im"]])
    for pre in ("u", "w"):
        wr = a["U_re" if pre == "u" else "W_re"].cpu().numpy()
        wi = a["U_im" if pre == "u" else "W_im"].cpu().numpy()
        check_quantized(wr, wi, a["codes_" + pre].cpu().numpy(), a["scales_" + pre].cpu().numpy(), T)


def test_fused_block_of_seven_layers_equals_two_pass():
    """The LLaMA-2-7B-shaped block (seven real layers, 2 stages) in one grouped call."""
    cfg = W.config("llama7b")
    Rs = [to_dev(W.real_weight(cfg, i)) for i in range(len(cfg.layers))]
    a = fused(Rs, cfg.T)
    b = two_pass(Rs, cfg.T)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert_same(x, y)
    # sampled rows of the first layer against the oracle conversion
    rng = np.random.default_rng(3)
    R0 = W.real_weight(cfg, 0)
    check_convert(R0, [a[0]["U_re"], a[0]["U_im"], a[0]["W_re"], a[0]["W_im"]],
                  rows=sample_rows(cfg.layers[0].N, 64, rng))


def test_fused_nonfinite_and_overflow():
    """A NaN in R, and finite R entries whose sum overflows float32 in U: both
    paths code those entries 0 and flag them; all other outputs agree."""
    n, m, T = 8, 64, 2
    rng = np.random.default_rng(11)
    R = (0.02 * rng.standard_normal((2 * n, 2 * m))).astype(np.float32)
    R[1, 5] = np.nan                      # R11 -> U_re, W_re of (1, 5) are NaN
    R[2, 7] = R[n + 2, m + 7] = 3.0e38    # R11 + R22 overflows: U_re(2, 7) = +Inf
    Rd = to_dev(R)
    st1, st2 = status_word(), status_word()
    a = fused([Rd], T, st1)[0]
    b = two_pass([Rd], T, st2)[0]
    torch.cuda.synchronize()
    assert int(st1.item()) & Q.IFQ_DEV_NONFINITE
    assert int(st2.item()) & Q.IFQ_DEV_NONFINITE
    assert_same(a, b)
    cu = a["codes_u"].cpu().numpy()
    assert (cu[0, 1, 5 // 4] >> (2 * (5 % 4))) & 3 == 0
    assert (cu[0, 2, 7 // 4] >> (2 * (7 % 4))) & 3 == 0


def test_fused_argument_errors_on_the_device_path():
    R = torch.zeros((4, 12), dtype=torch.float32, device=DEV)   # cols % 8 != 0
    d = _outputs(2, 6, 1)
    d["R"] = R
    with pytest.raises(Q.IfqError):
        Q.ifq_widely_linear_quantize_pack([d], 1, torch.empty(4096, dtype=torch.uint8, device=DEV))
