"""GPU parity of ifq_dequantize (bf16 dequantized weights for training) with the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import workloads as W
import oracle as O
from ifq_testlib import DEV, gpu_quantize, run_gemv, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


def _bf16_as_f32(t):
    return (t.to(torch.int32).cpu().numpy().astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("shapes,T", [([(37, 100)], 1), ([(129, 256), (1, 4)], 3), ([(16, 320)], 8),
                                      ([(300, 1028), (64, 64), (5, 12)], 2)])
def test_dequantize_bit_exact(shapes, T):
    rng = np.random.default_rng(sum(n * k for n, k in shapes) + T)
    ws = [(to_dev((0.02 * rng.standard_normal((n, k))).astype(np.float32)),
           to_dev((0.02 * rng.standard_normal((n, k))).astype(np.float32))) for n, k in shapes]
    outs = gpu_quantize(ws, T)
    planes = [(torch.empty((n, k), dtype=torch.int16, device=DEV), torch.empty((n, k), dtype=torch.int16, device=DEV))
              for n, k in shapes]
    Q.ifq_dequantize([(c, s, pr, pi) for (c, s), (pr, pi) in zip(outs, planes)], T)
    torch.cuda.synchronize()
    for (c, s), (pr, pi) in zip(outs, planes):
        want_re, want_im = O.dequantize_bf16(c.cpu().numpy(), s.cpu().numpy())
        np.testing.assert_array_equal(_bf16_as_f32(pr).view(np.uint32), want_re.view(np.uint32))
        np.testing.assert_array_equal(_bf16_as_f32(pi).view(np.uint32), want_im.view(np.uint32))


def test_dequantize_block_layer_and_forward():
    """The llama7b gate layer (5504 x 2048, T = 2): bit-exact weights, and the training forward pass
    x W_hat^T (a plain bf16 matmul of the planes) agrees with the quantized product."""
    cfg = W.config("llama7b")
    spec = cfg.layers[4]
    rng = np.random.default_rng(9)
    wr = to_dev((0.02 * rng.standard_normal((spec.N, spec.K))).astype(np.float32))
    wi = to_dev((0.02 * rng.standard_normal((spec.N, spec.K))).astype(np.float32))
    (c, s), = gpu_quantize([(wr, wi)], 2)
    pr = torch.empty((spec.N, spec.K), dtype=torch.int16, device=DEV)
    pi = torch.empty_like(pr)
    Q.ifq_dequantize([(c, s, pr, pi)], 2)
    torch.cuda.synchronize()
    cn, sn = c.cpu().numpy(), s.cpu().numpy()
    want_re, want_im = O.dequantize_bf16(cn, sn)
    np.testing.assert_array_equal(_bf16_as_f32(pr).view(np.uint32), want_re.view(np.uint32))
    np.testing.assert_array_equal(_bf16_as_f32(pi).view(np.uint32), want_im.view(np.uint32))
    # training forward through the bf16 planes vs the quantized product (U only, B = 4 tokens)
    B = 4
    xr32 = rng.standard_normal((B, spec.K)).astype(np.float32)
    xi32 = rng.standard_normal((B, spec.K)).astype(np.float32)
    xr = torch.from_numpy(xr32).to(torch.bfloat16).to(DEV)
    xi = torch.from_numpy(xi32).to(torch.bfloat16).to(DEV)
    d = dict(codes_u=c, scales_u=s, codes_w=None, scales_w=None, N=spec.N, K=spec.K, x_re=xr, x_im=xi,
             y_re=torch.empty((B, spec.N), device=DEV), y_im=torch.empty((B, spec.N), device=DEV))
    run_gemv([d], 2, B)
    Wr = torch.from_numpy(want_re).to(DEV).double()
    Wi = torch.from_numpy(want_im).to(DEV).double()
    xrd, xid = xr.double(), xi.double()
    f_re = xrd @ Wr.T - xid @ Wi.T
    f_im = xrd @ Wi.T + xid @ Wr.T
    torch.cuda.synchronize()
    exact = O.dequantize(cn, sn)
    xrn, xin = xr.float().cpu().numpy(), xi.float().cpu().numpy()
    # |forward - product| <= bf16 rounding of W_hat (2^-8 relative) + the product's tolerance
    absw = np.abs(exact.real) + np.abs(exact.imag)
    bound = 2.0 ** -8 * (np.abs(xrn) + np.abs(xin)) @ absw.T + O.tolerance_bound(sn, None, xrn, xin)[:, None]
    err = np.abs((f_re.cpu().numpy() + 1j * f_im.cpu().numpy())
                 - (d["y_re"].cpu().numpy() + 1j * d["y_im"].cpu().numpy()))
    assert np.all(err <= bound), float(np.max(err / bound))
