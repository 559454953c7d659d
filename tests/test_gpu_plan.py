"""Prepared decode calls: ifq_gemv_prepare + ifq_gemv_run give the outputs of ifq_gemv bit for bit on
each path (integer tensor cores at B <= 2, bf16 mma.sync above, CUDA cores for a narrow width), also after new
activations are written into the same buffers between runs."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from ifq_testlib import DEV, gpu_quantize, layer_desc, run_gemv, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


@pytest.mark.parametrize("B,K", [(1, 2048), (2, 4160), (3, 1088), (8, 2048), (2, 100)])
def test_prepared_call_equals_ifq_gemv(B, K):
    rng = np.random.default_rng(B * 7 + K)
    N, T = 200, 2
    ws = [tuple((0.02 * rng.standard_normal((N, K))).astype(np.float32) for _ in range(2)) for _ in range(2)]
    (cu, su), (cw, sw) = gpu_quantize([(to_dev(a), to_dev(b)) for a, b in ws], T)
    x = [torch.from_numpy(rng.standard_normal((B, K)).astype(np.float32)).to(torch.bfloat16).to(DEV)
         for _ in range(2)]
    d_plan = layer_desc(cu, su, cw, sw, x[0], x[1], N, K, B)
    d_ref = layer_desc(cu, su, cw, sw, x[0], x[1], N, K, B)
    nws = max(16, Q.ifq_gemv_workspace_bytes([d_plan], T, B))
    wsp = torch.zeros(nws, dtype=torch.uint8, device=DEV)
    plan = Q.GemvPlan([d_plan], T, B, workspace=wsp)
    for rep in range(3):
        if rep:
            for t in x:
                t.copy_(torch.from_numpy(rng.standard_normal((B, K)).astype(np.float32)).to(torch.bfloat16))
        plan.run()
        run_gemv([d_ref], T, B)
        torch.cuda.synchronize()
        for part in ("y_re", "y_im"):
            assert torch.equal(d_plan[part].view(torch.int32), d_ref[part].view(torch.int32)), (rep, part)


@pytest.mark.parametrize("B,K", [(1, 2048), (2, 5504), (3, 1088)])
def test_activations_and_outputs_in_pinned_host_memory(B, K):
    """x read from and y written to pinned host memory by the kernels (unified addressing) give the
    outputs of device buffers bit for bit, directly and through a prepared call."""
    rng = np.random.default_rng(B * 11 + K)
    N, T = 300, 2
    ws = [tuple((0.02 * rng.standard_normal((N, K))).astype(np.float32) for _ in range(2)) for _ in range(2)]
    (cu, su), (cw, sw) = gpu_quantize([(to_dev(a), to_dev(b)) for a, b in ws], T)
    x = [torch.from_numpy(rng.standard_normal((B, K)).astype(np.float32)).to(torch.bfloat16) for _ in range(2)]
    d_dev = layer_desc(cu, su, cw, sw, x[0].to(DEV), x[1].to(DEV), N, K, B)
    d_host = dict(d_dev, x_re=x[0].pin_memory(), x_im=x[1].pin_memory(),
                  y_re=torch.empty((B, N), dtype=torch.float32).pin_memory(),
                  y_im=torch.empty((B, N), dtype=torch.float32).pin_memory())
    run_gemv([d_dev], T, B)
    run_gemv([d_host], T, B)
    torch.cuda.synchronize()
    for part in ("y_re", "y_im"):
        assert torch.equal(d_host[part].view(torch.int32), d_dev[part].cpu().view(torch.int32)), part
    d_host["y_re"].zero_()
    nws = max(16, Q.ifq_gemv_workspace_bytes([d_host], T, B))
    plan = Q.GemvPlan([d_host], T, B, workspace=torch.zeros(nws, dtype=torch.uint8, device=DEV))
    plan.run()
    torch.cuda.synchronize()
    assert torch.equal(d_host["y_re"].view(torch.int32), d_dev["y_re"].cpu().view(torch.int32))
