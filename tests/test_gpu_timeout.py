"""Failure detection of the tensor-core GEMM without a GPU fault: a wait limit of 1 ns makes the first
pipeline wait that is not already complete give up.  The call must return, report IFQ_DEV_TIMEOUT in
the device status word, drain its copies and MMAs and free its TMEM -- the next normal call on the same
context must then pass parity."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import workloads as W
from ifq_testlib import DEV, check_product, gpu_quantize, layer_desc, status_word, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


def test_gemm_wait_that_runs_out_sets_timeout_and_the_next_call_is_correct():
    rng = np.random.default_rng(12)
    N, K, T, M = 192, 512, 2, 128
    ws = [tuple((0.02 * rng.standard_normal((N, K))).astype(np.float32) for _ in range(2)) for _ in range(2)]
    outs = gpu_quantize([(to_dev(a), to_dev(b)) for a, b in ws], T)
    (cu, su), (cw, sw) = outs
    xr = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    xi = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    d = layer_desc(cu, su, cw, sw, xr.to(DEV), xi.to(DEV), N, K, M)
    for rep in range(2):
        st = status_word()
        Q.ifq_gemm_wait_limit([d], T, M, 1, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) & Q.IFQ_DEV_TIMEOUT, f"call {rep}: the 1 ns limit did not run out"
    st = status_word()
    Q.ifq_gemm([d], T, M, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    host = [(c.cpu().numpy(), s.cpu().numpy()) for c, s in outs]
    check_product(d["y_re"].cpu().numpy(), d["y_im"].cpu().numpy(), host[0][0], host[0][1], host[1][0], host[1][1],
                  W.bf16_to_f32_numpy(xr), W.bf16_to_f32_numpy(xi))
