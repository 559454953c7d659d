"""ifq_quantize_pack_static: the allocation-free form of ifq_quantize_pack,
whose scratch is a fixed array inside libifq.  Its results must equal those of
the workspace entry point bit for bit (same kernels, same reduction order), on
two calls in a row; calls beyond the fixed scratch are refused on the host.
This file is collected last so that the GPU test also runs after all others."""
import numpy as np
import pytest

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import _lib as L

FAKE = 0x10000  # non-null, 16-byte aligned, never dereferenced by validation


def _static(tensors, T):
    arr = (L.QTensor * len(tensors))(*tensors)
    return Q.load().ifq_quantize_pack_static(arr, len(tensors), T, None, None)


def test_static_scratch_limit_is_checked_on_the_host():
    lib = Q.load()
    big = L.QTensor(FAKE, FAKE, 65536, 65536, FAKE, FAKE)           # 2^32 weights: 32 MiB of scratch
    arr = (L.QTensor * 1)(big)
    assert lib.ifq_quantize_workspace_bytes(arr, 1, 2) > Q.IFQ_QUANT_STATIC_SCRATCH_BYTES
    assert _static([big], 2) == 10
    assert Q.ifq_status_string(10)
    # the limit itself: 262144 x 1024 complex weights need exactly the fixed scratch (32 bytes per
    # 4096 weights); checked on the sizes alone, since a call with these fake pointers would launch
    at = L.QTensor(FAKE, FAKE, 262144, 1024, FAKE, FAKE)
    assert lib.ifq_quantize_workspace_bytes((L.QTensor * 1)(at), 1, 1) == Q.IFQ_QUANT_STATIC_SCRATCH_BYTES
    # one row more is refused before anything is launched
    edge = L.QTensor(FAKE, FAKE, 262144 + 1, 1024, FAKE, FAKE)
    assert lib.ifq_quantize_workspace_bytes((L.QTensor * 1)(edge), 1, 1) > Q.IFQ_QUANT_STATIC_SCRATCH_BYTES
    assert _static([edge], 1) == 10
    # the usual argument errors come first, as for ifq_quantize_pack
    assert _static([L.QTensor(FAKE, None, 64, 128, FAKE, FAKE)], 1) == 1
    assert _static([L.QTensor(FAKE, FAKE, 64, 126, FAKE, FAKE)], 1) == 2
    assert _static([L.QTensor(FAKE + 8, FAKE, 64, 128, FAKE, FAKE)], 1) == 3
    assert _static([L.QTensor(FAKE, FAKE, 64, 128, FAKE, FAKE)], 9) == 4
    assert Q.load().ifq_quantize_pack_static(None, 1, 1, None, None) == 1


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point():
    import torch
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    rng = np.random.default_rng(7)
    T = 3
    shapes = [(96, 256), (300, 1088), (1, 4), (517, 2052)]
    planes = []
    for n, k in shapes:
        w = rng.standard_normal((2, n, k)).astype(np.float32) * 0.02
        planes.append((torch.from_numpy(w[0]).to(dev), torch.from_numpy(w[1]).to(dev)))

    def outputs():
        return [(torch.full((T, n, k // 4), 0xA5, dtype=torch.uint8, device=dev),
                 torch.full((T, 2), float("nan"), dtype=torch.float32, device=dev)) for n, k in shapes]

    ref = outputs()
    tensors = [(wr, wi, c, s) for (wr, wi), (c, s) in zip(planes, ref)]
    ws = torch.empty(Q.ifq_quantize_workspace_bytes(tensors, T), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    Q.ifq_quantize_pack(tensors, T, ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for call in range(2):
        got = outputs()
        tensors = [(wr, wi, c, s) for (wr, wi), (c, s) in zip(planes, got)]
        Q.ifq_quantize_pack_static(tensors, T, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status"
        for (rc, rs), (gc, gs) in zip(ref, got):
            assert torch.equal(rc, gc), f"call {call}: codes differ"
            assert torch.equal(rs.view(torch.int32), gs.view(torch.int32)), f"call {call}: scales differ"
