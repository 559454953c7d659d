"""Row split through the library on one GPU: two shards of each tensor quantized stage by stage with
ifq_quantize_stage, their tile partials joined in row order (what the all-gather of a multi-GPU run
delivers) and finished with ifq_quantize_finish.  Codes and scales must equal ifq_quantize_pack on
the whole tensors bit for bit, and the decode product of each shard's rows must equal the rows of
the whole-tensor product: bit for bit on the bf16 path (B >= 3), whose outputs depend only on their
own row's codes, and within float rounding on the integer path (B <= 2)."""
import numpy as np
import pytest
import torch

import bit_complex_quantized_b200 as Q
from bit_complex_quantized_b200 import shard
from ifq_testlib import DEV, layer_desc, run_gemv

pytestmark = pytest.mark.gpu

T = 3
SHAPES = [(1000, 2048), (300, 1088)]   # rows, K


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Q.load()


def _planes(rng, n, k):
    return [torch.from_numpy((0.02 * rng.standard_normal((n, k))).astype(np.float32)).to(DEV) for _ in range(2)]


def test_row_split_quantize_and_gemv_equal_whole_tensor():
    rng = np.random.default_rng(31)
    ws = [_planes(rng, n, k) for n, k in SHAPES for _ in range(2)]   # U and W of each shape
    shapes = [s for s in SHAPES for _ in range(2)]
    whole = [(wr, wi, torch.empty((T, n, k // 4), dtype=torch.uint8, device=DEV),
              torch.empty((T, 2), dtype=torch.float32, device=DEV)) for (wr, wi), (n, k) in zip(ws, shapes)]
    wsb = torch.empty(Q.ifq_quantize_workspace_bytes(whole, T), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Q.ifq_quantize_pack(whole, T, wsb, dev_status=st)

    world = 2
    bounds = [shard.row_shards(n, k, world) for n, k in shapes]
    shards = []
    for r in range(world):
        mine = []
        for (wr, wi), (n, k), b in zip(ws, shapes, bounds):
            n0, n1 = b[r]
            mine.append((wr[n0:n1].contiguous(), wi[n0:n1].contiguous(),
                         torch.empty((T, n1 - n0, k // 4), dtype=torch.uint8, device=DEV),
                         torch.empty((T, 2), dtype=torch.float32, device=DEV)))
        shards.append(mine)
    per = [[shard.tiles(b[r][1] - b[r][0], k) * shard.PARTIAL_BYTES for r in range(world)]
           for b, (_, k) in zip(bounds, shapes)]
    for t in range(1, T + 1):
        parts = []
        for r in range(world):
            buf = torch.empty(Q.ifq_quantize_workspace_bytes(shards[r], t), dtype=torch.uint8, device=DEV)
            Q.ifq_quantize_stage(shards[r], t, buf, dev_status=st)
            parts.append(buf)
        joined = []
        for i in range(len(shapes)):
            pieces = [parts[r][sum(per[j][r] for j in range(i)):][:per[i][r]] for r in range(world)]
            joined.append(torch.cat(pieces))
        for r in range(world):
            Q.ifq_quantize_finish([(joined[i], shapes[i][0], shapes[i][1], shards[r][i][3])
                                   for i in range(len(shapes))], t)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i in range(len(shapes)):
        codes = torch.cat([shards[r][i][2] for r in range(world)], dim=1)
        assert torch.equal(codes, whole[i][2]), f"tensor {i}: codes differ"
        for r in range(world):
            assert torch.equal(shards[r][i][3].view(torch.int32), whole[i][3].view(torch.int32)), f"tensor {i}: scales"

    # decode product of each shard's rows (U and W of the first shape) against the whole tensor
    n, k = SHAPES[0]
    for B in (1, 3, 8):
        xr = torch.from_numpy(rng.standard_normal((B, k)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        xi = torch.from_numpy(rng.standard_normal((B, k)).astype(np.float32)).to(torch.bfloat16).to(DEV)
        d = layer_desc(whole[0][2], whole[0][3], whole[1][2], whole[1][3], xr, xi, n, k, B)
        run_gemv([d], T, B)
        ys = []
        for r in range(world):
            n0, n1 = bounds[0][r]
            dr = layer_desc(shards[r][0][2], shards[r][0][3], shards[r][1][2], shards[r][1][3], xr, xi, n1 - n0, k, B)
            run_gemv([dr], T, B)
            ys.append(dr)
        torch.cuda.synchronize()
        for part in ("y_re", "y_im"):
            got = torch.cat([y[part] for y in ys], dim=1)
            if B >= 3:
                # bf16 path: each output is summed over its own row's codes in a fixed order
                assert torch.equal(got.view(torch.int32), d[part].view(torch.int32)), f"B = {B}: {part} differs"
            else:
                # integer path: the exact int32 sums are merged in float per piece, and the pieces of a
                # row follow the warps' shares of the whole call, which differ between the shard and
                # the whole tensor; the two differ by float rounding only, far inside the product bound
                sc = sum(float(whole[i][3][:, 0].sum() + whole[i][3][:, 1].sum()) for i in (0, 1))
                bound = 1e-6 * sc * (xr.float().abs() + xi.float().abs()).sum(dim=1, keepdim=True)
                assert bool(((got - d[part]).abs() <= bound).all()), f"B = {B}: {part} differs beyond rounding"
