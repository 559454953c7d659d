"""Row split of the quantizer across ranks (host logic on CPU, two gloo ranks on 127.0.0.1).

bit_complex_quantized_b200.shard splits each tensor's rows on quantizer-tile boundaries, runs one
stage at a time on every rank's rows, gathers the stage's tile partials and finishes the whole
tensor's scales from them.  Here the stage and finish steps are stand-ins written with the oracle
(the library's kernels need a GPU; tests/test_gpu_shard.py runs those): per-tile fp64 class sums of
the oracle's residuals and codes, reduced tile by tile.  The split's codes and scales must equal
the single-rank run of the same steps bit for bit, for T = 3 and two tensors of different widths."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PART = np.dtype([("s_re", "<f8"), ("s_im", "<f8"), ("c_re", "<u8"), ("pad", "<u8")])
SHAPES = [(300, 96), (1100, 200)]   # rows, K: shard boundaries at 128 and 512 rows
T = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def np_stage(tensors, t, partials):
    """Stand-in for ifq_quantize_stage: the oracle's rule on the residual of stages < t, and one
    partial (class sums, class-0 count) per 4096-weight tile of the rows given."""
    import oracle as O
    from bit_complex_quantized_b200.shard import PARTIAL_BYTES, TILE_WEIGHTS, tiles
    off = 0
    for wr, wi, codes, sc in tensors:
        n, K = wr.shape
        prev = [O.unpack_codes(codes[u].numpy(), K) for u in range(t - 1)]
        a, b = O.residual_after(wr.numpy(), wi.numpy(), prev, [tuple(sc[u].numpy()) for u in range(t - 1)])
        k = O.phase_code(a, b)
        codes[t - 1] = torch.from_numpy(O.pack_codes(k))
        af, bf, kf = np.abs(a).ravel(), np.abs(b).ravel(), k.ravel()
        nt = tiles(n, K)
        rec = np.zeros(nt, dtype=PART)
        for i in range(nt):
            sl = slice(i * TILE_WEIGHTS, (i + 1) * TILE_WEIGHTS)
            c0 = (kf[sl] & 1) == 0
            rec["s_re"][i] = np.sum(af[sl][c0], dtype=np.float64)
            rec["s_im"][i] = np.sum(bf[sl][~c0], dtype=np.float64)
            rec["c_re"][i] = np.count_nonzero(c0)
        partials[off:off + nt * PARTIAL_BYTES] = torch.from_numpy(rec.view(np.uint8).copy())
        off += nt * PARTIAL_BYTES


def np_finish(parts, t):
    """Stand-in for ifq_quantize_finish: tile partials of a whole tensor added in tile order."""
    from oracle.phasequant import scales_from_sums
    for whole, N, K, sc in parts:
        rec = whole.numpy().view(PART)
        s_re = s_im = 0.0
        c_re = 0
        for r in rec:
            s_re += float(r["s_re"])
            s_im += float(r["s_im"])
            c_re += int(r["c_re"])
        sc[t - 1] = torch.tensor(scales_from_sums(s_re, c_re, s_im, N * K - c_re))


def _weights():
    rng = np.random.default_rng(21)
    return [(0.02 * rng.standard_normal((n, k))).astype(np.float32) for n, k in SHAPES for _ in range(2)]


def _shards(rank, world):
    from bit_complex_quantized_b200.shard import row_shards
    w = _weights()
    out = []
    for i, (n, k) in enumerate(SHAPES):
        n0, n1 = row_shards(n, k, world)[rank]
        out.append(dict(w_re=torch.from_numpy(w[2 * i][n0:n1].copy()), w_im=torch.from_numpy(w[2 * i + 1][n0:n1].copy()),
                        codes=torch.zeros((T, n1 - n0, k // 4), dtype=torch.uint8),
                        scales=torch.zeros((T, 2), dtype=torch.float32), N=n))
    return out


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from bit_complex_quantized_b200 import shard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = _shards(rank, world)
        shard.quantize_row_split(mine, T, rank, world, stage=np_stage, finish=np_finish)
        q.put((rank, [(s["codes"].numpy(), s["scales"].numpy()) for s in mine]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_row_shards_fall_on_tiles_and_cover_the_rows():
    from bit_complex_quantized_b200.shard import TILE_WEIGHTS, row_shards
    for N, K, world in [(300, 96, 2), (1100, 200, 2), (5504, 2048, 8), (37, 4, 3), (1, 64, 4), (4096, 5504, 8)]:
        b = row_shards(N, K, world)
        assert b[0][0] == 0 and b[-1][1] == N
        for (a0, a1), (c0, _) in zip(b, b[1:]):
            assert a1 == c0 and a0 <= a1
            assert (a1 * K) % TILE_WEIGHTS == 0 or a1 == N


def test_row_split_quantization_equals_single_rank_bit_for_bit():
    from bit_complex_quantized_b200 import shard
    whole = _shards(0, 1)
    shard.quantize_row_split(whole, T, 0, 1, stage=np_stage, finish=np_finish, gather=lambda local, sizes: [local])
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for i, s in enumerate(whole):
        codes = np.concatenate([res[r][i][0] for r in range(2)], axis=1)
        np.testing.assert_array_equal(codes, s["codes"].numpy())
        for r in range(2):
            np.testing.assert_array_equal(res[r][i][1].view(np.uint32), s["scales"].numpy().view(np.uint32))
    # the stand-ins are the oracle's definition: the whole-tensor scales match its quantizer
    import oracle as O
    w = _weights()
    for i, s in enumerate(whole):
        _, sc, _ = O.quantize_tensor(w[2 * i], w[2 * i + 1], T)
        np.testing.assert_allclose(s["scales"].numpy(), sc, rtol=1e-6, atol=0)


def test_misaligned_shards_are_refused():
    from bit_complex_quantized_b200 import shard
    s = _shards(0, 2)
    s[0]["w_re"] = s[0]["w_re"][:-1]
    with pytest.raises(ValueError):
        shard.quantize_row_split(s, T, 0, 2, stage=np_stage, finish=np_finish, gather=lambda l, z: [l, l])


def _gather_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from bit_complex_quantized_b200.shard import gather_rows, row_shards
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, K, rows = 1100, 200, 3
        full = torch.arange(rows * N, dtype=torch.float32).reshape(rows, N)
        n0, n1 = row_shards(N, K, world)[rank]
        got = gather_rows(full[:, n0:n1].contiguous(), N, rank, world, K)
        q.put((rank, bool(torch.equal(got, full))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gather_rows_reassembles_the_outputs_of_a_row_split():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res == {0: True, 1: True}
