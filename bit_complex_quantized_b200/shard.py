"""Row split of the quantizer and the decode product across GPUs (one process per GPU).

The product shards by output rows with no exchange: each GPU holds the codes of
its rows ([T][rows][K/4]) and writes those outputs.  The quantizer's scales are
means over the whole tensor ("Fairy2i write-up" §3.2), so each stage of a
row-split quantization exchanges the stage's tile partials (32 bytes per 4096
weights) before the next stage; with shard boundaries on whole tiles, codes
and scales equal those of the whole tensor quantized on one GPU bit for bit.

Host logic only: the arithmetic runs in libifq (ifq_quantize_stage,
ifq_quantize_finish, ifq_gemv); the exchange is a torch.distributed
all-gather (NCCL on GPUs).
"""
import math

import torch

from . import _lib as L

TILE_WEIGHTS = 4096   # complex weights per quantizer tile
PARTIAL_BYTES = 32    # one tile partial: float64 S_re, float64 S_im, uint64 C_re, padding


def row_shards(N, K, world):
    """Rows [n0, n1) of each of `world` ranks: nearly equal, every boundary a multiple of the rows
    whose K weights fill whole quantizer tiles, so that the shards' tiles are the tensor's tiles."""
    if N < 1 or K < 4 or K % 4 or world < 1:
        raise ValueError("bad shape or world size")
    step = TILE_WEIGHTS // math.gcd(K, TILE_WEIGHTS)
    steps = -(-N // step)
    b = [min(N, step * (steps * r // world)) for r in range(world + 1)]
    return [(b[r], b[r + 1]) for r in range(world)]


def tiles(rows, K):
    """Quantizer tiles of a [rows][K] tensor (the last one may be partial)."""
    return -(-rows * K // TILE_WEIGHTS)


def all_gather_bytes(local, sizes, group=None):
    """Every rank's byte buffer (rank r holds sizes[r] bytes), in rank order; an all-gather of
    equal-sized padded buffers."""
    import torch.distributed as dist
    m = max(sizes)
    buf = torch.zeros(m, dtype=torch.uint8, device=local.device)
    buf[:local.numel()] = local
    outs = [torch.empty_like(buf) for _ in sizes]
    dist.all_gather(outs, buf, group=group)
    return [o[:s] for o, s in zip(outs, sizes)]


def quantize_row_split(shards, T, rank, world, stage=None, finish=None, gather=None, dev_status=None):
    """T-stage PhaseQuant of tensors whose rows are split across `world` ranks.

    shards: this rank's part of each tensor, dicts with w_re, w_im ([rows][K] float32), codes
    ([T][rows][K/4] uint8), scales ([T][2] float32) and N (the whole tensor's rows); every rank's
    rows are those of row_shards(N, K, world)[rank].
    Per stage t: stage(tensors, t, partials) writes the shard's codes and tile partials;
    gather(local_bytes, sizes) returns every rank's partials in rank order; finish(parts, t)
    writes the scales of whole tensors from their gathered partials.  The defaults are the
    library's calls and an all-gather over the default process group."""
    stage = stage or (lambda ts, t, part: L.ifq_quantize_stage(ts, t, part, dev_status=dev_status))
    finish = finish or L.ifq_quantize_finish
    gather = gather or all_gather_bytes
    tensors = [(s["w_re"], s["w_im"], s["codes"], s["scales"]) for s in shards]
    K = [s["w_re"].shape[1] for s in shards]
    bounds = [row_shards(s["N"], k, world) for s, k in zip(shards, K)]
    for s, k, bd in zip(shards, K, bounds):
        n0, n1 = bd[rank]
        if s["w_re"].shape[0] != n1 - n0:
            raise ValueError("a shard's rows differ from row_shards() of its tensor")
    # bytes of each tensor's partials on each rank
    per = [[tiles(b[r][1] - b[r][0], k) * PARTIAL_BYTES for r in range(world)] for b, k in zip(bounds, K)]
    sizes = [sum(p[r] for p in per) for r in range(world)]
    dev = shards[0]["w_re"].device
    local = torch.empty(max(sizes[rank], 16), dtype=torch.uint8, device=dev)
    for t in range(1, T + 1):
        stage(tensors, t, local)
        got = gather(local[:sizes[rank]], sizes)
        parts = []
        for i, (s, k) in enumerate(zip(shards, K)):
            pieces = []
            for r in range(world):
                off = sum(per[j][r] for j in range(i))
                pieces.append(got[r][off:off + per[i][r]])
            whole = torch.cat(pieces) if len(pieces) > 1 else pieces[0].clone()
            parts.append((whole, s["N"], k, s["scales"]))
        finish(parts, t)
    return shards


def gather_rows(y_local, N, rank, world, K, group=None):
    """The whole output [rows][N] from every rank's [rows][n1 - n0] slice of a row-split product
    (an all-gather; not needed when each GPU consumes its own rows)."""
    import torch.distributed as dist
    bounds = row_shards(N, K, world)
    width = max(b[1] - b[0] for b in bounds)
    pad = torch.zeros((y_local.shape[0], width), dtype=y_local.dtype, device=y_local.device)
    pad[:, :y_local.shape[1]] = y_local
    outs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(outs, pad, group=group)
    return torch.cat([o[:, :b[1] - b[0]] for o, b in zip(outs, bounds)], dim=1)
