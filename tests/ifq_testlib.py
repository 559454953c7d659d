"""Helpers shared by the GPU parity tests: run libifq on device tensors and
compare with the oracle under the acceptance rules:

  * conversion planes bit-exact;
  * stage-1 codes / packed bytes bit-exact;
  * later stages: the oracle's stage-t rule on residuals rebuilt from the GPU's
    own earlier codes and float32 scales; a mismatch is allowed only on an
    entry the oracle flags as near a decision boundary (counted, reported);
  * scales within 1e-6 relative of an independent oracle chain;
  * every output |y - y_ref| <= 1e-5 sum_{t,branch}(s_re + s_im) sum_j(|Re x_j| + |Im x_j|),
    with y_ref the complex128 product of the same codes, scales and bf16 x.
"""
import json
import os

import numpy as np
import torch

import bit_complex_quantized_b200 as Q
import oracle as O
from oracle import cref

DEV = "cuda"


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# ------------------------------------------------------------------ GPU calls
def gpu_convert(R):
    """R: numpy float32 [2n][2m] -> four device planes (U_re, U_im, W_re, W_im)."""
    Rd = to_dev(R)
    n, m = R.shape[0] // 2, R.shape[1] // 2
    planes = [torch.empty((n, m), dtype=torch.float32, device=DEV) for _ in range(4)]
    Q.ifq_widely_linear_from_real(Rd, *planes)
    return planes


def gpu_quantize(ws, T, dev_status=None):
    """ws: list of (w_re, w_im) device float32 [N][K].  Returns list of (codes [T][N][K/4], scales [T][2])."""
    outs = []
    for (wr, wi) in ws:
        N, K = wr.shape
        outs.append((torch.empty((T, N, K // 4), dtype=torch.uint8, device=DEV),
                     torch.empty((T, 2), dtype=torch.float32, device=DEV)))
    tensors = [(wr, wi, c, s) for (wr, wi), (c, s) in zip(ws, outs)]
    nbytes = Q.ifq_quantize_workspace_bytes(tensors, T)
    wsbuf = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    Q.ifq_quantize_pack(tensors, T, wsbuf, dev_status=dev_status)
    return outs


def run_gemv(descs, T, B, workspace=None, dev_status=None):
    """Decode product through the C ABI; allocates a zero-filled workspace when none is given."""
    if workspace is None:
        n = Q.ifq_gemv_workspace_bytes(descs, T, B)
        workspace = torch.zeros(max(n, 16), dtype=torch.uint8, device=DEV)
    Q.ifq_gemv(descs, T, B, workspace=workspace, dev_status=dev_status)
    return workspace


def layer_desc(cu, su, cw, sw, x_re, x_im, N, K, rows):
    y_re = torch.empty((rows, N), dtype=torch.float32, device=DEV)
    y_im = torch.empty((rows, N), dtype=torch.float32, device=DEV)
    return dict(codes_u=cu, scales_u=su, codes_w=cw, scales_w=sw, N=N, K=K, x_re=x_re, x_im=x_im,
                y_re=y_re, y_im=y_im)


# ------------------------------------------------------------------ checks
def check_convert(R, planes, rows=None):
    """Bit-exact conversion on all rows (or a row subset of the complex planes)."""
    n, m = R.shape[0] // 2, R.shape[1] // 2
    rows = np.arange(n) if rows is None else np.asarray(rows)
    Rsub = np.concatenate([R[rows], R[n + rows]], axis=0)
    want = O.widely_linear_planes_fp32(Rsub)
    for got, w in zip(planes, want):
        g = got[torch.as_tensor(rows, device=DEV)].cpu().numpy()
        np.testing.assert_array_equal(g.view(np.uint32), w.view(np.uint32))


def check_quantized(w_re, w_im, codes_gpu, scales_gpu, T, full_scales=True):
    """w_*: numpy float32 [N][K]; codes_gpu uint8 [T][N][K/4]; scales_gpu float32 [T][2] (numpy).
    Returns the number of near-boundary mismatches per stage."""
    N, K = w_re.shape
    flat_codes = codes_gpu.reshape(T, -1)
    mism = []
    for t in range(T):
        want, _, near = cref.stage(w_re, w_im, t, flat_codes[:t], scales_gpu[:t], want_near=(t > 0))
        got = flat_codes[t]
        if t == 0:
            np.testing.assert_array_equal(got, want, err_msg="stage-1 bytes differ")
            mism.append(0)
            continue
        diff_bytes = np.nonzero(got != want)[0]
        bad = 0
        for q in diff_bytes:
            for e in range(4):
                if ((got[q] >> (2 * e)) & 3) != ((want[q] >> (2 * e)) & 3):
                    assert near[4 * q + e], f"stage {t + 1}: code mismatch at entry {4 * q + e} off the boundary"
                    bad += 1
        mism.append(bad)
    if full_scales:
        _, s_ind = cref.quantize_tensor(w_re, w_im, T)
        rel = np.abs(scales_gpu.astype(np.float64) - s_ind.astype(np.float64))
        denom = np.maximum(np.abs(s_ind.astype(np.float64)), 1e-300)
        assert np.all((rel <= 1e-6 * denom) | (rel == 0)), (scales_gpu, s_ind)
    return mism


def check_product(y_re, y_im, cu, su, cw, sw, x_re, x_im, rows=None, slack=1.0):
    """y_*: numpy float32 [B][N] (GPU); codes/scales numpy; x_*: numpy float32 [B][K] (bf16 values).
    Compares the selected output columns (all if rows is None).  Returns max |err| / bound."""
    N = y_re.shape[1]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    ref = O.product_rows(cu, su, cw, sw, x_re, x_im, rows)          # [B][len(rows)]
    got = y_re[:, rows].astype(np.float64) + 1j * y_im[:, rows].astype(np.float64)
    bound = O.tolerance_bound(su, sw, x_re, x_im)[:, None] * slack
    err = np.abs(got - ref)
    worst = float(np.max(err / bound))
    assert np.all(err <= bound), f"max err/bound = {worst}"
    return worst


def record(name, payload):
    """Write a JSON record of a test's counts to $IFQ_RECORD_DIR/<name>.json when that variable is set
    (the near-boundary mismatch counts that the acceptance rules ask to report)."""
    d = os.environ.get("IFQ_RECORD_DIR")
    if not d:
        return
    os.makedirs(d, exist_ok=True)
    with open(os.path.join(d, name + ".json"), "w") as f:
        json.dump(payload, f, indent=1)


def tile_rows(N, rng, tile=64, group=16):
    """Output columns that cover every product tile: both edges of each `tile`-wide block of
    outputs and one random column inside each `group`-wide run of it (sorted, unique)."""
    cols = set()
    for t0 in range(0, N, tile):
        t1 = min(N, t0 + tile)
        cols.update((t0, t1 - 1))
        for g0 in range(t0, t1, group):
            cols.add(int(rng.integers(g0, min(t1, g0 + group))))
    return np.array(sorted(cols))


def sample_rows(N, k, rng):
    """First and last 16 rows plus k random rows (sorted, unique)."""
    base = list(range(min(16, N))) + list(range(max(0, N - 16), N))
    extra = rng.choice(N, size=min(k, N), replace=False).tolist()
    return np.array(sorted(set(base + extra)))
