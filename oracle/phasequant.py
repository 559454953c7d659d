"""fp64 reference for the widely-linear transform, PhaseQuant and the quantized product.

TEST INFRASTRUCTURE ONLY: the CUDA library never imports, links or runs this
file.  Every routine is the plain definition from the pages, in float64 NumPy,
with no blocking, fusion or reordering beyond what the definition states.

Notation (all planar): a complex tensor is N x K (N outputs, K inputs);
code k in {0,1,2,3} stands for the codebook entry [1, i, -1, -i][k]; a stage
t stores codes plus one scale pair (s_re, s_im) per tensor.
"""
import numpy as np

# Codebook order of the phase-rule sketch ("Fairy2i write-up" §3.1): index k -> value.
CODEBOOK = (1.0 + 0.0j, 0.0 + 1.0j, -1.0 + 0.0j, 0.0 - 1.0j)


# ---------------------------------------------------------------------------
# Widely-linear transform ("Fairy2i write-up" §2.1)
# ---------------------------------------------------------------------------
def widely_linear_from_real(R):
    """Split a real 2n x 2m layer R into complex n x m matrices (U, W) in fp64.

    With R11 = R[:n,:m], R12 = R[:n,m:], R21 = R[n:,:m], R22 = R[n:,m:]:
    U = (R11+R22)/2 + i (R21-R12)/2 and W = (R11-R22)/2 + i (R12+R21)/2,
    so that R [x_re; x_im] = U x + W conj(x) for x = x_re + i x_im
    (the real vector's first half is the real part, the second the imaginary).
    """
    R = np.asarray(R, dtype=np.float64)
    rows, cols = R.shape
    if rows % 2 or cols % 2:
        raise ValueError("R must have even dimensions")
    n, m = rows // 2, cols // 2
    R11, R12 = R[:n, :m], R[:n, m:]
    R21, R22 = R[n:, :m], R[n:, m:]
    U = 0.5 * (R11 + R22) + 1j * (0.5 * (R21 - R12))
    W = 0.5 * (R11 - R22) + 1j * (0.5 * (R12 + R21))
    return U, W


def widely_linear_planes_fp32(R):
    """(U_re, U_im, W_re, W_im) as float32 planes, each the fp64 value rounded to nearest-even."""
    U, W = widely_linear_from_real(R)
    return (U.real.astype(np.float32), U.imag.astype(np.float32),
            W.real.astype(np.float32), W.imag.astype(np.float32))


# ---------------------------------------------------------------------------
# Phase rule ("Fairy2i write-up" §3.1; "iFairy talk notes" §2.2.2)
# ---------------------------------------------------------------------------
def phase_code_atan2(a, b):
    """The rule as printed: theta = arg(w), k = floor(2 theta / pi + 0.5) mod 4.

    Evaluated in fp64 with atan2.  One reading is added: w = 0 (either signed
    zero) gives k = 0, the entry 1, where arg(-0 + 0i) = pi would give -1.
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    theta = np.arctan2(b, a)
    k = np.mod(np.floor(2.0 * theta / np.pi + 0.5), 4.0).astype(np.uint8)
    k[(a == 0) & (b == 0)] = 0
    return k


def phase_code(a, b):
    """Exact form of the same rule: the sector of w = a + ib decided by comparisons.

    floor(2 theta/pi + 0.5) mod 4 picks the sector [-pi/4, pi/4) -> 0,
    [pi/4, 3pi/4) -> 1, [3pi/4, pi] and (-pi, -3pi/4) -> 2, [-3pi/4, -pi/4) -> 3,
    so a tie on a diagonal goes to the sector counter-clockwise of it:
      k = 0  iff  a > |b|   or (b = -a and a > 0)
      k = 1  iff  b > |a|   or (a = b and b > 0)
      k = 2  iff -a > |b|   or (b = -a and a < 0)
      k = 3  iff -b > |a|   or (a = b and b < 0)
    and w = 0 gives k = 0.  No rounding enters, so this is the form the parity checks use.
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    aa, ab = np.abs(a), np.abs(b)
    k1 = (b > aa) | ((a == b) & (b > 0))
    k2 = (-a > ab) | ((b == -a) & (a < 0))
    k3 = (-b > aa) | ((a == b) & (b < 0))
    return np.where(k1, np.uint8(1), np.where(k2, np.uint8(2), np.where(k3, np.uint8(3), np.uint8(0))))


def code_to_br_bi(k):
    """Real and imaginary parts of the codebook entry: Br, Bi in {-1, 0, +1} (int8)."""
    k = np.asarray(k)
    sign = 1 - 2 * (k >> 1).astype(np.int8)
    cls = (k & 1).astype(np.int8)
    br = (sign * (1 - cls)).astype(np.int8)
    bi = (sign * cls).astype(np.int8)
    return br, bi


# ---------------------------------------------------------------------------
# Axis scales ("Fairy2i write-up" §3.2) and one quantizer stage
# ---------------------------------------------------------------------------
def stage_sums(a, b, k):
    """Per-class sums for one stage: (S_re, C_re, S_im, C_im).

    S_re sums |Re r| over entries coded +-1 (k even), S_im sums |Im r| over
    entries coded +-i (k odd); C_* count them.  Sums are fp64.
    """
    k = np.asarray(k)
    re_cls = (k & 1) == 0
    s_re = float(np.sum(np.abs(np.asarray(a, np.float64)[re_cls]), dtype=np.float64))
    s_im = float(np.sum(np.abs(np.asarray(b, np.float64)[~re_cls]), dtype=np.float64))
    return s_re, int(np.count_nonzero(re_cls)), s_im, int(np.count_nonzero(~re_cls))


def scales_from_sums(S_re, C_re, S_im, C_im):
    """s = S / C in fp64, rounded to nearest-even fp32; an empty class gives 0."""
    s_re = np.float32(S_re / C_re) if C_re > 0 else np.float32(0.0)
    s_im = np.float32(S_im / C_im) if C_im > 0 else np.float32(0.0)
    return s_re, s_im


def quantize_stage(a, b):
    """Codes and fp32 scales of one PhaseQuant stage applied to residual a + ib (fp64)."""
    k = phase_code(a, b)
    sums = stage_sums(a, b, k)
    return k, scales_from_sums(*sums), sums


# ---------------------------------------------------------------------------
# Recursive residual ("Fairy2i write-up" §4.1)
# ---------------------------------------------------------------------------
def _finite_weights(w_re, w_im):
    """fp64 copy of w; an entry with a non-finite part is taken as 0 (reading for unstated inputs)."""
    a = np.asarray(w_re, dtype=np.float64).copy()
    b = np.asarray(w_im, dtype=np.float64).copy()
    bad = ~(np.isfinite(a) & np.isfinite(b))
    a[bad] = 0.0
    b[bad] = 0.0
    return a, b, bad


def residual_after(w_re, w_im, codes, scales):
    """r = w - sum_u w_hat_u over the given stages, in fp64, one stage at a time in order.

    `codes` is a sequence of unpacked code arrays (uint8, same shape as w) and
    `scales` a sequence of (s_re, s_im) fp32 pairs; w_hat_u = s_re Br + i s_im Bi.
    """
    a, b, _ = _finite_weights(w_re, w_im)
    for k, (s_re, s_im) in zip(codes, scales):
        br, bi = code_to_br_bi(k)
        a = a - np.float64(s_re) * br.astype(np.float64)
        b = b - np.float64(s_im) * bi.astype(np.float64)
    return a, b


def quantize_tensor(w_re, w_im, T, row_chunk=None):
    """T-stage PhaseQuant of one tensor, each stage on the residual of the stages before.

    Returns (packed codes uint8 [T][N][K/4], scales float32 [T][2], sums list).
    Rows are processed in chunks of `row_chunk` so that large tensors fit in host
    memory; the per-stage sums are the in-order fp64 sums of the chunk sums.
    """
    w_re = np.asarray(w_re)
    w_im = np.asarray(w_im)
    N, K = w_re.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    rc = N if row_chunk is None else max(1, int(row_chunk))
    packed = np.zeros((T, N, K // 4), dtype=np.uint8)
    scales = np.zeros((T, 2), dtype=np.float32)
    all_sums = []
    for t in range(T):
        S_re = S_im = 0.0
        C_re = C_im = 0
        for r0 in range(0, N, rc):
            r1 = min(N, r0 + rc)
            prev = [unpack_codes(packed[u, r0:r1], K) for u in range(t)]
            a, b = residual_after(w_re[r0:r1], w_im[r0:r1], prev, [tuple(scales[u]) for u in range(t)])
            k = phase_code(a, b)
            packed[t, r0:r1] = pack_codes(k)
            sr, cr, si, ci = stage_sums(a, b, k)
            S_re += sr
            C_re += cr
            S_im += si
            C_im += ci
        scales[t] = scales_from_sums(S_re, C_re, S_im, C_im)
        all_sums.append((S_re, C_re, S_im, C_im))
    return packed, scales, all_sums


def near_boundary_mask(a, b, prev_scale_sum):
    """Entries whose phase sits within 1e-6 (relative) of a sector edge, or whose
    residual is within 1e-6 of the earlier stages' scale sum of zero."""
    aa = np.abs(np.asarray(a, np.float64))
    ab = np.abs(np.asarray(b, np.float64))
    edge = np.abs(aa - ab) <= 1e-6 * (aa + ab)
    tiny = (aa + ab) <= 1e-6 * float(prev_scale_sum)
    return edge | tiny


# ---------------------------------------------------------------------------
# Packing: four 2-bit codes per byte, code j of a row in bits 2(j%4), 2(j%4)+1
# of byte j//4 (little-endian within the byte).
# ---------------------------------------------------------------------------
def pack_codes(k):
    k = np.asarray(k, dtype=np.uint8)
    if k.shape[-1] % 4:
        raise ValueError("last dimension must be a multiple of 4")
    q = k.reshape(k.shape[:-1] + (k.shape[-1] // 4, 4)).astype(np.uint16)
    byte = q[..., 0] | (q[..., 1] << 2) | (q[..., 2] << 4) | (q[..., 3] << 6)
    return byte.astype(np.uint8)


def unpack_codes(packed, K=None):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1], 4), dtype=np.uint8)
    for q in range(4):
        out[..., q] = (p >> (2 * q)) & 3
    out = out.reshape(p.shape[:-1] + (p.shape[-1] * 4,))
    if K is not None and K != out.shape[-1]:
        raise ValueError("K does not match the packed width")
    return out


# ---------------------------------------------------------------------------
# Product ("Fairy2i write-up" §2.1 and §4.2; "iFairy article" §二.2)
# ---------------------------------------------------------------------------
def dequantize(packed, scales, rows=None):
    """W_hat = sum_t (s_re,t Br_t + i s_im,t Bi_t) as complex128, optionally for a row subset."""
    packed = np.asarray(packed)
    scales = np.asarray(scales, dtype=np.float32)
    T = packed.shape[0]
    sel = packed if rows is None else packed[:, rows]
    K = sel.shape[-1] * 4
    acc = np.zeros(sel.shape[1:-1] + (K,), dtype=np.complex128)
    for t in range(T):
        br, bi = code_to_br_bi(unpack_codes(sel[t]))
        acc += np.float64(scales[t, 0]) * br + 1j * (np.float64(scales[t, 1]) * bi)
    return acc


def dequantize_bf16(packed, scales):
    """Dequantized weights for training ("iFairy talk notes" §2.2.1), as the library states them:
    per entry the stage terms +-s_re (real axis) or +-s_im (imaginary axis) are added in float32 in
    stage order starting from +0, and each sum is rounded once to bf16 (nearest-even).  Returns
    (re, im) float32 arrays holding bf16 values."""
    packed = np.asarray(packed)
    scales = np.asarray(scales, dtype=np.float32)
    T = packed.shape[0]
    K = packed.shape[-1] * 4
    re = np.zeros(packed.shape[1:-1] + (K,), dtype=np.float32)
    im = np.zeros_like(re)
    for t in range(T):
        br, bi = code_to_br_bi(unpack_codes(packed[t]))   # exactly one of the two is +-1
        re = np.where(br != 0, re + np.where(br > 0, scales[t, 0], -scales[t, 0]).astype(np.float32), re)
        im = np.where(bi != 0, im + np.where(bi > 0, scales[t, 1], -scales[t, 1]).astype(np.float32), im)
    return bf16_round(re), bf16_round(im)


def product_rows(codes_u, scales_u, codes_w, scales_w, x_re, x_im, rows=None):
    """y[b, n] = sum_t (U_hat_t x_b + W_hat_t conj(x_b)) for the selected rows (complex128).

    x_re, x_im: [B][K] arrays of bf16-representable values.  codes_w = None means
    no conjugate branch.  The matrices are dequantized with the given fp32 scales
    and multiplied in complex128 (the page's sketch scales its two output parts
    differently; this follows the definition w_hat = s_re Re b + i s_im Im b).
    """
    x = np.asarray(x_re, np.float64) + 1j * np.asarray(x_im, np.float64)
    if x.ndim == 1:
        x = x[None, :]
    U = dequantize(codes_u, scales_u, rows)
    y = x @ U.T
    if codes_w is not None:
        W = dequantize(codes_w, scales_w, rows)
        y = y + np.conj(x) @ W.T
    return y


def product(codes_u, scales_u, codes_w, scales_w, x_re, x_im):
    return product_rows(codes_u, scales_u, codes_w, scales_w, x_re, x_im, None)


def tolerance_bound(scales_u, scales_w, x_re, x_im, rel=1e-5):
    """Per-token bound rel * sum_{t,branch}(s_re + s_im) * sum_j(|Re x_j| + |Im x_j|)."""
    s = float(np.sum(np.asarray(scales_u, np.float64)))
    if scales_w is not None:
        s += float(np.sum(np.asarray(scales_w, np.float64)))
    xr = np.abs(np.asarray(x_re, np.float64))
    xi = np.abs(np.asarray(x_im, np.float64))
    if xr.ndim == 1:
        xr, xi = xr[None, :], xi[None, :]
    return rel * s * np.sum(xr + xi, axis=1)


# ---------------------------------------------------------------------------
# Adjacent decode-block steps: complex rotary position encoding of the q / k
# projections ("iFairy article" §三: in the complex domain the rotation is one
# complex multiplication; "iFairy talk notes" §2.1.3) and the attention score
# Re(q^T conj(k)) ("Fairy2i write-up" §2.2, item 2; "iFairy talk notes" §2.1.4).
# The pages fix no frequencies: the rotation factors are inputs.
# ---------------------------------------------------------------------------
def rotate_outputs(y, rot_re, rot_im):
    """y (complex [rows][N]) times the per-output rotation rot_re + i rot_im, in complex128."""
    rot = np.asarray(rot_re, np.float64) + 1j * np.asarray(rot_im, np.float64)
    return np.asarray(y, np.complex128) * rot


def score(q, k):
    """Real part of the Hermitian inner product: Re(sum_j q_j conj(k_j)), over the last axis."""
    q = np.asarray(q, np.complex128)
    k = np.asarray(k, np.complex128)
    return np.real(np.sum(q * np.conj(k), axis=-1))


# ---------------------------------------------------------------------------
# bf16 helpers (exact conversions only)
# ---------------------------------------------------------------------------
def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_round(x):
    """Round float32 values to the nearest-even bf16 and return them as float32 (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    return (r.astype(np.uint32) << 16).view(np.float32)
