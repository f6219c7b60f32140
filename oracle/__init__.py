"""Float64 CPU oracle for layer-wise GPTQ + QEP weight quantisation.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA path.

Sources (cited by page title and section; the pages print no equations, so each
formula below is stated in full where it is used):

[OneComp-release]  "OneComp v1.1.0" release summary, easyvibecoding.app/curated/1062,
                   section "量化錯誤傳播 (QEP)" (QEP: propagate earlier layers'
                   quantisation error into a correction of the layer's weights;
                   Arai & Ichikawa, NeurIPS 2025) and section "v1.1.0全新量化方法"
                   (group quantisation example "4-bit, groupsize=128").
[OneComp-hub]      "富士通 One Compression" hub page, pomoai.com/hubs/FujitsuResearch/
                   OneCompression, section "核心功能拆解": the quantiser table (GPTQ =
                   2-4 bit Hessian-optimal rounding; RTN = nearest rounding), the
                   AutoBit + QEP pipeline, and the API ``GPTQ(wbits, groupsize)``,
                   ``qep=True``.
GPTQ               Frantar et al., "GPTQ: Accurate Post-Training Quantization for
                   Generative Pre-trained Transformers" (arXiv:2210.17323): the
                   column-by-column optimal-brain-quantiser sweep with the upper
                   Cholesky factor of the inverse Hessian and lazy block updates.

Notation: W is d_out x d_in (m x n); calibration inputs X, Xh (X-hat, the inputs
the quantised layer sees) are n_tok x n, token-major.  In this layout the
column-notation products X Xh^T and Xh Xh^T of the method become Xh^T X-style
n x n products below.

Readings taken where the sources leave a step open:
  * H = 2 Xh^T Xh, unnormalised, accumulated across calls.
  * QEP: W' = W + alpha * (W d) A^-1 with d = (X - Xh)^T Xh, A = Xh^T Xh + lam I,
    lam = damp * mean(diag(Xh^T Xh)); alpha = 0 returns W.
  * GPTQ prep: dead columns (diag H == 0) get H_jj = 1 and W[:, j] = 0; act_order
    processes columns by a stable descending sort of diag(H); H_d = H + damp *
    mean(diag H) * I.
  * Group grid: asymmetric min/max over the group's values, zero NOT forced into
    the range; equal min and max widen to [min-1, max+1]; scale = (max-min)/(2^b-1);
    zero = clip(rint(-min/scale), 0, 2^b-1); code q = clip(rint(w/scale) + zero,
    0, 2^b-1); rint rounds half to even.
  * Without act_order the group parameters are computed when the sweep reaches the
    group's first column, from the group's current (error-updated) values; with
    act_order they are computed up front from W' in original column order and
    groups stay contiguous in original order.
  * Packing: per row an LSB-first bitstream of b-bit codes along d_in in original
    column order, stored as uint32 words (b = 3 runs across word boundaries).
  * LPCD (layer-projected coordinate descent): the pages give no formula; the
    reading for a two-layer linear submodule is stated above ``lpcd_left_project``.
    Its functions are pinned to that reading's own mathematics (brute-force least
    squares); parity against the pages' LPCD itself is unpinned.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg as sla

__all__ = [
    "hessian", "qep_cross", "qep_correct", "gptq_prepare", "inv_chol_upper",
    "inv_chol_upper_reversed", "group_params", "quantize_values", "gptq_sweep",
    "gptq_sweep_unblocked", "gptq_quantize", "pack_codes", "unpack_codes",
    "layer_errors", "teacher_forced_check", "gptq_objective",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------- Hessian

def hessian(xhat, H0=None, chunk: int = 8192):
    """H0 + 2 * Xh^T Xh (Hessian of the layer-wise squared error in W), in float64.

    GPTQ's "Hessian-optimal rounding" [OneComp-hub, quantiser table, GPTQ row]
    uses the Hessian of ||W Xh^T - Q Xh^T||_F^2 with respect to a row of W,
    which is 2 Xh^T Xh.  Accumulates chunk by chunk over tokens.
    """
    xhat = np.asarray(xhat)
    n = xhat.shape[1]
    S = np.zeros((n, n))
    for t0 in range(0, xhat.shape[0], chunk):
        blk = _f64(xhat[t0:t0 + chunk])
        S += blk.T @ blk
    H = 2.0 * S
    return H if H0 is None else _f64(H0) + H


# ----------------------------------------------------------------------------- QEP

def qep_cross(x, xhat, chunk: int = 8192):
    """d = (X - Xh)^T Xh, the cross term of QEP's correction, in float64."""
    x = np.asarray(x)
    xhat = np.asarray(xhat)
    n = x.shape[1]
    d = np.zeros((n, n))
    for t0 in range(0, x.shape[0], chunk):
        xb = _f64(x[t0:t0 + chunk])
        hb = _f64(xhat[t0:t0 + chunk])
        d += (xb - hb).T @ hb
    return d


def qep_correct(W, x, xhat, alpha: float, damp: float, H=None, chunk: int = 8192, d=None):
    """QEP weight correction [OneComp-release, section "量化錯誤傳播 (QEP)"].

    The corrected weight makes the quantised layer, fed the perturbed inputs Xh,
    reproduce the full-precision output W X^T: it minimises
    ||W X^T - W' Xh^T||_F^2 + lam ||W' - W||_F^2, whose minimiser is
        W* = W + W d A^-1,  d = (X - Xh)^T Xh,  A = Xh^T Xh + lam I,
    and QEP moves a fraction alpha of the way: W' = W + alpha * W d A^-1, with
    lam = damp * mean(diag(Xh^T Xh)).  If H (= 2 Xh^T Xh over the same tokens)
    is given it replaces the recomputation of Xh^T Xh; likewise d (= the
    qep_cross of the same tokens) replaces the recomputation of the cross
    term, and x, xhat are then not read.
    """
    W = _f64(W)
    S = hessian(xhat, chunk=chunk) / 2.0 if H is None else _f64(H) / 2.0
    d = qep_cross(x, xhat, chunk=chunk) if d is None else _f64(d)
    n = S.shape[0]
    lam = damp * float(np.mean(np.diag(S)))
    A = S + lam * np.eye(n)
    G = W @ d
    # G A^-1 = (A^-1 G^T)^T since A is symmetric positive definite.
    corr = sla.cho_solve(sla.cho_factor(A, lower=True), G.T).T
    return W + alpha * corr


# ----------------------------------------------------------------------------- GPTQ prep

def gptq_prepare(W, H, damp: float, act_order: bool, perm=None):
    """Dead columns, act_order permutation and dampening (GPTQ's preparation).

    Returns dict(W = W with dead columns zeroed, permuted to processing order;
    Hd = dampened, permuted Hessian; perm = processing order as original column
    indices; dead = boolean mask of dead columns (original order); W_dead = W with
    dead columns zeroed, original order).  ``perm`` overrides the act_order order
    (used to replay another implementation's tie-breaking); it must be a
    permutation of range(n).
    """
    W = _f64(W).copy()
    H = _f64(H).copy()
    n = H.shape[0]
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    W[:, dead] = 0.0
    if perm is not None:
        perm = np.asarray(perm)
        if not np.array_equal(np.sort(perm), np.arange(n)):
            raise ValueError("perm is not a permutation")
    elif act_order:
        perm = np.argsort(-np.diag(H), kind="stable")
    else:
        perm = np.arange(n)
    Hp = H[np.ix_(perm, perm)]
    lam = damp * float(np.mean(np.diag(Hp)))
    Hd = Hp + lam * np.eye(n)
    return {"W": W[:, perm], "Hd": Hd, "perm": perm, "dead": dead, "W_dead": W}


def inv_chol_upper(Hd):
    """U = upper Cholesky factor of Hd^-1 (U^T U = Hd^-1, diag U > 0).

    Route: Cholesky of Hd, inverse from the factor, Cholesky of the
    (symmetrised) inverse, transposed.
    """
    Hd = _f64(Hd)
    n = Hd.shape[0]
    c = sla.cho_factor(Hd, lower=True)
    Hinv = sla.cho_solve(c, np.eye(n))
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T


def inv_chol_upper_reversed(Hd):
    """Same factor by the reversed-order route: with J the index reversal,
    J Hd J = L L^T gives Hd = R R^T for the upper R = J L J, so Hd^-1 =
    (R^-1)^T R^-1 and U = R^-1 = J L^-1 J.  Unique, so it must equal
    ``inv_chol_upper``."""
    Hd = _f64(Hd)
    n = Hd.shape[0]
    rev = np.arange(n)[::-1]
    L = np.linalg.cholesky(Hd[np.ix_(rev, rev)])
    # triangular inverse (LAPACK trtri): L^-1, lower
    Linv, info = sla.lapack.dtrtri(L, lower=1)
    if info != 0:
        raise np.linalg.LinAlgError(f"trtri failed ({info})")
    return np.tril(Linv)[np.ix_(rev, rev)]


# ----------------------------------------------------------------------------- grid

def _grid_raw(vals, maxq: int):
    vals = _f64(vals)
    xmin = vals.min(axis=1)
    xmax = vals.max(axis=1)
    same = xmax == xmin
    xmin = np.where(same, xmin - 1.0, xmin)
    xmax = np.where(same, xmax + 1.0, xmax)
    scale = (xmax - xmin) / maxq
    return scale, -xmin / scale


def group_params(vals, maxq: int):
    """Asymmetric min/max grid of one group for every row.

    vals: rows x group-width.  Returns (scale, zero) float64 arrays, one per row:
    scale = (max - min) / maxq, zero = clip(rint(-min / scale), 0, maxq), with
    min and max widened by 1 each way when they are equal.
    """
    scale, zraw = _grid_raw(vals, maxq)
    return scale, np.clip(np.rint(zraw), 0, maxq)


def quantize_values(w, scale, zero, maxq: int):
    """q = clip(rint(w/scale) + zero, 0, maxq) and its dequantised value."""
    q = np.clip(np.rint(_f64(w) / scale) + zero, 0, maxq)
    return q, scale * (q - zero)


def _group_size(groupsize: int, n: int) -> int:
    return n if groupsize in (-1, 0) else int(groupsize)


# ----------------------------------------------------------------------------- sweep

def gptq_sweep_unblocked(Wp, U, wbits: int, groupsize: int, perm=None, static=None):
    """Textbook GPTQ sweep: column by column, full trailing update after each.

    For column j in processing order: q = quantise(w_j); e = (w_j - deq(q)) / U_jj;
    w_k -= e * U_jk for every later column k.  Dynamic groups take their grid at
    the group's first column from its current values; ``static`` = (scales, zeros)
    in original group order selects act_order's fixed grid instead.
    """
    W1 = _f64(Wp).copy()
    U = _f64(U)
    m, n = W1.shape
    maxq = (1 << wbits) - 1
    G = _group_size(groupsize, n)
    perm = np.arange(n) if perm is None else np.asarray(perm)
    codes = np.zeros((m, n), dtype=np.int64)
    deq = np.zeros((m, n))
    ng = n // G
    scales = np.zeros((m, ng))
    zeros = np.zeros((m, ng))
    if static is not None:
        scales, zeros = _f64(static[0]).copy(), _f64(static[1]).copy()
    for j in range(n):
        if static is None:
            if j % G == 0:
                s, z = group_params(W1[:, j:j + G], maxq)
                scales[:, j // G], zeros[:, j // G] = s, z
            g = j // G
        else:
            g = perm[j] // G
        q, dq = quantize_values(W1[:, j], scales[:, g], zeros[:, g], maxq)
        e = (W1[:, j] - dq) / U[j, j]
        W1[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        codes[:, j] = q
        deq[:, j] = dq
    return codes, deq, scales, zeros


def gptq_sweep(Wp, U, wbits: int, groupsize: int, perm=None, static=None, block: int = 256):
    """Lazy-blocked GPTQ sweep (same result as the unblocked form up to rounding).

    Inside a block of ``block`` columns the rank-1 updates are applied to the
    block only; the block's scaled errors E then update all later columns at
    once, W[:, b1:] -= E U[b0:b1, b1:].  A dynamic group must lie inside a block
    or start at a block start (groupsize divides the block, or the block divides
    groupsize), which keeps every group's values current at its first column.
    """
    W1 = _f64(Wp).copy()
    U = _f64(U)
    m, n = W1.shape
    maxq = (1 << wbits) - 1
    G = _group_size(groupsize, n)
    if static is None and not (block % G == 0 or G % block == 0 or G == n):
        raise ValueError("groupsize must divide the block or be a multiple of it")
    perm = np.arange(n) if perm is None else np.asarray(perm)
    codes = np.zeros((m, n), dtype=np.int64)
    deq = np.zeros((m, n))
    ng = n // G
    scales = np.zeros((m, ng))
    zeros = np.zeros((m, ng))
    if static is not None:
        scales, zeros = _f64(static[0]).copy(), _f64(static[1]).copy()
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        Wb = W1[:, b0:b1].copy()
        Eb = np.zeros((m, b1 - b0))
        for jj in range(b1 - b0):
            j = b0 + jj
            if static is None:
                if j % G == 0:
                    vals = W1[:, j:j + G] if jj == 0 else Wb[:, jj:jj + G]
                    s, z = group_params(vals, maxq)
                    scales[:, j // G], zeros[:, j // G] = s, z
                g = j // G
            else:
                g = perm[j] // G
            q, dq = quantize_values(Wb[:, jj], scales[:, g], zeros[:, g], maxq)
            e = (Wb[:, jj] - dq) / U[j, j]
            Wb[:, jj + 1:] -= np.outer(e, U[j, b0 + jj + 1:b1])
            Eb[:, jj] = e
            codes[:, j] = q
            deq[:, j] = dq
        W1[:, b0:b1] = Wb
        if b1 < n:
            W1[:, b1:] -= Eb @ U[b0:b1, b1:]
    return codes, deq, scales, zeros


def gptq_quantize(W, H, wbits: int, groupsize: int, damp: float, act_order: bool,
                  block: int = 256, unblocked: bool = False, perm=None, U=None):
    """GPTQ with per-group asymmetric grid, returning outputs in original order.

    Returns dict(codes = m x n int codes in original column order, packed = the
    uint32 bitstream, scales, zeros = m x (n/G), deq = dequantised weights in
    original order, perm = processing order, U = the inverse-Hessian factor).
    ``perm`` overrides the act_order order (used to replay another
    implementation's tie-breaking).  ``U``, if given, is the factor of this
    same preparation (inv_chol_upper of its Hd, e.g. from an earlier call on
    other rows of W) and is used instead of recomputing it.
    """
    prep = gptq_prepare(W, H, damp, act_order, perm=perm)
    perm = prep["perm"]
    n = perm.shape[0]
    maxq = (1 << wbits) - 1
    G = _group_size(groupsize, n)
    U = inv_chol_upper(prep["Hd"]) if U is None else _f64(U)
    static = None
    if act_order:
        Wd = prep["W_dead"]
        ng = n // G
        s = np.zeros((Wd.shape[0], ng))
        z = np.zeros((Wd.shape[0], ng))
        for g in range(ng):
            s[:, g], z[:, g] = group_params(Wd[:, g * G:(g + 1) * G], maxq)
        static = (s, z)
    if unblocked:
        codes_p, deq_p, scales, zeros = gptq_sweep_unblocked(prep["W"], U, wbits, groupsize,
                                                             perm, static)
    else:
        codes_p, deq_p, scales, zeros = gptq_sweep(prep["W"], U, wbits, groupsize, perm,
                                                   static, block=block)
    codes = np.empty_like(codes_p)
    codes[:, perm] = codes_p
    deq = np.empty_like(deq_p)
    deq[:, perm] = deq_p
    packed = pack_codes(codes, wbits) if (n * wbits) % 32 == 0 else None
    return {"codes": codes, "packed": packed, "scales": scales,
            "zeros": zeros, "deq": deq, "perm": perm, "U": U, "Hd": prep["Hd"]}


def gptq_objective(W, deq, H):
    """Sum over rows of (w - w_hat) H (w - w_hat)^T (the layer-wise loss GPTQ greedily lowers)."""
    E = _f64(W) - _f64(deq)
    return float(np.einsum("ij,jk,ik->", E, _f64(H), E))


# ----------------------------------------------------------------------------- packing

def pack_codes(codes, wbits: int):
    """Pack m x n integer codes (original order) into m x (n*wbits/32) uint32.

    Row-wise LSB-first bitstream: code c of a row occupies bits
    [c*wbits, c*wbits + wbits) of that row's stream; bit k of the stream is bit
    (k mod 32) of word k // 32.
    """
    codes = np.asarray(codes, dtype=np.uint64)
    m, n = codes.shape
    if (n * wbits) % 32:
        raise ValueError("n * wbits must be a multiple of 32")
    bits = (codes[:, :, None] >> np.arange(wbits, dtype=np.uint64)) & np.uint64(1)
    bits = bits.reshape(m, n * wbits // 32, 32)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (bits * weights).sum(axis=2).astype(np.uint32)


def unpack_codes(packed, wbits: int, n: int):
    """Inverse of ``pack_codes``."""
    packed = np.asarray(packed, dtype=np.uint64)
    m = packed.shape[0]
    bits = (packed[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    bits = bits.reshape(m, n, wbits)
    return (bits << np.arange(wbits, dtype=np.uint64)).sum(axis=2).astype(np.int64)


# ----------------------------------------------------------------------------- errors

def layer_errors(W, deq, x, xhat, W_prime=None):
    """Output errors of the quantised layer on the given tokens.

    e_lit  = ||(W - Q) X^T||_F        (original W, full-precision X),
    e_qep  = ||W X^T - Q Xh^T||_F     (QEP's end-to-end objective),
    e_gptq = ||(W' - Q) Xh^T||_F      (what GPTQ minimises, when W' is given).
    """
    W = _f64(W)
    Q = _f64(deq)
    X = _f64(x)
    Xh = _f64(xhat)
    out = {"e_lit": float(np.linalg.norm((W - Q) @ X.T)),
           "e_qep": float(np.linalg.norm(W @ X.T - Q @ Xh.T))}
    if W_prime is not None:
        out["e_gptq"] = float(np.linalg.norm((_f64(W_prime) - Q) @ Xh.T))
    return out


# ----------------------------------------------------------------------------- teacher forcing

def _half_dist(v):
    """Distance of v to the nearest rounding boundary (a half-integer)."""
    return np.abs(v - (np.floor(v) + 0.5))


def teacher_forced_check(W, H, wbits: int, groupsize: int, damp: float, act_order: bool,
                         codes, scales, zeros, perm=None, rows=None, block: int = 256,
                         boundary_tol: float = 1e-3, U=None):
    """Replay the sweep with another implementation's decisions forced in.

    Runs the float64 sweep row by row, but for every column uses the candidate's
    code (and, for dynamic groups, its scale and zero) so that one legitimately
    flipped rounding does not cascade.  At every column where the candidate's
    code differs from the oracle's own rounding of the same pre-rounding value
    v = w/scale, it measures v's distance to the nearest half-integer.  Returns
    counts and the worst distances; the candidate passes when every mismatch is
    a single step within ``boundary_tol`` of a boundary and every scale is within
    the caller's tolerance of the oracle's.  ``U``, if given, is the factor of
    this same preparation (as in gptq_quantize).
    """
    codes = np.asarray(codes)
    scales = _f64(scales)
    zeros = _f64(zeros)
    W = _f64(W)
    if rows is not None:
        rows = np.asarray(rows)
        W, codes, scales, zeros = W[rows], codes[rows], scales[rows], zeros[rows]
    m, n = W.shape
    maxq = (1 << wbits) - 1
    G = _group_size(groupsize, n)
    if not act_order and not (block % G == 0 or G % block == 0 or G == n):
        # the same constraint as gptq_sweep: a dynamic group's values are read
        # at its first column, so it must not start inside a block and run past it
        raise ValueError("groupsize must divide the block or be a multiple of it")
    prep = gptq_prepare(W, H, damp, act_order, perm=perm)
    perm = prep["perm"]
    U = inv_chol_upper(prep["Hd"]) if U is None else _f64(U)
    codes_p = codes[:, perm]
    stats = {"n_codes": m * n, "n_mismatch": 0, "n_bad": 0, "max_mismatch_dist": 0.0,
             "scale_max_rel": 0.0, "zero_mismatch": 0, "zero_bad": 0}

    def check_grid(vals, g):
        s_or, zraw = _grid_raw(vals, maxq)
        z_or = np.clip(np.rint(zraw), 0, maxq)
        rel = np.abs(scales[:, g] - s_or) / np.abs(s_or)
        stats["scale_max_rel"] = max(stats["scale_max_rel"], float(rel.max(initial=0.0)))
        zmis = zeros[:, g] != z_or
        if zmis.any():
            v = zraw[zmis]
            stats["zero_mismatch"] += int(zmis.sum())
            bad = (_half_dist(v) > boundary_tol) | (np.abs(zeros[zmis, g] - z_or[zmis]) > 1)
            stats["zero_bad"] += int(bad.sum())

    if act_order:
        Wd = prep["W_dead"]
        for g in range(n // G):
            check_grid(Wd[:, g * G:(g + 1) * G], g)
    W1 = prep["W"].copy()
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        Wb = W1[:, b0:b1].copy()
        Eb = np.zeros((m, b1 - b0))
        for jj in range(b1 - b0):
            j = b0 + jj
            if not act_order:
                g = j // G
                if j % G == 0:
                    check_grid(W1[:, j:j + G] if jj == 0 else Wb[:, jj:jj + G], g)
            else:
                g = perm[j] // G
            s, z = scales[:, g], zeros[:, g]
            v = Wb[:, jj] / s
            q_or = np.clip(np.rint(v) + z, 0, maxq)
            q = codes_p[:, j].astype(np.float64)
            mis = q_or != q
            if mis.any():
                d = _half_dist(v[mis])
                stats["n_mismatch"] += int(mis.sum())
                stats["max_mismatch_dist"] = max(stats["max_mismatch_dist"], float(d.max()))
                bad = (d > boundary_tol) | (np.abs(q_or[mis] - q[mis]) > 1)
                stats["n_bad"] += int(bad.sum())
            dq = s * (q - z)
            e = (Wb[:, jj] - dq) / U[j, j]
            Wb[:, jj + 1:] -= np.outer(e, U[j, b0 + jj + 1:b1])
            Eb[:, jj] = e
        W1[:, b0:b1] = Wb
        if b1 < n:
            W1[:, b1:] -= Eb @ U[b0:b1, b1:]
    return stats


# ----------------------------------------------------------------------------- propagation chain

def dequantize(packed, scales, zeros, wbits: int, groupsize: int, n: int):
    """Q = scale * (q - zero) from packed codes (original column order)."""
    codes = unpack_codes(np.asarray(packed), wbits, n)
    G = _group_size(groupsize, n)
    s = np.repeat(_f64(scales), G, axis=1)
    z = np.repeat(_f64(zeros), G, axis=1)
    return s * (codes - z)


def dequant_gemv(packed, scales, zeros, wbits: int, groupsize: int, n: int, x):
    """y = x Q^T with Q = dequantize(packed, scales, zeros): the quantised
    layer applied to a few bf16 activation rows x [batch x n] (the served
    model's linear layer, One Compression hub page section "4. vLLM 插件：
    量化模型直接推理": quantised models run inference from their GPTQ codes).
    Float64; returns [batch x m]."""
    return _f64(x) @ dequantize(packed, scales, zeros, wbits, groupsize, n).T


_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127   # largest finite bf16 number


def _bf16(a):
    """Round every value to the nearest bf16 number, ties to even, in one step
    from float64 (no intermediate float32).  bf16 has 8 significant bits and
    the float32 exponent range: a normal value x = m 2^e (0.5 <= |m| < 1) is
    rounded to a multiple of 2^(e-8); below the smallest normal 2^-126 the
    spacing stays 2^-133 (subnormals).  Results beyond the largest finite bf16
    become +-inf, as round-to-nearest overflow does; zeros (with their sign),
    infinities and NaN pass through.  Returns float64."""
    x = _f64(a)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0.0)
    v = x[fin]
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)          # exponent of the spacing at v
    y = np.ldexp(np.rint(np.ldexp(v, -q)), q)   # scaling by 2^-q is exact; rint ties to even
    y = np.where(np.abs(y) > _BF16_MAX, np.copysign(np.inf, y), y)
    out[fin] = y
    return out


def _act(y, act: str):
    if act == "silu":
        return y / (1.0 + np.exp(-y))
    if act == "none":
        return y
    raise ValueError(act)


def quantize_chain(Ws, x0, alpha: float, damp: float, wbits: int, groupsize: int, act_order: bool,
                   act: str = "silu"):
    """Quantise a chain of linear layers with true error propagation (QEP's
    setting, OneComp release summary section "量化錯誤傳播 (QEP)").

    Layer l maps d_in = Ws[l].shape[1] features to d_out = Ws[l].shape[0].  Two
    activation streams run through the chain: the full-precision one,
    X_{l+1} = f(X_l W_l^T), and the quantised one, Xh_{l+1} = f(Xh_l Q_l^T),
    starting from Xh_0 = X_0.  Layer l is quantised on its own pair
    (X_l, Xh_l): H = 2 Xh_l^T Xh_l, W' = qep_correct(W_l, X_l, Xh_l), GPTQ of W'.
    Weights and activations enter each forward product as bf16 values, the
    product is rounded to bf16 and so is the activation of it (a bf16 model's
    linear layer and activation); sums are exact in float64 here.
    Returns a list of per-layer dicts (X, Xhat, H, W_prime, codes, packed,
    scales, zeros, deq) and the final pair (X_L, Xh_L).
    """
    x = _bf16(x0)
    xh = x.copy()
    layers = []
    for W in Ws:
        W = _f64(W)
        H = hessian(xh)
        Wp = qep_correct(W, x, xh, alpha, damp, H=H)
        q = gptq_quantize(Wp, H, wbits, groupsize, damp, act_order)
        layers.append({"X": x, "Xhat": xh, "H": H, "W_prime": Wp, **q})
        x = _bf16(_act(_bf16(x @ _bf16(W).T), act))
        xh = _bf16(_act(_bf16(xh @ _bf16(q["deq"]).T), act))
    return layers, (x, xh)


# ----------------------------------------------------------------------------- LPCD (two-layer submodule)
#
# Layer-projected coordinate descent [OneComp-release, section "v1.1.0全新量化方法"
# (LPCD bullet) and section "量化錯誤傳播 (QEP)"; OneComp-hub, section "3. LPCD：
# 子模块联合优化"]: related linear layers are quantised together by optimising a
# relaxed (continuous) objective of the submodule's output, one layer at a time,
# and projecting each layer's relaxed solution with the layer-wise quantiser.
# The pages give neither the objective nor the update; the reading taken here is
# the plainest one for a two-layer linear submodule y = x W1^T W2^T (V/O without
# the attention mixing, or any two linear layers in sequence):
#   objective  E(Q1, Q2) = || x W1^T W2^T - xh Q1^T Q2^T ||_F^2
#   start      the layer-wise method: QEP (alpha) + GPTQ of W1 on (x, xh), then of
#              W2 on (z, zh) with z = x W1^T, zh = xh Q1^T (bf16 forward products)
#   each round layer-1 step: with Q2 fixed, the relaxed minimiser of E over Q1
#              (ridge-regularised on both sides) is
#                 W1* = (Q2^T Q2 + mu I)^-1 Q2^T W2 . W1 (x^T xh + lam I)(xh^T xh + lam I)^-1
#              and the second factor is QEP's correction with alpha = 1; GPTQ of
#              W1* with H1 = 2 xh^T xh projects it.
#              layer-2 step: with Q1 fixed, the relaxed minimiser over Q2 is QEP's
#              correction with alpha = 1 on (z, zh); GPTQ with H2 = 2 zh^T zh
#              projects it.
#   lam = damp mean(diag(xh^T xh)) as in QEP; mu = damp mean(diag(Q2^T Q2)).

def lpcd_left_project(B, W2, V, damp: float):
    """(B^T B + mu I)^-1 B^T W2 V with mu = damp * mean(diag(B^T B)): the left
    factor of LPCD's relaxed layer-1 step (B = the quantised second layer,
    W2 = its full-precision weights, V = QEP-corrected first layer with
    alpha = 1).  It is the ridge-regression minimiser of
    ||B W - W2 V||_F^2 + mu ||W||_F^2 over W (d x n)."""
    B, W2, V = _f64(B), _f64(W2), _f64(V)
    M = B.T @ B
    mu = damp * float(np.mean(np.diag(M)))
    M = M + mu * np.eye(M.shape[0])
    return sla.cho_solve(sla.cho_factor(M), B.T @ (W2 @ V))


def submodule_error(W1, W2, Q1, Q2, x, xh):
    """E = ||x W1^T W2^T - xh Q1^T Q2^T||_F^2 and the same for the reference
    output alone (float64, no rounding)."""
    y = (_f64(x) @ _f64(W1).T) @ _f64(W2).T
    yh = (_f64(xh) @ _f64(Q1).T) @ _f64(Q2).T
    return float(np.sum((y - yh) ** 2)), float(np.sum(y ** 2))


def lpcd_pair(W1, W2, x, xh, alpha: float, damp: float, wbits: int, groupsize: int, act_order: bool,
              rounds: int = 1):
    """Quantise the two-layer submodule (W1: d x n, W2: m x d) by the reading
    above: the layer-wise QEP start, then `rounds` rounds of the layer-1 and
    layer-2 projected steps.  Forward products use bf16 weights and activations
    and round the product to bf16, as ``quantize_chain`` does.  Returns a dict
    with the final quantised layers (q1, q2: gptq_quantize outputs), the
    relaxed layer-1 solutions of each round (W1_star) with the quantised second
    layer each was solved against (Q2_used), and the submodule error after the
    start and after every round (errors, ref)."""
    W1, W2 = _f64(W1), _f64(W2)
    x, xh = _bf16(x), _bf16(xh)
    H1 = hessian(xh)
    q1 = gptq_quantize(qep_correct(W1, x, xh, alpha, damp, H=H1), H1, wbits, groupsize, damp, act_order)
    z = _bf16(x @ _bf16(W1).T)
    zh = _bf16(xh @ _bf16(q1["deq"]).T)
    H2 = hessian(zh)
    q2 = gptq_quantize(qep_correct(W2, z, zh, alpha, damp, H=H2), H2, wbits, groupsize, damp, act_order)
    e, ref = submodule_error(W1, W2, q1["deq"], q2["deq"], x, xh)
    errors, stars, q2_used = [e], [], []
    V1 = qep_correct(W1, x, xh, 1.0, damp, H=H1)
    for _ in range(rounds):
        W1s = lpcd_left_project(q2["deq"], W2, V1, damp)
        stars.append(W1s)
        q2_used.append(q2["deq"])
        q1 = gptq_quantize(W1s, H1, wbits, groupsize, damp, act_order)
        zh = _bf16(xh @ _bf16(q1["deq"]).T)
        H2 = hessian(zh)
        q2 = gptq_quantize(qep_correct(W2, z, zh, 1.0, damp, H=H2), H2, wbits, groupsize, damp, act_order)
        errors.append(submodule_error(W1, W2, q1["deq"], q2["deq"], x, xh)[0])
    return {"q1": q1, "q2": q2, "W1_star": stars, "Q2_used": q2_used, "V1": V1, "errors": errors, "ref": ref}


# ----------------------------------------------------------------------------- Hadamard rotation

def hadamard(b: int):
    """Sylvester Hadamard matrix of order b (a power of two): H_1 = [1],
    H_2k = [[H_k, H_k], [H_k, -H_k]]."""
    if b < 1 or b & (b - 1):
        raise ValueError("b must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def hadamard_rotate(x, b: int):
    """x (I (x) H_b) / sqrt(b) along the last axis (rotation preprocessing,
    OneComp release summary section "進階預處理與後處理")."""
    x = _f64(x)
    n = x.shape[-1]
    if n % b:
        raise ValueError("b must divide the last axis")
    Hb = hadamard(b) / np.sqrt(b)
    return (x.reshape(-1, n // b, b) @ Hb).reshape(x.shape)
