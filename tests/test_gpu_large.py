"""Parity of the fused layer call on the large layer shapes: the Llama-2-7B MLP
down_proj (d_in 11008, 3-bit g128, act_order), the Llama-3-70B-shaped MLP
down_proj (d_in 28672, d_out 8192, 2-bit g64, act_order) and the gate/up shape
of the 7B model (d_in 4096, d_out 11008, 3-bit g128, its full 131072
calibration tokens).

At their full calibration sizes the float64 oracle cannot redo the two wide
layers in a test, so each of those is checked twice:
  * full d_in and d_out with fewer calibration tokens (same recipe, more
    tokens than d_in for the 11008-wide layer and enough to make the
    28672-wide Hessian full rank), against the oracle fed the same seeded
    inputs: the whole Hessian, W' (every row, or sampled rows), teacher-forced
    GPTQ on sampled rows, code identity, scales, the layer output error;
  * the full workload, as bench.py launches it: Hessian entries recomputed in
    float64 from sampled Xhat columns, and the invariants of the outputs
    (finite W', codes within range, positive scales, integral zeros).

Bars (the quantisation workload's stated tolerances): Hessian relative
Frobenius error <= 1e-4; scales relative error <= 1e-5 and zeros equal unless
-min/scale sits within 1e-3 of a rounding boundary; every code mismatch one
step within 1e-3 of a boundary when replayed with the candidate's earlier
decisions forced in, and >= 99.9% of the codes identical; the layer output
error ||(W - Q) X^T||_F within 1% of the oracle's.  W' to within 1e-5 of
max |W|: it differs from the oracle's by the rounding of X - Xhat to bf16
(at most 2^-9 of each difference, of random sign, about 1e-3 of the
correction, which is a few percent of W at most on these workloads), fp32
accumulation and the fp32 factor.
"""
import json
import os

import numpy as np
import pytest

import oracle
from synthetic import CONFIGS, llama7b_layers, make_layer_device

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

CHUNK = 8192
# (workload, calibration tokens for the oracle comparison, rows replayed, QEP rows)
CASES = {
    "down_proj_11008": (65536, 32, None),
    "down_proj_28672": (32768, 8, 16),
}


def gate_spec():
    """The gate projection of the 7B-shaped model's first block."""
    return next(s for s in llama7b_layers() if s.name.endswith("_gate"))


def log_numbers(name, **kw):
    """Append measured parity numbers to $OC_PARITY_LOG (JSON lines), if set."""
    path = os.environ.get("OC_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **kw}) + "\n")


def run_fused(spec, L):
    n = spec.d_in
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    H, W_out, codes, scales, zeros, perm = oc.oc_quantize_layer(
        L["W"], L["X"], L["Xhat"], spec.alpha, spec.damp, spec.wbits, spec.groupsize,
        spec.act_order, perm_out=perm)
    torch.cuda.synchronize()
    return H, W_out, codes, scales, zeros, perm


def oracle_terms(spec, L):
    """(H, d) of the call's calibration tokens, float64, from the oracle."""
    n = spec.d_in
    H = np.zeros((n, n))
    d = np.zeros((n, n))
    for t0 in range(0, spec.n_tok, CHUNK):
        xc = L["X"][t0:t0 + CHUNK].float().cpu().numpy()
        hc = L["Xhat"][t0:t0 + CHUNK].float().cpu().numpy()
        H = oracle.hessian(hc, H0=H)
        d += oracle.qep_cross(xc, hc)
    return H, d


def rel_fro(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def plain_identity(cg, ref_codes):
    return float(np.mean(cg == ref_codes))


def check_layer(name, spec, n_rows, qep_rows, seed=11):
    """The fused call on `spec` against the oracle on the same inputs."""
    m, n, G = spec.d_out, spec.d_in, spec.groupsize
    L = make_layer_device(spec, "cuda")
    Hg, Wg, codes, scales, zeros, perm = run_fused(spec, L)
    H, d = oracle_terms(spec, L)

    Hg = Hg.cpu().numpy()
    assert np.array_equal(Hg, Hg.T)
    h_rel = rel_fro(Hg, H)
    assert h_rel <= 1e-4, h_rel
    del Hg

    # QEP: every row of W' (or a sample of rows on the widest layer)
    W = L["W"].cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(seed)
    qrows = np.arange(m) if qep_rows is None else np.sort(rng.choice(m, qep_rows, replace=False))
    Wp = oracle.qep_correct(W[qrows], None, None, spec.alpha, spec.damp, H=H, d=d)
    del d
    E = Wg.cpu().numpy()[qrows] - Wp
    corr = Wp - W[qrows]
    w_err = float(np.abs(E).max() / np.abs(W).max())
    c_err = float(np.linalg.norm(E) / np.linalg.norm(corr))
    assert w_err <= 1e-5, (w_err, c_err)
    assert c_err <= 1e-2, (w_err, c_err)

    # GPTQ: sampled rows replayed from the oracle's W' and H, with the GPU's
    # processing order (act_order orders by the fp32 Hessian diagonal, so near
    # ties may swap: that order must be descending in the oracle's diagonal up
    # to the Hessian tolerance); the factor is computed once (reversed route,
    # pinned equal to the direct one)
    sel = np.sort(rng.choice(len(qrows), n_rows, replace=False))
    rows = qrows[sel]
    Wr = Wp[sel]
    pg = perm.cpu().numpy()
    if spec.act_order:
        dg = np.diag(H)[pg]
        rise = np.maximum(dg[1:] - dg[:-1], 0.0)
        assert np.all(rise <= 1e-4 * dg[:-1]), float(np.max(rise / dg[:-1]))
    else:
        assert np.array_equal(pg, np.arange(n))
    prep = oracle.gptq_prepare(Wr, H, spec.damp, spec.act_order, perm=pg)
    U = oracle.inv_chol_upper_reversed(prep["Hd"])
    del prep
    cg = oracle.unpack_codes(codes.cpu().numpy()[rows].view(np.uint32), spec.wbits, n)
    sg, zg = scales.cpu().numpy()[rows], zeros.cpu().numpy()[rows]
    st = oracle.teacher_forced_check(Wr, H, spec.wbits, G, spec.damp, spec.act_order, cg, sg, zg,
                                     perm=pg, U=U)
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= 1e-5, st
    ref = oracle.gptq_quantize(Wr, H, spec.wbits, G, spec.damp, spec.act_order, perm=pg, U=U)
    assert cg.size >= 100_000
    plain = plain_identity(cg, ref["codes"])
    forced = 1.0 - st["n_mismatch"] / st["n_codes"]
    # Layer output error ||(W - Q) X^T||_F of these rows within 1% of the
    # oracle's, Q the dequantised codes (original column order)
    X64 = L["X"][: min(spec.n_tok, 16384)].float().cpu().numpy()
    Wo = W[rows]
    deq_g = np.repeat(sg, G, axis=1) * (cg - np.repeat(zg, G, axis=1))
    e_g = oracle.layer_errors(Wo, deq_g, X64, X64)["e_lit"]
    e_o = oracle.layer_errors(Wo, ref["deq"], X64, X64)["e_lit"]
    del X64
    log_numbers(name, n_tok=spec.n_tok, h_rel=h_rel, w_err_over_max_w=w_err, corr_rel=c_err,
                scale_max_rel=st["scale_max_rel"], plain_identity=plain, forced_identity=forced,
                mismatches=st["n_mismatch"], codes=int(cg.size), e_lit_rel=abs(e_g - e_o) / e_o)
    assert abs(e_g - e_o) <= 0.01 * e_o, (e_g, e_o)
    # Code identity: >= 99.9% counted on the replay with the candidate's
    # earlier decisions forced in (each mismatch is a boundary case, above).
    # A plain count would also count the cascade after each legitimate flip:
    # one flip changes the error fed to every later column of its row.
    assert forced >= 0.999, (plain, forced, st)
    return {"spec": spec, "H": H, "Wr": Wr, "pg": pg, "U": U}


def check_identical_inputs(spec, ctx):
    """The GPTQ call alone on the sampled rows, given the oracle's W' and H as
    its fp32 inputs: scales within 1e-5 of the oracle's on identical inputs."""
    n, G = spec.d_in, spec.groupsize
    H, Wr, pg, U = ctx["H"], ctx["Wr"], ctx["pg"], ctx["U"]
    H32, W32 = H.astype(np.float32), Wr.astype(np.float32)
    c2, s2, z2, p2 = oc.oc_gptq_quantize(
        torch.from_numpy(W32).cuda(), torch.from_numpy(H32).cuda(), spec.wbits, G, spec.damp,
        spec.act_order, perm_out=torch.empty(n, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    p2 = p2.cpu().numpy()
    H64 = H32.astype(np.float64)
    if np.array_equal(p2, pg):
        # same order: H64 differs from H by fp32 rounding only (~1e-7 of the
        # factor), far below the 1e-3 boundary bar, so the factor is reused
        U2 = U
    else:
        prep = oracle.gptq_prepare(W32, H64, spec.damp, spec.act_order, perm=p2)
        U2 = oracle.inv_chol_upper_reversed(prep["Hd"])
        del prep
    c2 = oracle.unpack_codes(c2.cpu().numpy().view(np.uint32), spec.wbits, n)
    st2 = oracle.teacher_forced_check(W32.astype(np.float64), H64, spec.wbits, G, spec.damp,
                                      spec.act_order, c2, s2.cpu().numpy(), z2.cpu().numpy(),
                                      perm=p2, U=U2)
    assert st2["n_bad"] == 0 and st2["zero_bad"] == 0, st2
    assert st2["scale_max_rel"] <= 1e-5, st2
    assert 1.0 - st2["n_mismatch"] / st2["n_codes"] >= 0.999, st2


@pytest.mark.parametrize("name", list(CASES))
def test_large_layer_matches_oracle(name):
    T, n_rows, qep_rows = CASES[name]
    spec = CONFIGS[name].with_(n_tok=T)
    ctx = check_layer(name, spec, n_rows, qep_rows)
    check_identical_inputs(spec, ctx)


def test_gate_up_shape_full_calibration_matches_oracle():
    # d_in 4096 -> d_out 11008, 3-bit g128, act_order off, all 131072 tokens
    spec = gate_spec()
    assert (spec.d_in, spec.d_out, spec.n_tok, spec.wbits, spec.groupsize) == (4096, 11008, 131072, 3, 128)
    ctx = check_layer("gate_4096_11008", spec, n_rows=32, qep_rows=None)
    check_identical_inputs(spec, ctx)


@pytest.mark.parametrize("name", list(CASES))
def test_large_layer_full_size(name):
    spec = CONFIGS[name]
    m, n, G = spec.d_out, spec.d_in, spec.groupsize
    L = make_layer_device(spec, "cuda")
    Hg, Wg, codes, scales, zeros, perm = run_fused(spec, L)
    assert oc.oc_stream_status(None) == oc.OC_OK
    # Hessian entries from sampled Xhat columns (outlier channels included),
    # each against the float64 dot product over all tokens
    rng = np.random.default_rng(5)
    outl = L["outliers"].cpu().numpy()
    ii = np.concatenate([rng.integers(0, n, 24), outl[:8], rng.integers(0, n, 8)])
    jj = np.concatenate([rng.integers(0, n, 24), outl[-8:], rng.integers(0, n, 8)])
    jj[-8:] = ii[-8:]
    cols = np.unique(np.concatenate([ii, jj]))
    C = np.zeros((spec.n_tok, len(cols)))
    for t0 in range(0, spec.n_tok, CHUNK):
        C[t0:t0 + CHUNK] = L["Xhat"][t0:t0 + CHUNK][:, torch.from_numpy(cols).cuda()].float().cpu().numpy()
    pos = {c: k for k, c in enumerate(cols)}
    Hs = Hg[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].cpu().numpy().astype(np.float64)
    diag = 2.0 * np.sum(C * C, axis=0)
    ref = np.array([2.0 * float(C[:, pos[i]] @ C[:, pos[j]]) for i, j in zip(ii, jj)])
    scale = np.sqrt([diag[pos[i]] * diag[pos[j]] for i, j in zip(ii, jj)])
    assert np.abs(Hs - ref).max() <= 1e-4 * scale.max()
    assert float(np.max(np.abs(Hs - ref) / scale)) <= 1e-4
    # invariants of the outputs
    assert bool(torch.isfinite(Wg).all())
    maxq = (1 << spec.wbits) - 1
    cg = oracle.unpack_codes(codes[:64].cpu().numpy().view(np.uint32), spec.wbits, n)
    assert cg.min() >= 0 and cg.max() <= maxq
    s, z = scales.cpu().numpy(), zeros.cpu().numpy()
    assert np.all(s > 0) and np.all(np.isfinite(s))
    assert np.all(z == np.rint(z)) and z.min() >= 0 and z.max() <= maxq
    pg = perm.cpu().numpy()
    assert np.array_equal(np.sort(pg), np.arange(n))
    # act_order: processing order by decreasing Hessian diagonal
    dg = torch.diagonal(Hg).cpu().numpy()
    assert np.all(np.diff(dg[pg]) <= 0)
