"""Parity at the full size of the Llama-2-7B q_proj workload (d_in = d_out =
4096, 262144 calibration tokens), in the launch configuration bench.py times.

The float64 oracle cannot redo the whole layer here, so the checks use outputs
it can compute one by one or properties that hold at any size:
  * Hessian: sampled entries recomputed from the Xhat columns in float64;
  * GPTQ: sampled rows replayed by the oracle with the GPU's Hessian (teacher
    forcing, scale and zero tolerances, plain code identity on those rows);
  * QEP: the normal equations of the least-squares problem,
    (W X^T - W' Xhat^T) Xhat = lam (W' - W) at alpha = 1, on sampled rows,
    streamed over all tokens.  An error E in W' leaves the residual
    -E (Xhat^T Xhat + lam I); the test maps the residual back through that
    matrix (taken from the GPU's H, itself within 1e-5 of exact) and bounds E.
"""
import numpy as np
import pytest

import oracle
from synthetic import CONFIGS, make_layer_device

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

SPEC = CONFIGS["c2_q_proj"]


@pytest.fixture(scope="module")
def layer():
    L = make_layer_device(SPEC, "cuda")
    H = torch.zeros(SPEC.d_in, SPEC.d_in, device="cuda")
    oc.oc_hessian_accumulate(L["Xhat"], H)
    torch.cuda.synchronize()
    return L, H


def test_fullsize_hessian_sampled_entries(layer):
    L, H = layer
    Xh = L["Xhat"]
    n = SPEC.d_in
    rng = np.random.default_rng(0)
    outl = L["outliers"].cpu().numpy()
    ii = np.concatenate([rng.integers(0, n, 40), outl[:8], rng.integers(0, n, 8)])
    jj = np.concatenate([rng.integers(0, n, 40), outl[:8], rng.integers(0, n, 8)])
    jj[-8:] = ii[-8:]  # some diagonal entries
    cols = np.unique(np.concatenate([ii, jj]))
    C = Xh[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    pos = {c: k for k, c in enumerate(cols)}
    Hg = H.cpu().numpy()
    assert np.array_equal(Hg, Hg.T)
    diag = 2.0 * np.sum(C * C, axis=0)
    err2 = ref2 = 0.0
    worst = 0.0
    for i, j in zip(ii, jj):
        ref = 2.0 * float(C[:, pos[i]] @ C[:, pos[j]])
        worst = max(worst, abs(Hg[i, j] - ref) / np.sqrt(diag[pos[i]] * diag[pos[j]]))
        err2 += (Hg[i, j] - ref) ** 2
        ref2 += ref ** 2
    # The sample over-weights the diagonal (where fp32 accumulation error is
    # largest relative to the entry), so its relative Frobenius error bounds
    # the matrix-wide one from above; the bar is 1e-4.
    assert np.sqrt(err2 / ref2) <= 1e-4, np.sqrt(err2 / ref2)
    assert worst <= 1e-4, worst


def test_fullsize_gptq_sampled_rows(layer):
    L, H = layer
    m, n = SPEC.d_out, SPEC.d_in
    W = L["W"]
    codes, scales, zeros, _ = oc.oc_gptq_quantize(W, H, SPEC.wbits, SPEC.groupsize, SPEC.damp,
                                                  SPEC.act_order)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(m, 32, replace=False))
    Hh = H.cpu().numpy().astype(np.float64)
    Wr = W.cpu().numpy()[rows].astype(np.float64)
    cg = oracle.unpack_codes(codes.cpu().numpy()[rows].view(np.uint32), SPEC.wbits, n)
    sg = scales.cpu().numpy()[rows]
    zg = zeros.cpu().numpy()[rows]
    st = oracle.teacher_forced_check(Wr, Hh, SPEC.wbits, SPEC.groupsize, SPEC.damp,
                                     SPEC.act_order, cg, sg, zg)
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= 1e-5, st
    ref = oracle.gptq_quantize(Wr, Hh, SPEC.wbits, SPEC.groupsize, SPEC.damp, SPEC.act_order)
    G = SPEC.groupsize
    za, zb = np.repeat(zg, G, axis=1), np.repeat(ref["zeros"], G, axis=1)
    same = za == zb
    ident = float(np.mean((cg - za)[same] == (ref["codes"] - zb)[same]))
    assert cg.size >= 100_000 and ident >= 0.999, (ident, st)


def test_fullsize_qep_normal_equations(layer):
    L, H = layer
    W, X, Xh = L["W"], L["X"], L["Xhat"]
    damp = SPEC.damp
    W1 = oc.oc_qep_correct(W, X, Xh, 1.0, damp, H_opt=H)
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.random.default_rng(2).choice(SPEC.d_out, 4, replace=False)).cuda()
    Wr = W[rows].double().cpu().numpy()
    W1r = W1[rows].double().cpu().numpy()
    n = SPEC.d_in
    lhs = np.zeros((4, n))
    diag = np.zeros(n)
    for t0 in range(0, SPEC.n_tok, 16384):
        xc = X[t0:t0 + 16384].float().cpu().numpy().astype(np.float64)
        hc = Xh[t0:t0 + 16384].float().cpu().numpy().astype(np.float64)
        a = Wr @ xc.T - W1r @ hc.T
        lhs += a @ hc
        diag += np.sum(hc * hc, axis=0)
    lam = damp * diag.mean()
    resid = lhs - lam * (W1r - Wr)
    A = H.double().cpu().numpy() / 2.0 + lam * np.eye(n)
    import scipy.linalg as sla
    E = -sla.cho_solve(sla.cho_factor(A), resid.T).T
    corr = W1r - Wr
    # the correction itself to within 1% and W' to within 1e-5 of max |W|
    assert np.linalg.norm(E) <= 1e-2 * np.linalg.norm(corr), (np.linalg.norm(E), np.linalg.norm(corr))
    assert np.abs(E).max() <= 1e-5 * np.abs(Wr).max()
