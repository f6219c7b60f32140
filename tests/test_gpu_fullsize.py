"""Parity at the full size of the Llama-2-7B q_proj workload (d_in = d_out =
4096, 262144 calibration tokens), through the fused layer call that bench.py
times, in its launch configuration.

Every expected value comes from the float64 oracle fed the same seeded bf16
inputs: the Hessian H = 2 Xh^T Xh and the cross term d = (X - Xh)^T Xh are
accumulated by oracle.hessian / oracle.qep_cross over 8192-token chunks
streamed from the device (both are sums over tokens), and everything after
them is the oracle's own arithmetic:
  * Hessian: the whole matrix, relative Frobenius error;
  * QEP: the corrected weight W' of every row, against oracle.qep_correct;
  * GPTQ: sampled rows replayed by the oracle from its own W' and H (teacher
    forcing, scale and zero tolerances, plain code identity on those rows).
The same checks run on the standalone GPTQ call given the oracle's W' and H
rounded to fp32, so that its scales are compared on identical inputs.
"""
import numpy as np
import pytest

import oracle
from synthetic import CONFIGS, make_layer_device

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

SPEC = CONFIGS["q_proj_4096"]
CHUNK = 8192
N_ROWS = 32  # rows replayed by the oracle sweep


@pytest.fixture(scope="module")
def layer():
    return make_layer_device(SPEC, "cuda")


@pytest.fixture(scope="module")
def oracle_terms(layer):
    """(H, d) of the whole calibration set, float64, from the oracle."""
    X, Xh = layer["X"], layer["Xhat"]
    n = SPEC.d_in
    H = np.zeros((n, n))
    d = np.zeros((n, n))
    for t0 in range(0, SPEC.n_tok, CHUNK):
        xc = X[t0:t0 + CHUNK].float().cpu().numpy()
        hc = Xh[t0:t0 + CHUNK].float().cpu().numpy()
        H = oracle.hessian(hc, H0=H)
        d += oracle.qep_cross(xc, hc)
    return H, d


@pytest.fixture(scope="module")
def fused(layer):
    """One fused layer call at full size, as bench.py launches it."""
    W, X, Xh = layer["W"], layer["X"], layer["Xhat"]
    m, n, G = SPEC.d_out, SPEC.d_in, SPEC.groupsize
    H = torch.zeros(n, n, device="cuda")
    W_out = torch.empty_like(W)
    codes = torch.empty(m, n * SPEC.wbits // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(m, n // G, device="cuda")
    zeros = torch.empty(m, n // G, device="cuda")
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    oc.oc_quantize_layer(W, X, Xh, SPEC.alpha, SPEC.damp, SPEC.wbits, SPEC.groupsize,
                         SPEC.act_order, H=H, W_out=W_out, codes=codes, scales=scales,
                         zeros=zeros, perm_out=perm)
    torch.cuda.synchronize()
    return {"H": H.cpu().numpy(), "W_out": W_out.cpu().numpy(), "codes": codes.cpu().numpy(),
            "scales": scales.cpu().numpy(), "zeros": zeros.cpu().numpy(),
            "perm": perm.cpu().numpy()}


@pytest.fixture(scope="module")
def oracle_wprime(layer, oracle_terms):
    H, d = oracle_terms
    W = layer["W"].cpu().numpy().astype(np.float64)
    return oracle.qep_correct(W, None, None, SPEC.alpha, SPEC.damp, H=H, d=d)


def rel_fro(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def test_fullsize_hessian_whole_matrix(fused, oracle_terms):
    H, _ = oracle_terms
    Hg = fused["H"]
    assert np.array_equal(Hg, Hg.T)
    assert rel_fro(Hg, H) <= 1e-4, rel_fro(Hg, H)


def test_fullsize_hessian_standalone_call(layer, oracle_terms):
    H, _ = oracle_terms
    Hg = torch.zeros(SPEC.d_in, SPEC.d_in, device="cuda")
    oc.oc_hessian_accumulate(layer["Xhat"], Hg)
    torch.cuda.synchronize()
    assert rel_fro(Hg.cpu().numpy(), H) <= 1e-4


def test_fullsize_qep_every_row(layer, fused, oracle_wprime):
    W = layer["W"].cpu().numpy().astype(np.float64)
    E = fused["W_out"] - oracle_wprime
    corr = oracle_wprime - W
    # the correction to within 1% (Frobenius) and every weight to within
    # 1e-5 of max |W|
    assert np.linalg.norm(E) <= 1e-2 * np.linalg.norm(corr), (np.linalg.norm(E), np.linalg.norm(corr))
    assert np.abs(E).max() <= 1e-5 * np.abs(W).max(), np.abs(E).max()


def _check_rows(Wp_rows, H, codes, scales, zeros, perm):
    """Teacher-forced replay and code identity of a few rows (oracle inputs)."""
    n = SPEC.d_in
    cg = oracle.unpack_codes(codes.view(np.uint32), SPEC.wbits, n)
    st = oracle.teacher_forced_check(Wp_rows, H, SPEC.wbits, SPEC.groupsize, SPEC.damp,
                                     SPEC.act_order, cg, scales, zeros, perm=perm)
    ref = oracle.gptq_quantize(Wp_rows, H, SPEC.wbits, SPEC.groupsize, SPEC.damp, SPEC.act_order)
    G = SPEC.groupsize
    za, zb = np.repeat(zeros, G, axis=1), np.repeat(ref["zeros"], G, axis=1)
    same = za == zb
    ident = float(np.mean((cg - za)[same] == (ref["codes"] - zb)[same]))
    return st, ident, cg.size


def test_fullsize_gptq_sampled_rows_fused(fused, oracle_terms, oracle_wprime):
    H, _ = oracle_terms
    rows = np.sort(np.random.default_rng(1).choice(SPEC.d_out, N_ROWS, replace=False))
    st, ident, size = _check_rows(oracle_wprime[rows], H, fused["codes"][rows],
                                  fused["scales"][rows], fused["zeros"][rows], fused["perm"])
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= 1e-5, st
    assert size >= 100_000 and ident >= 0.999, (ident, st)


def test_fullsize_gptq_standalone_on_oracle_inputs(oracle_terms, oracle_wprime):
    # The GPTQ call alone, given the oracle's W' and H (rounded to fp32, the
    # call's input type); the oracle replays the same fp32 values.
    H, _ = oracle_terms
    H32 = H.astype(np.float32)
    W32 = oracle_wprime.astype(np.float32)
    codes, scales, zeros, perm = oc.oc_gptq_quantize(
        torch.from_numpy(W32).cuda(), torch.from_numpy(H32).cuda(), SPEC.wbits, SPEC.groupsize,
        SPEC.damp, SPEC.act_order, perm_out=torch.empty(SPEC.d_in, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(4).choice(SPEC.d_out, N_ROWS, replace=False))
    st, ident, size = _check_rows(W32[rows].astype(np.float64), H32.astype(np.float64),
                                  codes.cpu().numpy()[rows], scales.cpu().numpy()[rows],
                                  zeros.cpu().numpy()[rows], perm.cpu().numpy())
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= 1e-5, st
    assert size >= 100_000 and ident >= 0.999, (ident, st)
