"""LPCD on the GPU against the float64 oracle: the relaxed first-layer step
(oc_lpcd_left_project) element by element, and the two-layer submodule loop
(lpcd_pair) step by step with the GPU's own quantised second layer fed to the
oracle (the loop's GPTQ projections are GPTQ calls whose parity the layer tests
cover)."""
import numpy as np
import pytest

import oracle
from synthetic import random_layer_host

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

# max |GPU - oracle| over max |oracle| for the relaxed step: 3xTF32 products
# (about fp32) and an fp32 factorisation of B^T B + mu I, so the error grows
# with that matrix's condition number kappa: allowed c * kappa * u with the
# fp32 unit roundoff u = 2^-24 and a growth constant c = 64
def left_tol(B, damp):
    M = np.asarray(B, np.float64).T @ np.asarray(B, np.float64)
    M += damp * np.mean(np.diag(M)) * np.eye(M.shape[0])
    ev = np.linalg.eigvalsh(M)
    return 64.0 * (ev[-1] / ev[0]) * 2.0 ** -24


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(torch.bfloat16)


def _left_case(m, d, n, seed):
    rng = np.random.default_rng(seed)
    B = rng.standard_normal((m, d)).astype(np.float32)
    W2 = (B + 0.05 * rng.standard_normal((m, d))).astype(np.float32)
    V = rng.standard_normal((d, n)).astype(np.float32)
    return B, W2, V


@pytest.mark.parametrize("m,d,n,damp", [
    (256, 192, 320, 0.01),
    (4, 64, 8, 0.05),        # B of rank 4: only the damping makes B^T B + mu I definite
    (2048, 1024, 516, 0.01),  # a factorisation with tensor-core products, ragged n
])
def test_left_project_matches_oracle(m, d, n, damp):
    B, W2, V = _left_case(m, d, n, seed=m + d + n)
    got = oc.oc_lpcd_left_project(dev(B), dev(W2), dev(V), damp).cpu().numpy()
    ref = oracle.lpcd_left_project(B, W2, V, damp)
    assert np.max(np.abs(got - ref)) <= left_tol(B, damp) * np.max(np.abs(ref))


def test_left_project_in_place_and_bad_sizes():
    B, W2, V = _left_case(128, 128, 64, seed=9)
    out = oc.oc_lpcd_left_project(dev(B), dev(W2), dev(V), 0.01)
    Vd = dev(V)
    oc.oc_lpcd_left_project(dev(B), dev(W2), Vd, 0.01, W_out=Vd)
    assert torch.equal(out, Vd)
    with pytest.raises(oc.OcError) as e:
        oc.oc_lpcd_left_project(dev(B[:, :100]), dev(W2[:, :100]), dev(V[:100]), 0.01)
    assert e.value.status == oc.OC_ERR_INVALID_ARG
    with pytest.raises(oc.OcError) as e:
        oc.oc_lpcd_left_project(dev(B), dev(W2), dev(V), -1.0)
    assert e.value.status == oc.OC_ERR_INVALID_ARG


def _submodule(n=256, d=192, m=128, N=4096, seed=41):
    L1 = random_layer_host(d, n, N, seed=seed)
    L2 = random_layer_host(m, d, 8, seed=seed + 1)
    return L1["W"].astype(np.float64), L2["W"].astype(np.float64), L1["X"], L1["Xhat"]


@pytest.mark.parametrize("wbits,G", [(4, 64), (3, 32)])
def test_lpcd_pair_steps_match_oracle(wbits, G):
    W1, W2, X, Xh = _submodule()
    damp = 0.01
    r = oc.lpcd_pair(dev(W1), dev(W2), bf16_dev(X), bf16_dev(Xh), 0.5, damp, wbits, G, False, rounds=2)
    torch.cuda.synchronize()
    # QEP with alpha = 1 of the first layer (the relaxed step's right factor)
    V1 = oracle.qep_correct(W1, X, Xh, 1.0, damp)
    assert np.max(np.abs(r["V1"].cpu().numpy() - V1)) <= 1e-4 * np.max(np.abs(W1))
    # every round's relaxed first layer, against the quantised second layer it used
    for Ws, Q2 in zip(r["W1_star"], r["Q2_used"]):
        ref = oracle.lpcd_left_project(Q2.cpu().numpy(), W2, V1, damp)
        got = Ws.cpu().numpy()
        assert np.max(np.abs(got - ref)) <= 1e-3 * np.max(np.abs(ref))
    # the dequantised layers are the returned codes' values
    c1, s1, z1, _ = r["q1"]
    Q1 = oracle.dequantize(c1.cpu().numpy().view(np.uint32), s1.cpu().numpy(), z1.cpu().numpy(), wbits, G,
                           W1.shape[1])
    assert np.allclose(r["Q1"].cpu().numpy(), Q1, rtol=0, atol=1e-6 * np.max(np.abs(Q1)))


def test_lpcd_pair_round_improves_on_the_layer_wise_start():
    W1, W2, X, Xh = _submodule(seed=43)
    r = oc.lpcd_pair(dev(W1), dev(W2), bf16_dev(X), bf16_dev(Xh), 0.5, 0.01, 3, 64, False, rounds=1)
    ref = oracle.lpcd_pair(W1, W2, X, Xh, 0.5, 0.01, 3, 64, False, rounds=1)
    e_gpu = np.array(r["errors"]) / r["ref"]
    e_ref = np.array(ref["errors"]) / ref["ref"]
    assert e_gpu[1] < 0.7 * e_gpu[0]
    # same quality as the oracle's run of the same method (decisions near
    # rounding ties may differ, so the errors agree only approximately)
    assert np.all(np.abs(e_gpu - e_ref) <= 0.1 * e_ref)
