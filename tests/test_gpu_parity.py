"""GPU parity: the CUDA path (called through the C ABI) against the float64
oracle on the same seeded inputs.

Tolerances (the quantisation workload's stated bars):
  Hessian           relative Frobenius error <= 1e-4 (oracle fed the same bf16 inputs);
  codes             >= 99.9% identical, and every mismatch, replayed with the
                    candidate's earlier decisions forced in, lies within 1e-3 of a
                    rounding boundary (in units of the scale).  Identity is counted
                    on the integer levels q - zero over the groups whose zero point
                    both sides chose alike: a zero decided at a rounding boundary
                    (allowed by the zero tolerance) shifts its whole group;
  scales / zeros    relative error <= 1e-5 (zeros: equal unless -min/scale sits
                    within 1e-3 of a rounding boundary);
  layer error       ||(W - Q) X^T||_F within 1% of the oracle's.
QEP output: max |W'_gpu - W'_oracle| <= 1e-5 * max |W|.  The library forms the
cross term from D = bf16(X - Xhat), each difference rounded once (relative
error <= 2^-9, of random sign), so the correction W' - W carries about 1e-3 of
its own size from that rounding, plus fp32 accumulation and the fp32 factor;
on these layers the correction is a few percent of W at most.
"""
import numpy as np
import pytest

import oracle
from synthetic import CONFIGS, make_layer_host, random_layer_host

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

H_TOL = 1e-4
SCALE_TOL = 1e-5
CODE_FRAC = 0.999
BOUNDARY = 1e-3
QEP_TOL = 1e-5


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def bf16_dev(a):
    # values are already bf16-representable (synthetic rounds them): exact cast
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(torch.bfloat16)


def rel_fro(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def gpu_hessian(xhat_np, H0=None):
    n = xhat_np.shape[1]
    H = dev(np.zeros((n, n)) if H0 is None else H0)
    oc.oc_hessian_accumulate(bf16_dev(xhat_np), H)
    torch.cuda.synchronize()
    return H.cpu().numpy()


# ----------------------------------------------------------------------------- Hessian

@pytest.mark.parametrize("n,n_tok", [(64, 100), (256, 1000), (384, 777), (512, 2048), (640, 4096 + 33)])
def test_hessian_matches_oracle(n, n_tok):
    L = random_layer_host(8, n, n_tok, seed=100 + n)
    Hg = gpu_hessian(L["Xhat"])
    Ho = oracle.hessian(L["Xhat"])
    assert rel_fro(Hg, Ho) <= H_TOL
    assert np.array_equal(Hg, Hg.T)


def test_bounded_wait_runs_out_and_the_library_recovers():
    # A barrier nothing releases (oc_test_inject_stall): the kernel's bounded
    # wait gives up, the call reports OC_ERR_TIMEOUT, and the next call runs
    # normally on the same device.
    L = random_layer_host(8, 256, 1000, seed=104)
    H = dev(np.zeros((256, 256)))
    oc.oc_test_inject_stall()
    with pytest.raises(oc.OcError) as e:
        oc.oc_hessian_accumulate(bf16_dev(L["Xhat"]), H)
    assert e.value.status == oc.OC_ERR_TIMEOUT
    assert oc.oc_stream_status(None) == oc.OC_OK   # the error was collected once
    Hg = gpu_hessian(L["Xhat"])
    assert rel_fro(Hg, oracle.hessian(L["Xhat"])) <= H_TOL


def test_hessian_accumulates_and_ignores_empty():
    L = random_layer_host(8, 256, 1500, seed=7)
    H1 = gpu_hessian(L["Xhat"][:700])
    H2 = gpu_hessian(L["Xhat"][700:], H0=H1)
    Ho = oracle.hessian(L["Xhat"])
    assert rel_fro(H2, Ho) <= H_TOL
    H = dev(H2)
    oc.oc_hessian_accumulate(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), H)
    assert np.array_equal(H.cpu().numpy(), H2)


# ----------------------------------------------------------------------------- QEP

def _qep_case(n=256, m=96, n_tok=3000, seed=11):
    L = random_layer_host(m, n, n_tok, seed=seed)
    return L["W"], L["X"], L["Xhat"]


@pytest.mark.parametrize("use_h", [False, True])
@pytest.mark.parametrize("shape", [(96, 256, 3000), (512, 512, 2048), (130, 384, 1111)])
def test_qep_matches_oracle(use_h, shape):
    m, n, n_tok = shape
    W, X, Xh = _qep_case(n=n, m=m, n_tok=n_tok, seed=m + n)
    alpha, damp = 0.5, 0.01
    Ho = oracle.hessian(Xh)
    Wo = oracle.qep_correct(W, X, Xh, alpha, damp, H=Ho)
    Hg = dev(gpu_hessian(Xh)) if use_h else None
    Wg = oc.oc_qep_correct(dev(W), bf16_dev(X), bf16_dev(Xh), alpha, damp, H_opt=Hg).cpu().numpy()
    err = np.abs(Wg - Wo).max()
    corr = np.abs(Wo - W).max()
    assert err <= QEP_TOL * np.abs(W).max(), (err, corr)
    # the correction itself is reproduced to a small fraction of its size
    assert np.abs((Wg - W) - (Wo - W)).max() <= 2e-3 * corr


def _large_channel(X, Xh, channel=5):
    # one channel scaled by 2^15 (exact in bf16): its values pass fp16's
    # largest finite 65504, which the per-feature scales of the cross
    # product's fp16 operands must absorb
    X, Xh = X.copy(), Xh.copy()
    X[:, channel] *= 32768.0
    Xh[:, channel] *= 32768.0
    assert np.abs(Xh).max() > 65504.0
    return X, Xh


def _far_difference(X, Xh, channel=5, token=17):
    # one value of X far from Xhat's: X - Xhat there exceeds 4 times the
    # column's norm sqrt(sum_t Xhat^2), beyond what the fp16 scale taken from
    # the Hessian diagonal allows, so the cross product must take its bf16 path
    X = X.copy()
    r = float(np.sqrt(np.sum(Xh[:, channel].astype(np.float64) ** 2)))
    X[token, channel] = oracle._bf16(np.array([Xh[token, channel] + 64.0 * r]))[0]
    return X, Xh


@pytest.mark.parametrize("use_h", [False, True])
@pytest.mark.parametrize("case", ["large_channel", "far_difference"])
def test_qep_cross_operands_outside_fp16_range(use_h, case):
    W, X, Xh = _qep_case(n=256, m=96, n_tok=3000, seed=19)
    X, Xh = (_large_channel if case == "large_channel" else _far_difference)(X, Xh)
    Ho = oracle.hessian(Xh)
    Wo = oracle.qep_correct(W, X, Xh, 0.5, 0.01, H=Ho)
    Hg = dev(gpu_hessian(Xh)) if use_h else None
    Wg = oc.oc_qep_correct(dev(W), bf16_dev(X), bf16_dev(Xh), 0.5, 0.01, H_opt=Hg).cpu().numpy()
    assert np.all(np.isfinite(Wg))
    E, corr = Wg - Wo, Wo - W
    if case == "large_channel":
        # scaled fp16 operands: D to 11 significant bits
        assert np.abs(E).max() <= QEP_TOL * np.abs(W).max()
        assert np.linalg.norm(E) <= 2e-3 * np.linalg.norm(corr), np.linalg.norm(E) / np.linalg.norm(corr)
    else:
        # bf16 operands: D to 8 significant bits, about 1e-3 of the correction,
        # which the planted difference makes as large as W itself
        assert np.abs(E).max() <= 5e-3 * np.abs(corr).max(), np.abs(E).max() / np.abs(corr).max()
        assert np.linalg.norm(E) <= 5e-3 * np.linalg.norm(corr), np.linalg.norm(E) / np.linalg.norm(corr)


def test_qep_alpha_zero_is_identity_bitwise():
    W, X, Xh = _qep_case()
    Wd = dev(W)
    out = oc.oc_qep_correct(Wd, bf16_dev(X), bf16_dev(Xh), 0.0, 0.01)
    assert torch.equal(out, Wd)
    same = oc.oc_qep_correct(Wd, bf16_dev(X), bf16_dev(Xh), 0.0, 0.01, W_out=Wd)
    assert torch.equal(same, dev(W))


def test_qep_identical_inputs_leave_w():
    W, X, _ = _qep_case()
    out = oc.oc_qep_correct(dev(W), bf16_dev(X), bf16_dev(X), 0.5, 0.01).cpu().numpy()
    assert np.abs(out - W).max() <= 1e-6 * np.abs(W).max()


def test_qep_in_place():
    W, X, Xh = _qep_case()
    Wd = dev(W)
    ref = oc.oc_qep_correct(Wd, bf16_dev(X), bf16_dev(Xh), 0.5, 0.01).clone()
    oc.oc_qep_correct(Wd, bf16_dev(X), bf16_dev(Xh), 0.5, 0.01, W_out=Wd)
    assert torch.allclose(Wd, ref, rtol=0, atol=1e-7)


# ----------------------------------------------------------------------------- GPTQ

def gpu_gptq(W, H, wbits, G, damp, act_order):
    m, n = W.shape
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    codes, scales, zeros, _ = oc.oc_gptq_quantize(dev(W), dev(H), wbits, G, damp, act_order,
                                                  perm_out=perm)
    torch.cuda.synchronize()
    words = codes.cpu().numpy().view(np.uint32)
    return (oracle.unpack_codes(words, wbits, n), scales.cpu().numpy(), zeros.cpu().numpy(),
            perm.cpu().numpy(), words)


def code_frac_for(n_codes):
    """The 99.9% identity bar applies to workload-sized matrices.  One decision
    taken legitimately on the other side of a rounding boundary (teacher forcing
    checks each) changes the later feedback of its row, and on a unit-test
    matrix of a few thousand codes that one row can exceed 0.1%; there the bar
    is 99% and the teacher-forced checks carry the parity."""
    return CODE_FRAC if n_codes >= 100_000 else 0.99


def level_identity(codes_a, zeros_a, codes_b, zeros_b, G):
    """Fraction of identical integer levels q - zero, over the groups whose
    zero point both sides chose alike.  A zero decided at a rounding boundary
    (judged separately by the zero tolerance) moves every level of its group
    that meets the clamp; those groups are left out of the count."""
    n = codes_a.shape[1]
    G = n if G == -1 else G
    za = np.repeat(zeros_a, G, axis=1)
    zb = np.repeat(zeros_b, G, axis=1)
    same = za == zb
    if not same.any():
        return 1.0
    return float(np.mean((codes_a - za)[same] == (codes_b - zb)[same]))


def oracle_block(n, G):
    """The oracle's lazy-batch width: 256, or GPTQ's 128 where a group wider
    than 128 does not tile 256 (a dynamic group must start at a block start or
    lie inside one block)."""
    Gn = n if G == -1 else G
    return 256 if (256 % Gn == 0 or Gn % 256 == 0 or Gn == n) else 128


def check_gptq(W, H, wbits, G, damp, act_order, gpu=None):
    codes, scales, zeros, perm, words = gpu if gpu is not None else gpu_gptq(W, H, wbits, G, damp, act_order)
    blk = oracle_block(W.shape[1], G)
    ref = oracle.gptq_quantize(W, H, wbits, G, damp, act_order, block=blk)
    assert np.array_equal(perm, ref["perm"])
    ident = level_identity(codes, zeros, ref["codes"], ref["zeros"], G)
    st = oracle.teacher_forced_check(W, H, wbits, G, damp, act_order, codes, scales, zeros, perm=perm,
                                     block=blk)
    assert st["n_bad"] == 0, st
    assert st["scale_max_rel"] <= SCALE_TOL, st
    assert st["zero_bad"] == 0, st
    assert ident >= code_frac_for(codes.size), (ident, st)
    assert np.array_equal(words, ref["packed"]) or ident < 1.0
    return ident, st


@pytest.mark.parametrize("m,n,wbits,G,act", [
    (512, 512, 4, 128, False),   # the 512 x 512 workload's settings
    (200, 384, 3, 64, True),
    (96, 320, 2, 32, False),     # ragged last block (64 columns)
    (64, 512, 4, 256, False),    # group wider than a block
    (64, 256, 3, -1, True),
    (33, 192, 4, -1, False),     # one group of 192 columns across two blocks
    (7, 128, 2, 4, False),       # tiny groups, fewer rows than a CTA's warps
    (40, 1536, 4, 384, False),   # groups that start inside a 512-column superblock
    (24, 1536, 3, 768, False),   # and ones that cross into the next superblock
])
def test_gptq_matches_oracle(m, n, wbits, G, act):
    L = random_layer_host(m, n, max(2 * n, 512), seed=1000 + m + n)
    H = oracle.hessian(L["Xhat"]).astype(np.float32).astype(np.float64)
    check_gptq(L["W"].astype(np.float64), H, wbits, G, 0.01, act)


@pytest.mark.parametrize("m,n,wbits,G,act", [
    (256, 1024, 4, 128, False),
    (192, 2048, 3, 128, True),   # halves of 1024: the factor's large products on the tensor cores
])
def test_gptq_matches_oracle_large_factor(m, n, wbits, G, act):
    L = random_layer_host(m, n, 2 * n, seed=2000 + n)
    H = oracle.hessian(L["Xhat"]).astype(np.float32).astype(np.float64)
    check_gptq(L["W"].astype(np.float64), H, wbits, G, 0.01, act)


def test_qep_matches_oracle_large_factor():
    W, X, Xh = _qep_case(n=1024, m=128, n_tok=4096, seed=77)
    Ho = oracle.hessian(Xh)
    Wo = oracle.qep_correct(W, X, Xh, 0.5, 0.01, H=Ho)
    Wg = oc.oc_qep_correct(dev(W), bf16_dev(X), bf16_dev(Xh), 0.5, 0.01,
                           H_opt=dev(gpu_hessian(Xh))).cpu().numpy()
    corr = np.abs(Wo - W).max()
    assert np.abs(Wg - Wo).max() <= QEP_TOL * np.abs(W).max()
    assert np.abs((Wg - W) - (Wo - W)).max() <= 2e-3 * corr


def test_gptq_identity_hessian_is_rtn():
    r = np.random.default_rng(3)
    W = (r.standard_normal((64, 256)) * 0.02).astype(np.float32).astype(np.float64)
    H = np.eye(256)
    codes, scales, zeros, perm, _ = gpu_gptq(W, H, 4, 64, 0.01, False)
    ref = oracle.gptq_quantize(W, H, 4, 64, 0.01, False)
    assert np.array_equal(codes, ref["codes"])


def test_gptq_dead_columns():
    L = random_layer_host(48, 256, 1024, seed=21)
    x = L["Xhat"].copy()
    x[:, [3, 100, 255]] = 0.0
    H = oracle.hessian(x).astype(np.float32).astype(np.float64)
    for act in (False, True):
        check_gptq(L["W"].astype(np.float64), H, 4, 64, 0.01, act)


def test_gptq_not_spd_reports_error():
    n = 128
    r = np.random.default_rng(5)
    Q, _ = np.linalg.qr(r.standard_normal((n, n)))
    ev = np.linspace(1.0, 2.0, n)
    ev[17] = -0.5
    H = (Q * ev) @ Q.T
    W = r.standard_normal((16, n)) * 0.02
    with pytest.raises(oc.OcError) as e:
        oc.oc_gptq_quantize(dev(W), dev(H), 4, 128, 0.0, False)
    assert e.value.status == oc.OC_ERR_NOT_SPD
    # the library stays usable afterwards
    check_gptq(W, np.eye(n) * 2.0, 4, 128, 0.0, False)


def test_gptq_nonfinite_reports_error():
    n = 128
    H = np.eye(n)
    H[5, 5] = np.nan
    W = np.zeros((8, n))
    with pytest.raises(oc.OcError) as e:
        oc.oc_gptq_quantize(dev(W), dev(H), 4, 128, 0.01, False)
    assert e.value.status == oc.OC_ERR_NONFINITE


# ----------------------------------------------------------------------------- end to end

def test_end_to_end_512_workload():
    spec = CONFIGS["layer_512"]
    L = make_layer_host(spec)
    W, X, Xh = L["W"].astype(np.float64), L["X"], L["Xhat"]
    # oracle
    Ho = oracle.hessian(Xh)
    Wpo = oracle.qep_correct(W, X, Xh, spec.alpha, spec.damp, H=Ho)
    ref = oracle.gptq_quantize(Wpo, Ho, spec.wbits, spec.groupsize, spec.damp, spec.act_order)
    # CUDA path
    Hg = dev(np.zeros((spec.d_in, spec.d_in)))
    Xd, Xhd = bf16_dev(X), bf16_dev(Xh)
    oc.oc_hessian_accumulate(Xhd, Hg)
    Wp = oc.oc_qep_correct(dev(W), Xd, Xhd, spec.alpha, spec.damp, H_opt=Hg)
    perm = torch.empty(spec.d_in, dtype=torch.int32, device="cuda")
    codes, scales, zeros, _ = oc.oc_gptq_quantize(Wp, Hg, spec.wbits, spec.groupsize, spec.damp,
                                                  spec.act_order, perm_out=perm)
    torch.cuda.synchronize()
    assert rel_fro(Hg.cpu().numpy(), Ho) <= H_TOL
    cg = oracle.unpack_codes(codes.cpu().numpy().view(np.uint32), spec.wbits, spec.d_in)
    sg, zg = scales.cpu().numpy(), zeros.cpu().numpy()
    ident = level_identity(cg, zg, ref["codes"], ref["zeros"], spec.groupsize)
    assert cg.size >= 100_000 and ident >= CODE_FRAC
    st = oracle.teacher_forced_check(Wpo, Ho, spec.wbits, spec.groupsize, spec.damp,
                                     spec.act_order, cg, sg, zg, perm=perm.cpu().numpy())
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= SCALE_TOL, st
    G = spec.groupsize
    deq = np.repeat(sg, G, axis=1) * (cg - np.repeat(zg, G, axis=1))
    eg = oracle.layer_errors(W, deq, X, Xh)["e_lit"]
    eo = oracle.layer_errors(W, ref["deq"], X, Xh)["e_lit"]
    assert abs(eg - eo) <= 0.01 * eo


# ----------------------------------------------------------------------------- fused layer call

@pytest.mark.parametrize("m,n,n_tok,wbits,G,act,dead,big", [
    (512, 512, 2048, 4, 128, False, False, False),
    (256, 384, 1500, 3, 64, True, False, False),
    (96, 256, 1024, 4, 64, True, True, False),     # dead columns: two factorisations
    (128, 1024, 4096, 2, 64, True, False, False),  # large enough for tensor-core factor nodes
    (160, 256, 1500, 4, 64, False, False, True),   # a difference beyond fp16's scaled range: bf16 cross product
])
def test_fused_layer_matches_oracle(m, n, n_tok, wbits, G, act, dead, big):
    L = random_layer_host(m, n, n_tok, seed=3000 + n + m)
    W, X, Xh = L["W"].astype(np.float64), L["X"].copy(), L["Xhat"].copy()
    if dead:
        X[:, [7, 100]] = 0.0
        Xh[:, [7, 100]] = 0.0
    if big:
        X, Xh = _far_difference(X, Xh)
    Ho = oracle.hessian(Xh)
    Wpo = oracle.qep_correct(W, X, Xh, 0.5, 0.01, H=Ho)
    ref = oracle.gptq_quantize(Wpo, Ho, wbits, G, 0.01, act)
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    Hg, Wpg, codes, scales, zeros, _ = oc.oc_quantize_layer(dev(W), bf16_dev(X), bf16_dev(Xh), 0.5, 0.01,
                                                            wbits, G, act, perm_out=perm)
    torch.cuda.synchronize()
    assert rel_fro(Hg.cpu().numpy(), Ho) <= H_TOL
    Wpg = Wpg.cpu().numpy()
    if big:
        # bf16 cross-product operands on a correction as large as W itself:
        # W' to about 1e-3 of the correction, and GPTQ judged on the GPU's
        # own W' (a difference of that size moves group ranges by more than
        # the scale tolerance)
        assert np.abs(Wpg - Wpo).max() <= 5e-3 * np.abs(Wpo - W).max()
        Wpo = Wpg.astype(np.float64)
        ref = oracle.gptq_quantize(Wpo, Ho, wbits, G, 0.01, act)
    else:
        assert np.abs(Wpg - Wpo).max() <= QEP_TOL * np.abs(W).max()
    cg = oracle.unpack_codes(codes.cpu().numpy().view(np.uint32), wbits, n)
    sg, zg = scales.cpu().numpy(), zeros.cpu().numpy()
    pg = perm.cpu().numpy()
    st = oracle.teacher_forced_check(Wpo, Ho, wbits, G, 0.01, act, cg, sg, zg, perm=pg)
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= SCALE_TOL, st
    ident = level_identity(cg, zg, ref["codes"], ref["zeros"], G)
    assert ident >= code_frac_for(cg.size), (ident, st)


def test_fused_layer_async_returns_before_its_stream_finishes():
    # In asynchronous mode the fused call only enqueues work: no step of it
    # (not the dead-column decision either) waits for the device.  A spinning
    # kernel ahead of it keeps the stream busy for about a second; the call
    # must return while the stream still runs, and its results must equal a
    # synchronous call's.
    m, n, G = 256, 512, 128
    L = random_layer_host(m, n, 2048, seed=3500)
    W, X, Xh = dev(L["W"]), bf16_dev(L["X"]), bf16_dev(L["Xhat"])
    ref = oc.oc_quantize_layer(W, X, Xh, 0.5, 0.01, 4, G, True)   # synchronous; sets up workspace and graphs
    torch.cuda.synchronize()
    out = dict(H=torch.empty(n, n, device="cuda"), W_out=torch.empty_like(W),
               codes=torch.empty(m, n * 4 // 32, dtype=torch.int32, device="cuda"),
               scales=torch.empty(m, n // G, device="cuda"), zeros=torch.empty(m, n // G, device="cuda"))
    stream = torch.cuda.current_stream()
    oc.oc_set_sync(False)
    try:
        torch.cuda._sleep(int(2e9))
        oc.oc_quantize_layer(W, X, Xh, 0.5, 0.01, 4, G, True, **out)
        busy = not stream.query()
        status = oc.oc_stream_status(stream)
    finally:
        oc.oc_set_sync(True)
    assert busy, "the call waited for its stream"
    assert status == oc.OC_OK
    assert torch.allclose(out["W_out"], ref[1], rtol=0, atol=1e-6 * float(ref[1].abs().max()))
    assert float((out["codes"] == ref[2]).float().mean()) >= 0.99
    assert torch.allclose(out["scales"], ref[3], rtol=1e-5, atol=0)


# ----------------------------------------------------------------------------- layer groups

@pytest.mark.parametrize("ms,n,n_tok,wbits,G,act,dead", [
    ((256, 128, 384), 512, 2048, 4, 128, False, False),
    ((96, 200), 384, 1500, 3, 64, True, False),
    ((64, 128, 32), 256, 1024, 4, 64, True, True),   # dead columns: two factorisations
])
def test_layer_group_matches_oracle_per_layer(ms, n, n_tok, wbits, G, act, dead):
    # Layers fed the same inputs share H, d and the factor; each must match
    # the oracle run on that layer alone.
    L = random_layer_host(max(ms), n, n_tok, seed=5000 + n)
    X, Xh = L["X"].copy(), L["Xhat"].copy()
    if dead:
        X[:, [3, 50]] = 0.0
        Xh[:, [3, 50]] = 0.0
    rng = np.random.default_rng(77)
    Ws = [(0.02 * rng.standard_normal((m, n))).astype(np.float32) for m in ms]
    Ho = oracle.hessian(Xh)
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    Hg, Wouts, codes, scales, zeros, _ = oc.oc_quantize_layer_group(
        [dev(W) for W in Ws], bf16_dev(X), bf16_dev(Xh), 0.5, 0.01, wbits, G, act, perm_out=perm)
    torch.cuda.synchronize()
    assert rel_fro(Hg.cpu().numpy(), Ho) <= H_TOL
    pg = perm.cpu().numpy()
    for l, W in enumerate(Ws):
        W64 = W.astype(np.float64)
        Wpo = oracle.qep_correct(W64, X, Xh, 0.5, 0.01, H=Ho)
        ref = oracle.gptq_quantize(Wpo, Ho, wbits, G, 0.01, act)
        assert np.abs(Wouts[l].cpu().numpy() - Wpo).max() <= QEP_TOL * np.abs(W64).max(), l
        cg = oracle.unpack_codes(codes[l].cpu().numpy().view(np.uint32), wbits, n)
        sg, zg = scales[l].cpu().numpy(), zeros[l].cpu().numpy()
        st = oracle.teacher_forced_check(Wpo, Ho, wbits, G, 0.01, act, cg, sg, zg, perm=pg)
        assert st["n_bad"] == 0 and st["zero_bad"] == 0, (l, st)
        assert st["scale_max_rel"] <= SCALE_TOL, (l, st)
        ident = level_identity(cg, zg, ref["codes"], ref["zeros"], G)
        assert ident >= code_frac_for(cg.size), (l, ident, st)


def test_layer_group_of_one_is_the_layer_call():
    L = random_layer_host(192, 256, 1024, seed=5101)
    W, X, Xh = dev(L["W"]), bf16_dev(L["X"]), bf16_dev(L["Xhat"])
    _, Wa, ca, sa, za, _ = oc.oc_quantize_layer(W, X, Xh, 0.5, 0.01, 4, 64, True)
    _, Wb, cb, sb, zb, _ = oc.oc_quantize_layer_group([W], X, Xh, 0.5, 0.01, 4, 64, True)
    torch.cuda.synchronize()
    # same kernels in the same order; only the order of fp32 additions inside
    # the tensor-core reduction may differ between runs
    assert torch.allclose(Wa, Wb[0], rtol=0, atol=1e-6 * float(Wa.abs().max()))
    same = float((ca == cb[0]).float().mean())
    assert same >= 0.99
    assert torch.allclose(sa, sb[0], rtol=1e-5, atol=0)


def test_layer_group_rejects_bad_arguments():
    L = random_layer_host(64, 128, 512, seed=5102)
    W, X, Xh = dev(L["W"]), bf16_dev(L["X"]), bf16_dev(L["Xhat"])
    with pytest.raises(oc.OcError):
        oc.oc_quantize_layer_group([W, W], X, Xh, 0.5, 0.01, 4, 64, False, W_outs=[W.clone(), W])
    with pytest.raises(oc.OcError):
        oc.oc_quantize_layer_group([W] * 17, X, Xh, 0.5, 0.01, 4, 64, False)


# ----------------------------------------------------------------------------- dequantisation, chains

@pytest.mark.parametrize("wbits,G", [(2, 64), (3, 128), (4, 32)])
def test_dequantize_matches_oracle(wbits, G):
    rng = np.random.default_rng(90 + wbits)
    m, n = 37, 512
    codes = rng.integers(0, 1 << wbits, size=(m, n))
    packed = oracle.pack_codes(codes, wbits).view(np.int32)
    scales = rng.uniform(1e-3, 0.1, size=(m, n // G)).astype(np.float32)
    zeros = rng.integers(0, 1 << wbits, size=(m, n // G)).astype(np.float32)
    want = oracle.dequantize(packed.view(np.uint32), scales, zeros, wbits, G, n)
    c_d = torch.from_numpy(np.ascontiguousarray(packed)).cuda()
    s_d, z_d = dev(scales), dev(zeros)
    out32 = oc.oc_dequantize(c_d, s_d, z_d, n, wbits, G)
    out16 = oc.oc_dequantize(c_d, s_d, z_d, n, wbits, G, bf16=True)
    torch.cuda.synchronize()
    # fp32: the correctly rounded product; bf16: that rounded to nearest even
    assert np.array_equal(out32.cpu().numpy(), want.astype(np.float32))
    assert np.array_equal(out16.float().cpu().numpy(), oracle._bf16(want.astype(np.float32)).astype(np.float32))


def test_chain_matches_oracle():
    rng = np.random.default_rng(91)
    N = 2048
    x0 = rng.standard_normal((N, 256))
    x0[:, :3] *= 8.0
    x0 = oracle._bf16(x0)
    Ws = [(rng.standard_normal((256, 256)) / 16).astype(np.float32),
          (rng.standard_normal((192, 256)) / 16).astype(np.float32),
          (rng.standard_normal((128, 192)) / 14).astype(np.float32)]
    ref_layers, (xo, xho) = oracle.quantize_chain(Ws, x0, 0.5, 0.01, 4, 64, False)
    layers, (xg, xhg) = oc.quantize_chain([dev(W) for W in Ws], dev(x0), 0.5, 0.01, 4, 64, False)
    torch.cuda.synchronize()
    # layer 0 sees identical inputs: the full per-layer checks
    r0, g0 = ref_layers[0], layers[0]
    assert rel_fro(g0["H"].cpu().numpy(), r0["H"]) <= H_TOL
    cg = oracle.unpack_codes(g0["codes"].cpu().numpy().view(np.uint32), 4, 256)
    st = oracle.teacher_forced_check(r0["W_prime"], r0["H"], 4, 64, 0.01, False, cg,
                                     g0["scales"].cpu().numpy(), g0["zeros"].cpu().numpy())
    assert st["n_bad"] == 0 and st["zero_bad"] == 0 and st["scale_max_rel"] <= SCALE_TOL, st
    # the full-precision stream: bf16 products of identical bf16 operands
    x1g = layers[1]["X"].float().cpu().numpy()
    x1o = ref_layers[1]["X"]
    assert np.mean(x1g == x1o) >= 0.99
    assert np.abs(x1g - x1o).max() <= 2.0 ** -6 * np.abs(x1o).max()
    # end to end: the propagated quantisation error of the chain within 1% of
    # the oracle's
    eg = np.linalg.norm(xg.float().cpu().numpy() - xhg.float().cpu().numpy())
    eo = np.linalg.norm(xo - xho)
    assert abs(eg - eo) <= 0.01 * eo, (eg, eo)


def test_chain_qep_reduces_propagated_error_on_gpu():
    rng = np.random.default_rng(92)
    x0 = rng.standard_normal((4096, 128))
    x0[:, :2] *= 8.0
    Ws = [dev((rng.standard_normal((128, 128)) / 11).astype(np.float32)) for _ in range(4)]
    errs = {}
    for alpha in (0.0, 0.5):
        _, (x, xh) = oc.quantize_chain(Ws, dev(x0), alpha, 0.01, 3, 32, False)
        errs[alpha] = float((x.float() - xh.float()).norm() / x.float().norm())
    assert errs[0.5] < errs[0.0], errs


# ----------------------------------------------------------------------------- sharded layers

@pytest.mark.parametrize("act", [False, True])
def test_token_and_row_shards_match_whole_layer(act):
    # Two shards in one process: oc_qep_terms on each token half, their sum
    # (what the all-reduce of a 2-GPU run computes), oc_quantize_from_terms on
    # each half of the rows; against the oracle on the whole layer.
    from post_weight_quantization_07_b200.sharded import shard_range
    m, n, n_tok, wbits, G = 320, 512, 3000, 4, 128
    L = random_layer_host(m, n, n_tok, seed=8200)
    W64 = L["W"].astype(np.float64)
    Ho = oracle.hessian(L["Xhat"])
    Wpo = oracle.qep_correct(W64, L["X"], L["Xhat"], 0.5, 0.01, H=Ho)
    ref = oracle.gptq_quantize(Wpo, Ho, wbits, G, 0.01, act)
    Xd, Xhd, Wd = bf16_dev(L["X"]), bf16_dev(L["Xhat"]), dev(L["W"])
    H = torch.zeros(n, n, device="cuda")
    D = torch.zeros(n, n, device="cuda")
    for r in range(2):
        t0, t1 = shard_range(n_tok, r, 2, align=64)
        Hp, Dp = oc.oc_qep_terms(Xd[t0:t1].contiguous(), Xhd[t0:t1].contiguous())
        H += Hp
        D += Dp
    assert rel_fro(H.cpu().numpy(), Ho) <= H_TOL
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    for r in range(2):
        r0, r1 = shard_range(m, r, 2)
        Wp, codes, scales, zeros, _ = oc.oc_quantize_from_terms(Wd[r0:r1].contiguous(), H, D, 0.5, 0.01, wbits, G,
                                                                act, perm_out=perm)
        torch.cuda.synchronize()
        assert np.abs(Wp.cpu().numpy() - Wpo[r0:r1]).max() <= QEP_TOL * np.abs(W64).max()
        cg = oracle.unpack_codes(codes.cpu().numpy().view(np.uint32), wbits, n)
        sg, zg = scales.cpu().numpy(), zeros.cpu().numpy()
        st = oracle.teacher_forced_check(Wpo[r0:r1], Ho, wbits, G, 0.01, act, cg, sg, zg, perm=perm.cpu().numpy())
        assert st["n_bad"] == 0 and st["zero_bad"] == 0 and st["scale_max_rel"] <= SCALE_TOL, (r, st)
        ident = level_identity(cg, zg, ref["codes"][r0:r1], ref["zeros"][r0:r1], G)
        assert ident >= code_frac_for(cg.size), (r, ident)


def test_qep_terms_of_no_tokens_are_zero():
    H, D = oc.oc_qep_terms(torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"),
                           torch.empty(0, 128, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert float(H.abs().max()) == 0.0 and float(D.abs().max()) == 0.0


# ----------------------------------------------------------------------------- Hadamard rotation

@pytest.mark.parametrize("rows,n,block", [(3, 4096, 4096), (5, 4096, 2048), (7, 11008, 256), (4, 1536, 512),
                                          (9, 96, 32), (33, 64, 2), (2, 8192, 16)])
def test_hadamard_rotation_matches_oracle(rows, n, block):
    rng = np.random.default_rng(rows * 1000 + block)
    x = rng.standard_normal((rows, n)).astype(np.float32)
    x[:, :3] *= 20.0
    want = oracle.hadamard_rotate(x, block)
    y32 = oc.oc_hadamard_rotate(dev(x), block)
    torch.cuda.synchronize()
    # fp32: log2(block) rounded butterfly stages and one scaling, each adding
    # at most a few ulps of the (orthonormally bounded) magnitudes
    tol = 4e-7 * (np.log2(block) + 1) * np.abs(x).max()
    assert np.abs(y32.cpu().numpy() - want).max() <= tol
    xb = oracle._bf16(x)
    yb = oc.oc_hadamard_rotate(bf16_dev(xb), block)
    torch.cuda.synchronize()
    wantb = oracle.hadamard_rotate(xb, block)
    got = yb.float().cpu().numpy()
    # one rounding to bf16 of a value within fp32 error of the exact rotation
    assert np.mean(got == oracle._bf16(wantb)) >= 0.99
    assert np.abs(got - wantb).max() <= 2.0 ** -8 * np.abs(wantb).max()


def test_hadamard_rotation_in_place_and_layer_output_invariance():
    rng = np.random.default_rng(95)
    W = dev(rng.standard_normal((64, 4096)).astype(np.float32))
    X = dev(rng.standard_normal((300, 4096)).astype(np.float32))
    ref = W @ X.t()
    Wr = oc.oc_hadamard_rotate(W, 4096)
    oc.oc_hadamard_rotate(X, 4096, out=X)   # in place
    torch.cuda.synchronize()
    got = Wr.double() @ X.double().t()
    assert float((got - ref.double()).abs().max()) <= 1e-3 * float(ref.abs().max())


# ----------------------------------------------------------------------------- dequantising GEMV

def _gemv_case(m, n, wbits, G, nb, seed):
    rng = np.random.default_rng(seed)
    Gs = n if G == -1 else G
    codes = rng.integers(0, 2 ** wbits, size=(m, n))
    scales = rng.uniform(0.001, 0.02, size=(m, n // Gs)).astype(np.float32)
    zeros = rng.integers(0, 2 ** wbits, size=(m, n // Gs)).astype(np.float32)
    x = oracle._bf16(rng.standard_normal((nb, n)))
    return oracle.pack_codes(codes, wbits), scales, zeros, x


def _gemv_bound(packed, scales, zeros, wbits, G, n, x):
    # fp32: one rounding of each dequantised weight and of each product, n
    # additions: |error| <= gamma_{n+2} * sum_j |x_j q_ij|, gamma_k = k u / (1 - k u)
    Q = oracle.dequantize(packed, scales, zeros, wbits, G, n)
    u = 2.0 ** -24
    k = n + 2
    return (k * u / (1 - k * u)) * (np.abs(x) @ np.abs(Q).T)


@pytest.mark.parametrize("m,n,wbits,G,nb", [
    (37, 320, 4, 32, 1),
    (64, 4096, 4, 128, 8),
    (33, 192, 3, 64, 3),
    (16, 96, 3, -1, 2),
    (40, 256, 2, 16, 5),     # groups smaller than a 32-column segment
    (8, 128, 2, 4, 4),
    (300, 1024, 3, 8, 1),
])
def test_dequant_gemv_matches_oracle(m, n, wbits, G, nb):
    packed, scales, zeros, x = _gemv_case(m, n, wbits, G, nb, seed=m + n + wbits)
    y = oc.oc_dequant_gemv(dev(packed.view(np.int32), torch.int32), dev(scales), dev(zeros), n, wbits, G,
                           dev(x, torch.bfloat16)).cpu().numpy()
    ref = oracle.dequant_gemv(packed, scales, zeros, wbits, G, n, x)
    assert np.all(np.abs(y - ref) <= _gemv_bound(packed, scales, zeros, wbits, G, n, x))


def test_dequant_gemv_on_quantiser_output():
    L = random_layer_host(96, 512, 1024, seed=4321)
    H = oracle.hessian(L["Xhat"]).astype(np.float32)
    codes, scales, zeros, _ = oc.oc_gptq_quantize(dev(L["W"]), dev(H), 3, 128, 0.01, False)
    x = L["X"][:6]
    y = oc.oc_dequant_gemv(codes, scales, zeros, 512, 3, 128, bf16_dev(x)).cpu().numpy()
    p, s, z = codes.cpu().numpy().view(np.uint32), scales.cpu().numpy(), zeros.cpu().numpy()
    ref = oracle.dequant_gemv(p, s, z, 3, 128, 512, x)
    assert np.all(np.abs(y - ref) <= _gemv_bound(p, s, z, 3, 128, 512, x))


def test_dequant_gemv_rejects_bad_arguments():
    packed, scales, zeros, x = _gemv_case(8, 96, 4, 32, 9, seed=5)
    with pytest.raises(oc.OcError) as e:   # batch 9 > 8
        oc.oc_dequant_gemv(dev(packed.view(np.int32), torch.int32), dev(scales), dev(zeros), 96, 4, 32,
                           dev(x, torch.bfloat16))
    assert e.value.status == oc.OC_ERR_INVALID_ARG


def test_factor_and_sweep_repeat_bit_for_bit():
    """Many factorisation leaves, run again and again: every call succeeds and
    gives the same codes, scales and zeros bit for bit (the inverse factor and
    the sweep add nothing through atomics, so any difference would be a race).
    An 11008-wide H has 86 leaves a call; twelve calls run over a thousand."""
    n, m = 11008, 64
    g = torch.Generator(device="cuda").manual_seed(31)
    Xh = torch.randn(2 * n, n, device="cuda", generator=g)
    H = 2.0 * (Xh.T @ Xh)
    W = torch.randn(m, n, device="cuda", generator=g)
    ref = None
    for _ in range(12):
        codes, scales, zeros, _ = oc.oc_gptq_quantize(W, H, 4, 128, 0.01, False)
        torch.cuda.synchronize()
        got = (codes.cpu().numpy(), scales.cpu().numpy(), zeros.cpu().numpy())
        if ref is None:
            ref = got
        else:
            for a, b in zip(ref, got):
                assert np.array_equal(a, b)
