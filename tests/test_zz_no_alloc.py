"""The allocation-free GPTQ entry point against the allocating one.

oc_gptq_quantize_noalloc exists for callers that cannot let a library allocate
device memory behind their back (a process whose GPU memory belongs to its own
caching allocator, a service held to a fixed pre-reserved budget): it runs the
same kernels as oc_gptq_quantize with all scratch taken from an array built
into the library.  These tests call both through the C ABI with raw pointers
and require the same results, within the tolerances of the other GPTQ parity
tests, on two calls in a row; a call on the same shape after a call on other
data (which leaves its intermediates in the shared scratch at the same
offsets) must repeat its results bit for bit and pass the oracle's replay.
The file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from synthetic import random_layer_host

torch = pytest.importorskip("torch")
oc = pytest.importorskip("post_weight_quantization_07_b200")

pytestmark = pytest.mark.gpu

SCALE_TOL = 1e-5


def _bind():
    L = oc.lib
    f = L.oc_gptq_quantize_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    g = L.oc_gptq_quantize
    return f, g


def _call(fn, W, H, wbits, G, damp, act, check_free=False):
    m, n = W.shape
    ng = n // (n if G == -1 else G)
    codes = torch.empty(m, n * wbits // 32, dtype=torch.int32, device="cuda")
    scales = torch.empty(m, ng, device="cuda")
    zeros = torch.empty(m, ng, device="cuda")
    perm = torch.empty(n, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    st = fn(ctypes.c_void_p(W.data_ptr()), m, n, ctypes.c_void_p(H.data_ptr()), wbits, G, damp,
            1 if act else 0, ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
            ctypes.c_void_p(zeros.data_ptr()), ctypes.c_void_p(perm.data_ptr()), stream)
    torch.cuda.synchronize()
    assert st == oc.OC_OK, oc.oc_last_error()
    if check_free:
        # the call took no device memory (outputs were allocated beforehand)
        assert torch.cuda.mem_get_info()[0] == free0
    return codes.cpu().numpy(), scales.cpu().numpy(), zeros.cpu().numpy(), perm.cpu().numpy()


def _layer(m, n, seed):
    L = random_layer_host(m, n, 2 * n, seed=seed)
    H = oracle.hessian(L["Xhat"]).astype(np.float32)
    return (torch.from_numpy(L["W"]).cuda(), torch.from_numpy(H).cuda())


def _same(a, b, wbits, G):
    ca, sa, za, pa = a
    cb, sb, zb, pb = b
    n = pa.shape[0]
    assert np.array_equal(pa, pb)
    assert np.all(np.abs(sa - sb) <= SCALE_TOL * np.abs(sb))
    Gs = n if G == -1 else G
    la = oracle.unpack_codes(ca.view(np.uint32), wbits, n) - np.repeat(za, Gs, axis=1)
    lb = oracle.unpack_codes(cb.view(np.uint32), wbits, n) - np.repeat(zb, Gs, axis=1)
    assert np.mean(la == lb) >= 0.999


def test_noalloc_matches_allocating_entry_point_twice():
    noalloc, alloc = _bind()
    cases = [(384, 512, 4, 128, False, 31), (200, 256, 3, 64, True, 32)]
    for i, (m, n, wbits, G, act, seed) in enumerate(cases):
        W, H = _layer(m, n, seed)
        # the allocating call first: it grows its own workspace and loads every
        # kernel this case uses, so the second no-alloc call can be checked for
        # taking no device memory at all
        ref = _call(alloc, W, H, wbits, G, 0.01, act)
        got = _call(noalloc, W, H, wbits, G, 0.01, act, check_free=(i == 1))
        _same(got, ref, wbits, G)


def test_noalloc_rejects_layers_beyond_its_scratch():
    noalloc, _ = _bind()
    W = torch.zeros(4096, 1024, device="cuda")
    H = torch.eye(1024, device="cuda")
    out = torch.empty(4096, 1024 * 4 // 32, dtype=torch.int32, device="cuda")
    s = torch.empty(4096, 8, device="cuda")
    st = noalloc(ctypes.c_void_p(W.data_ptr()), 4096, 1024, ctypes.c_void_p(H.data_ptr()), 4, 128,
                 0.01, 0, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                 ctypes.c_void_p(s.data_ptr()), None, None)
    assert st == oc.OC_ERR_INVALID_ARG
    assert "scratch" in oc.oc_last_error()


def test_noalloc_same_shape_repeat_and_oracle():
    # Same shape three times: data A, data B, data A again.  The third call
    # finds B's intermediates in the shared scratch at the very offsets it
    # uses, and must still give A's results bit for bit; A's results must also
    # pass the oracle's teacher-forced replay.
    noalloc, _ = _bind()
    m, n, wbits, G, act = 256, 512, 4, 128, True
    Wa, Ha = _layer(m, n, 61)
    Wb, Hb = _layer(m, n, 62)
    first = _call(noalloc, Wa, Ha, wbits, G, 0.01, act)
    other = _call(noalloc, Wb, Hb, wbits, G, 0.01, act)
    again = _call(noalloc, Wa, Ha, wbits, G, 0.01, act)
    for x, y in zip(first, again):
        assert np.array_equal(x, y)
    assert not np.array_equal(first[1], other[1])
    codes, scales, zeros, perm = first
    W64, H64 = Wa.cpu().numpy().astype(np.float64), Ha.cpu().numpy().astype(np.float64)
    cg = oracle.unpack_codes(codes.view(np.uint32), wbits, n)
    st = oracle.teacher_forced_check(W64, H64, wbits, G, 0.01, act, cg, scales, zeros, perm=perm)
    assert st["n_bad"] == 0 and st["zero_bad"] == 0, st
    assert st["scale_max_rel"] <= SCALE_TOL, st
    ref = oracle.gptq_quantize(W64, H64, wbits, G, 0.01, act)
    assert np.array_equal(perm, ref["perm"])
    assert np.mean(cg == ref["codes"]) >= 0.99
