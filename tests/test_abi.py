"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything (no GPU
needed for any of these)."""
import ctypes
import subprocess

import pytest

import post_weight_quantization_07_b200 as oc


def test_library_exports_every_declared_symbol():
    declared = oc.declared_symbols()
    assert {"oc_hessian_accumulate", "oc_qep_correct", "oc_gptq_quantize"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", oc.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(oc.lib, s)


def test_status_strings_and_version():
    assert oc.oc_status_string(oc.OC_OK) == "OC_OK"
    assert oc.oc_status_string(oc.OC_ERR_NOT_SPD) == "OC_ERR_NOT_SPD"
    assert oc.oc_status_string(12345) == "OC_ERR_UNKNOWN"
    assert oc.oc_version() >= 100


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first


@pytest.mark.parametrize("args,why", [
    ((NULL, 10, 64, FAKE, NULL), "null X with tokens"),
    ((FAKE, 10, 64, NULL, NULL), "null H"),
    ((FAKE, 10, 48, FAKE, NULL), "n not a multiple of 64"),
    ((FAKE, -1, 64, FAKE, NULL), "negative n_tok"),
])
def test_hessian_rejects_bad_arguments(args, why):
    assert oc.lib.oc_hessian_accumulate(*args) == oc.OC_ERR_INVALID_ARG, why
    assert oc.oc_last_error() != ""


def test_hessian_zero_tokens_is_a_no_op():
    # no token: nothing is launched and X may be NULL
    assert oc.lib.oc_hessian_accumulate(NULL, 0, 64, FAKE, NULL) == oc.OC_OK


@pytest.mark.parametrize("kw,why", [
    (dict(wbits=5), "wbits"),
    (dict(wbits=1), "wbits"),
    (dict(groupsize=96), "groupsize neither power of two <= 128 nor multiple of 128"),
    (dict(groupsize=100), "groupsize does not divide n"),
    (dict(act_order=2), "act_order"),
    (dict(damp=-0.1), "negative damp"),
    (dict(m=0), "empty m"),
    (dict(n=96), "n not a multiple of 64"),
])
def test_gptq_rejects_bad_arguments(kw, why):
    a = dict(W=FAKE, m=16, n=384, H=FAKE, wbits=4, groupsize=128, damp=0.01, act_order=0,
             codes=FAKE, scales=FAKE, zeros=FAKE, perm=NULL, stream=NULL)
    a.update(kw)
    st = oc.lib.oc_gptq_quantize(a["W"], a["m"], a["n"], a["H"], a["wbits"], a["groupsize"],
                                 a["damp"], a["act_order"], a["codes"], a["scales"], a["zeros"],
                                 a["perm"], a["stream"])
    assert st == oc.OC_ERR_INVALID_ARG, why


def test_qep_rejects_bad_arguments():
    st = oc.lib.oc_qep_correct(FAKE, 8, 64, FAKE, FAKE, 0, 0.5, 0.01, NULL, FAKE, NULL)
    assert st == oc.OC_ERR_INVALID_ARG
    st = oc.lib.oc_qep_correct(FAKE, 8, 64, FAKE, FAKE, 10, float("nan"), 0.01, NULL, FAKE, NULL)
    assert st == oc.OC_ERR_INVALID_ARG
    st = oc.lib.oc_qep_correct(NULL, 8, 64, FAKE, FAKE, 10, 0.5, 0.01, NULL, FAKE, NULL)
    assert st == oc.OC_ERR_INVALID_ARG


@pytest.mark.parametrize("args,why", [
    ((NULL, FAKE, 64, 128, FAKE, 32, 0.01, FAKE, NULL), "null B"),
    ((FAKE, FAKE, 64, 100, FAKE, 32, 0.01, FAKE, NULL), "d not a multiple of 64"),
    ((FAKE, FAKE, 6, 128, FAKE, 32, 0.01, FAKE, NULL), "m not a multiple of 4"),
    ((FAKE, FAKE, 64, 128, FAKE, 0, 0.01, FAKE, NULL), "empty n"),
    ((FAKE, FAKE, 64, 128, FAKE, 32, -1.0, FAKE, NULL), "negative damp"),
    ((FAKE, FAKE, 64, 128, ctypes.c_void_p((1 << 20) + 4), 32, 0.01, FAKE, NULL), "unaligned V"),
])
def test_lpcd_left_project_rejects_bad_arguments(args, why):
    assert oc.lib.oc_lpcd_left_project(*args) == oc.OC_ERR_INVALID_ARG, why
    assert oc.oc_last_error() != ""


@pytest.mark.parametrize("kw,why", [
    (dict(codes=NULL), "null codes"),
    (dict(n=48), "n not a multiple of 32"),
    (dict(wbits=5), "wbits"),
    (dict(batch=0), "empty batch"),
    (dict(batch=9), "batch above 8"),
    (dict(groupsize=48, n=96), "group of 32 or more that is not a multiple of 32"),
    (dict(groupsize=12), "group below 32 that does not divide 32"),
    (dict(groupsize=64, n=96), "group that does not divide n"),
    (dict(x=ctypes.c_void_p((1 << 20) + 2)), "unaligned x"),
])
def test_dequant_gemv_rejects_bad_arguments(kw, why):
    a = dict(codes=FAKE, scales=FAKE, zeros=FAKE, m=8, n=128, wbits=4, groupsize=32, x=FAKE, batch=1, y=FAKE,
             stream=NULL)
    a.update(kw)
    st = oc.lib.oc_dequant_gemv(a["codes"], a["scales"], a["zeros"], a["m"], a["n"], a["wbits"], a["groupsize"],
                                a["x"], a["batch"], a["y"], a["stream"])
    assert st == oc.OC_ERR_INVALID_ARG, why
