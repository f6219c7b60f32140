"""B200-native layer-wise GPTQ + QEP weight quantisation.

Python binding of ``liboc.so`` (the C ABI in ``include/oc.h``).  The functions
below carry the C names and only marshal arguments: they check dtypes,
shapes and devices of torch tensors, allocate outputs the caller did not
supply, and pass raw device pointers and the current CUDA stream to the
library, whose kernels do every step of the computation.  The library is
loaded on first use; if it has not been built that first use raises an
ImportError with an explanation (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os
import re

__all__ = ["OC_OK", "OC_ERR_INVALID_ARG", "OC_ERR_UNSUPPORTED", "OC_ERR_NOT_SPD",
           "OC_ERR_NONFINITE", "OC_ERR_TIMEOUT", "OC_ERR_CUDA", "OC_ERR_OOM", "OcError",
           "LIB_PATH", "HEADER_PATH", "lib", "declared_symbols", "oc_hessian_accumulate",
           "oc_qep_correct", "oc_gptq_quantize", "oc_set_sync", "oc_stream_status",
           "oc_workspace_release", "oc_status_string", "oc_last_error", "oc_version",
           "oc_profile_enable", "oc_profile_read", "oc_launch_count", "oc_quantize_layer",
           "oc_lpcd_left_project", "lpcd_pair", "oc_dequant_gemv", "oc_test_inject_stall",
           "oc_test_unit_plan"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboc.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "oc.h")

OC_OK = 0
OC_ERR_INVALID_ARG = 1
OC_ERR_UNSUPPORTED = 2
OC_ERR_NOT_SPD = 3
OC_ERR_NONFINITE = 4
OC_ERR_TIMEOUT = 5
OC_ERR_CUDA = 6
OC_ERR_OOM = 7


class OcError(RuntimeError):
    """A liboc call returned a status other than OC_OK."""

    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)} ({detail})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m post_weight_quantization_07_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, f32, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
    L.oc_status_string.argtypes = [i32]
    L.oc_status_string.restype = ctypes.c_char_p
    L.oc_last_error.argtypes = []
    L.oc_last_error.restype = ctypes.c_char_p
    L.oc_version.argtypes = []
    L.oc_version.restype = i32
    L.oc_set_sync.argtypes = [i32]
    L.oc_set_sync.restype = None
    L.oc_stream_status.argtypes = [vp]
    L.oc_stream_status.restype = i32
    L.oc_workspace_release.argtypes = []
    L.oc_workspace_release.restype = i32
    L.oc_profile_enable.argtypes = [i32]
    L.oc_profile_enable.restype = i32
    L.oc_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64), i32]
    L.oc_profile_read.restype = i32
    L.oc_profile_phase_name.argtypes = [i32]
    L.oc_profile_phase_name.restype = ctypes.c_char_p
    L.oc_launch_count.argtypes = []
    L.oc_launch_count.restype = i64
    L.oc_test_inject_stall.argtypes = []
    L.oc_test_inject_stall.restype = i32
    L.oc_test_unit_plan.argtypes = [i64, i64, i64, vp]
    L.oc_test_unit_plan.restype = i32
    L.oc_hessian_accumulate.argtypes = [vp, i64, i64, vp, vp]
    L.oc_hessian_accumulate.restype = i32
    L.oc_qep_correct.argtypes = [vp, i64, i64, vp, vp, i64, f32, f32, vp, vp, vp]
    L.oc_qep_correct.restype = i32
    L.oc_gptq_quantize.argtypes = [vp, i64, i64, vp, i32, i32, f32, i32, vp, vp, vp, vp, vp]
    L.oc_gptq_quantize.restype = i32
    L.oc_quantize_layer.argtypes = [vp, i64, i64, vp, vp, i64, f32, f32, i32, i32, i32, vp, vp, vp, vp,
                                    vp, vp, vp]
    L.oc_quantize_layer.restype = i32
    L.oc_quantize_layer_group.argtypes = [i32, vp, vp, i64, vp, vp, i64, f32, f32, i32, i32, i32, vp, vp,
                                          vp, vp, vp, vp, vp]
    L.oc_quantize_layer_group.restype = i32
    L.oc_dequantize.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, i32, vp]
    L.oc_dequantize.restype = i32
    L.oc_qep_terms.argtypes = [vp, vp, i64, i64, vp, vp, vp]
    L.oc_qep_terms.restype = i32
    L.oc_quantize_from_terms.argtypes = [vp, i64, i64, vp, vp, f32, f32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.oc_quantize_from_terms.restype = i32
    L.oc_hadamard_rotate.argtypes = [vp, i64, i64, i32, vp, i32, vp]
    L.oc_hadamard_rotate.restype = i32
    L.oc_lpcd_left_project.argtypes = [vp, vp, i64, i64, vp, i64, f32, vp, vp]
    L.oc_lpcd_left_project.restype = i32
    L.oc_dequant_gemv.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp, i64, vp, vp]
    L.oc_dequant_gemv.restype = i32
    return L


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    # ``post_weight_quantization_07_b200.lib`` is the loaded ctypes library
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def declared_symbols():
    """Names of the functions ``include/oc.h`` declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+(oc_\w+)\s*\(", text, re.M)))


def _status_name(status: int) -> str:
    return _lib().oc_status_string(int(status)).decode()


def oc_status_string(status: int) -> str:
    return _status_name(status)


def oc_last_error() -> str:
    return _lib().oc_last_error().decode()


def oc_version() -> int:
    return _lib().oc_version()


def oc_set_sync(sync: bool) -> None:
    _lib().oc_set_sync(1 if sync else 0)


def _check(status: int, where: str):
    if status != OC_OK:
        raise OcError(status, where, oc_last_error())


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def oc_stream_status(stream=None) -> int:
    return _lib().oc_stream_status(_stream_handle(stream))


def oc_profile_enable(on: bool) -> None:
    _check(_lib().oc_profile_enable(1 if on else 0), "oc_profile_enable")


def oc_profile_read():
    """{phase name: (milliseconds, kernel launches)} accumulated since the last read."""
    k = 32
    ms = (ctypes.c_double * k)()
    ln = (ctypes.c_int64 * k)()
    nph = _lib().oc_profile_read(ms, ln, k)
    if nph < 0 or nph > k:
        raise OcError(nph, "oc_profile_read", oc_last_error())
    return {_lib().oc_profile_phase_name(i).decode(): (ms[i], ln[i]) for i in range(nph)}


def oc_launch_count() -> int:
    return _lib().oc_launch_count()


def oc_test_inject_stall() -> None:
    """Make the next tensor-core product launch stall on a barrier nothing
    releases: its bounded wait runs out and the call reports OC_ERR_TIMEOUT."""
    _check(_lib().oc_test_inject_stall(), "oc_test_inject_stall")


def oc_test_unit_plan(n_tok, n_tiles, clusters):
    """How the tensor-core product over tokens cuts its work (host logic only):
    returns (kc_stages, n_kc, split_k, full_units, units)."""
    out = (ctypes.c_int64 * 5)()
    _check(_lib().oc_test_unit_plan(int(n_tok), int(n_tiles), int(clusters), ctypes.cast(out, ctypes.c_void_p)),
           "oc_test_unit_plan")
    return tuple(int(v) for v in out)


def oc_workspace_release() -> None:
    _check(_lib().oc_workspace_release(), "oc_workspace_release")


def _dev_ptr(t, dtype, name, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def oc_hessian_accumulate(X, H, stream=None):
    """H += 2 X^T X for bf16 token-major X [n_tok, n] into fp32 H [n, n] (in place)."""
    import torch
    n_tok, n = X.shape
    st = _lib().oc_hessian_accumulate(_dev_ptr(X, torch.bfloat16, "X"), n_tok, n,
                                   _dev_ptr(H, torch.float32, "H", (n, n)), _stream_handle(stream))
    _check(st, "oc_hessian_accumulate")
    return H


def oc_qep_correct(W, X, Xhat, alpha, damp, H_opt=None, W_out=None, stream=None):
    """QEP correction W_out = W + alpha W (X - Xhat)^T Xhat (Xhat^T Xhat + lam I)^-1."""
    import torch
    m, n = W.shape
    n_tok = X.shape[0]
    if W_out is None:
        W_out = torch.empty_like(W)
    hp = _dev_ptr(H_opt, torch.float32, "H_opt", (n, n)) if H_opt is not None else None
    st = _lib().oc_qep_correct(_dev_ptr(W, torch.float32, "W"), m, n,
                            _dev_ptr(X, torch.bfloat16, "X", (n_tok, n)),
                            _dev_ptr(Xhat, torch.bfloat16, "Xhat", (n_tok, n)), n_tok,
                            float(alpha), float(damp), hp,
                            _dev_ptr(W_out, torch.float32, "W_out", (m, n)), _stream_handle(stream))
    _check(st, "oc_qep_correct")
    return W_out


def oc_gptq_quantize(W, H, wbits, groupsize, damp, act_order, codes=None, scales=None,
                     zeros=None, perm_out=None, stream=None):
    """GPTQ with per-group asymmetric grids; returns (codes, scales, zeros, perm_out)."""
    import torch
    m, n = W.shape
    G = n if groupsize == -1 else int(groupsize)
    ng = max(1, n // G)
    dev = W.device
    if codes is None:
        codes = torch.empty(m, n * wbits // 32, dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(m, ng, dtype=torch.float32, device=dev)
    if zeros is None:
        zeros = torch.empty(m, ng, dtype=torch.float32, device=dev)
    pp = _dev_ptr(perm_out, torch.int32, "perm_out", (n,)) if perm_out is not None else None
    st = _lib().oc_gptq_quantize(_dev_ptr(W, torch.float32, "W"), m, n,
                              _dev_ptr(H, torch.float32, "H", (n, n)), int(wbits), int(groupsize),
                              float(damp), 1 if act_order else 0,
                              _dev_ptr(codes, torch.int32, "codes", (m, n * wbits // 32)),
                              _dev_ptr(scales, torch.float32, "scales", (m, ng)),
                              _dev_ptr(zeros, torch.float32, "zeros", (m, ng)), pp,
                              _stream_handle(stream))
    _check(st, "oc_gptq_quantize")
    return codes, scales, zeros, perm_out


def oc_quantize_layer(W, X, Xhat, alpha, damp, wbits, groupsize, act_order, H=None, W_out=None,
                      codes=None, scales=None, zeros=None, perm_out=None, stream=None):
    """Hessian + QEP + GPTQ of one layer in one call (one factorisation when no
    column is dead).  Returns (H, W_out, codes, scales, zeros, perm_out)."""
    import torch
    m, n = W.shape
    n_tok = X.shape[0]
    G = n if groupsize == -1 else int(groupsize)
    ng = max(1, n // G)
    dev = W.device
    if H is None:
        H = torch.empty(n, n, dtype=torch.float32, device=dev)
    if W_out is None:
        W_out = torch.empty_like(W)
    if codes is None:
        codes = torch.empty(m, n * wbits // 32, dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(m, ng, dtype=torch.float32, device=dev)
    if zeros is None:
        zeros = torch.empty(m, ng, dtype=torch.float32, device=dev)
    pp = _dev_ptr(perm_out, torch.int32, "perm_out", (n,)) if perm_out is not None else None
    st = _lib().oc_quantize_layer(
        _dev_ptr(W, torch.float32, "W"), m, n, _dev_ptr(X, torch.bfloat16, "X", (n_tok, n)),
        _dev_ptr(Xhat, torch.bfloat16, "Xhat", (n_tok, n)), n_tok, float(alpha), float(damp),
        int(wbits), int(groupsize), 1 if act_order else 0, _dev_ptr(H, torch.float32, "H", (n, n)),
        _dev_ptr(W_out, torch.float32, "W_out", (m, n)),
        _dev_ptr(codes, torch.int32, "codes", (m, n * wbits // 32)),
        _dev_ptr(scales, torch.float32, "scales", (m, ng)),
        _dev_ptr(zeros, torch.float32, "zeros", (m, ng)), pp, _stream_handle(stream))
    _check(st, "oc_quantize_layer")
    return H, W_out, codes, scales, zeros, perm_out


def oc_quantize_layer_group(Ws, X, Xhat, alpha, damp, wbits, groupsize, act_order, H=None, W_outs=None,
                            codes=None, scales=None, zeros=None, perm_out=None, stream=None):
    """Hessian + QEP + GPTQ of several layers fed the same X, Xhat (one Hessian,
    one cross term and one factorisation for all).  Ws: list of fp32 [m_l x n]
    tensors.  Returns (H, W_outs, codes, scales, zeros, perm_out) with lists."""
    import torch
    count = len(Ws)
    n = Ws[0].shape[1]
    n_tok = X.shape[0]
    G = n if groupsize == -1 else int(groupsize)
    ng = max(1, n // G)
    dev = Ws[0].device
    ms = [int(W.shape[0]) for W in Ws]
    if H is None:
        H = torch.empty(n, n, dtype=torch.float32, device=dev)
    if W_outs is None:
        W_outs = [torch.empty_like(W) for W in Ws]
    if codes is None:
        codes = [torch.empty(m, n * wbits // 32, dtype=torch.int32, device=dev) for m in ms]
    if scales is None:
        scales = [torch.empty(m, ng, dtype=torch.float32, device=dev) for m in ms]
    if zeros is None:
        zeros = [torch.empty(m, ng, dtype=torch.float32, device=dev) for m in ms]
    ptrs = lambda xs: (ctypes.c_void_p * count)(*xs)
    w_p = ptrs([_dev_ptr(W, torch.float32, "W", (m, n)) for W, m in zip(Ws, ms)])
    wo_p = ptrs([_dev_ptr(W, torch.float32, "W_out", (m, n)) for W, m in zip(W_outs, ms)])
    c_p = ptrs([_dev_ptr(c, torch.int32, "codes", (m, n * wbits // 32)) for c, m in zip(codes, ms)])
    s_p = ptrs([_dev_ptr(x, torch.float32, "scales", (m, ng)) for x, m in zip(scales, ms)])
    z_p = ptrs([_dev_ptr(x, torch.float32, "zeros", (m, ng)) for x, m in zip(zeros, ms)])
    m_arr = (ctypes.c_int64 * count)(*ms)
    pp = _dev_ptr(perm_out, torch.int32, "perm_out", (n,)) if perm_out is not None else None
    st = _lib().oc_quantize_layer_group(
        count, w_p, m_arr, n, _dev_ptr(X, torch.bfloat16, "X", (n_tok, n)),
        _dev_ptr(Xhat, torch.bfloat16, "Xhat", (n_tok, n)), n_tok, float(alpha), float(damp), int(wbits),
        int(groupsize), 1 if act_order else 0, _dev_ptr(H, torch.float32, "H", (n, n)), wo_p, c_p, s_p, z_p, pp,
        _stream_handle(stream))
    _check(st, "oc_quantize_layer_group")
    return H, W_outs, codes, scales, zeros, perm_out


def oc_dequantize(codes, scales, zeros, n, wbits, groupsize, out=None, bf16=False, stream=None):
    """scale * (code - zero) of packed codes, [m x n] fp32 or bf16."""
    import torch
    m = codes.shape[0]
    G = n if groupsize == -1 else int(groupsize)
    dt = torch.bfloat16 if bf16 else torch.float32
    if out is None:
        out = torch.empty(m, n, dtype=dt, device=codes.device)
    st = _lib().oc_dequantize(_dev_ptr(codes, torch.int32, "codes", (m, n * wbits // 32)),
                              _dev_ptr(scales, torch.float32, "scales", (m, n // G)),
                              _dev_ptr(zeros, torch.float32, "zeros", (m, n // G)), m, n, int(wbits),
                              int(groupsize), _dev_ptr(out, dt, "out", (m, n)), 1 if bf16 else 0,
                              _stream_handle(stream))
    _check(st, "oc_dequantize")
    return out


def quantize_chain(Ws, X0, alpha, damp, wbits, groupsize, act_order, act="silu", stream=None):
    """Quantise a chain of linear layers with the quantisation error propagated.

    Two bf16 activation streams run through the chain, the full-precision
    X_{l+1} = f(X_l W_l^T) and the quantised Xh_{l+1} = f(Xh_l Q_l^T) from
    Xh_0 = X_0; layer l is quantised by oc_quantize_layer on its own pair
    (X_l, Xh_l), so its QEP correction sees the error of every layer before it.
    The forward products are plain bf16 GEMMs (cuBLAS through torch, fp32
    accumulation, bf16 result), f is SiLU (act="silu") or the identity, and
    Q_l comes from oc_dequantize.  Ws: fp32 [d_out x d_in] tensors whose
    d_in matches the previous d_out.  Returns (layers, (X_L, Xh_L)), each
    layer a dict with its inputs and oc_quantize_layer's outputs.
    """
    import torch
    import torch.nn.functional as F
    if act not in ("silu", "none"):
        raise ValueError("act must be 'silu' or 'none'")
    x = X0.to(torch.bfloat16).contiguous()
    xh = x.clone()
    layers = []
    for W in Ws:
        m, n = W.shape
        perm = torch.empty(n, dtype=torch.int32, device=W.device)
        H, Wp, codes, scales, zeros, _ = oc_quantize_layer(W, x, xh, alpha, damp, wbits, groupsize, act_order,
                                                           perm_out=perm, stream=stream)
        Q = oc_dequantize(codes, scales, zeros, n, wbits, groupsize, bf16=True, stream=stream)
        layers.append({"X": x, "Xhat": xh, "H": H, "W_prime": Wp, "codes": codes, "scales": scales,
                       "zeros": zeros, "perm": perm})
        y = x @ W.to(torch.bfloat16).t()
        yh = xh @ Q.t()
        if act == "silu":
            y, yh = F.silu(y), F.silu(yh)
        x, xh = y.contiguous(), yh.contiguous()
    return layers, (x, xh)


def oc_qep_terms(X, Xhat, H_part=None, D_part=None, stream=None):
    """(2 Xhat^T Xhat, (X - Xhat)^T Xhat) over these tokens, fp32 [n x n] each."""
    import torch
    n_tok, n = Xhat.shape
    if H_part is None:
        H_part = torch.empty(n, n, dtype=torch.float32, device=Xhat.device)
    if D_part is None:
        D_part = torch.empty(n, n, dtype=torch.float32, device=Xhat.device)
    xp = _dev_ptr(X, torch.bfloat16, "X", (n_tok, n)) if n_tok else None
    hp = _dev_ptr(Xhat, torch.bfloat16, "Xhat", (n_tok, n)) if n_tok else None
    st = _lib().oc_qep_terms(xp, hp, n_tok, n, _dev_ptr(H_part, torch.float32, "H_part", (n, n)),
                             _dev_ptr(D_part, torch.float32, "D_part", (n, n)), _stream_handle(stream))
    _check(st, "oc_qep_terms")
    return H_part, D_part


def oc_quantize_from_terms(W, H, D, alpha, damp, wbits, groupsize, act_order, W_out=None, codes=None,
                           scales=None, zeros=None, perm_out=None, stream=None):
    """QEP + GPTQ of W given the layer's global terms H and D.  Returns
    (W_out, codes, scales, zeros, perm_out)."""
    import torch
    m, n = W.shape
    G = n if groupsize == -1 else int(groupsize)
    ng = max(1, n // G)
    dev = W.device
    if W_out is None:
        W_out = torch.empty_like(W)
    if codes is None:
        codes = torch.empty(m, n * wbits // 32, dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(m, ng, dtype=torch.float32, device=dev)
    if zeros is None:
        zeros = torch.empty(m, ng, dtype=torch.float32, device=dev)
    pp = _dev_ptr(perm_out, torch.int32, "perm_out", (n,)) if perm_out is not None else None
    st = _lib().oc_quantize_from_terms(
        _dev_ptr(W, torch.float32, "W"), m, n, _dev_ptr(H, torch.float32, "H", (n, n)),
        _dev_ptr(D, torch.float32, "D", (n, n)), float(alpha), float(damp), int(wbits), int(groupsize),
        1 if act_order else 0, _dev_ptr(W_out, torch.float32, "W_out", (m, n)),
        _dev_ptr(codes, torch.int32, "codes", (m, n * wbits // 32)),
        _dev_ptr(scales, torch.float32, "scales", (m, ng)), _dev_ptr(zeros, torch.float32, "zeros", (m, ng)),
        pp, _stream_handle(stream))
    _check(st, "oc_quantize_from_terms")
    return W_out, codes, scales, zeros, perm_out


def oc_lpcd_left_project(B, W2, V, damp, W_out=None, stream=None):
    """(B^T B + mu I)^-1 B^T W2 V, mu = damp * mean(diag(B^T B)): LPCD's relaxed
    first-layer step (B, W2 fp32 [m x d]; V fp32 [d x n]; W_out may be V)."""
    import torch
    m, d = B.shape
    d2, n = V.shape
    if W2.shape != (m, d) or d2 != d:
        raise ValueError("B and W2 must be [m x d] and V [d x n]")
    if W_out is None:
        W_out = torch.empty(d, n, dtype=torch.float32, device=V.device)
    st = _lib().oc_lpcd_left_project(_dev_ptr(B, torch.float32, "B", (m, d)), _dev_ptr(W2, torch.float32, "W2", (m, d)),
                                     m, d, _dev_ptr(V, torch.float32, "V", (d, n)), n, float(damp),
                                     _dev_ptr(W_out, torch.float32, "W_out", (d, n)), _stream_handle(stream))
    _check(st, "oc_lpcd_left_project")
    return W_out


def oc_dequant_gemv(codes, scales, zeros, n, wbits, groupsize, x, y=None, stream=None):
    """y = x Q^T with Q the dequantised weight of packed codes [m x n*wbits/32];
    x bf16 [batch x n] (batch 1..8), y fp32 [batch x m]."""
    import torch
    m = codes.shape[0]
    nb = x.shape[0]
    ng = scales.shape[1]
    if y is None:
        y = torch.empty(nb, m, dtype=torch.float32, device=codes.device)
    st = _lib().oc_dequant_gemv(_dev_ptr(codes, torch.int32, "codes", (m, n * wbits // 32)),
                                _dev_ptr(scales, torch.float32, "scales", (m, ng)),
                                _dev_ptr(zeros, torch.float32, "zeros", (m, ng)), m, n, int(wbits),
                                int(groupsize), _dev_ptr(x, torch.bfloat16, "x", (nb, n)), nb,
                                _dev_ptr(y, torch.float32, "y", (nb, m)), _stream_handle(stream))
    _check(st, "oc_dequant_gemv")
    return y


def lpcd_pair(W1, W2, X, Xhat, alpha, damp, wbits, groupsize, act_order, rounds=1, stream=None,
              track_error=True):
    """Quantise a two-layer linear submodule y = x W1^T W2^T by layer-projected
    coordinate descent (OneComp release summary, LPCD bullet of section
    "v1.1.0全新量化方法"; hub page section "3. LPCD：子模块联合优化").

    Start: the layer-wise method, oc_quantize_layer of W1 on (X, Xhat) and of
    W2 on (Z, Zh) with Z = X W1^T and Zh = Xhat Q1^T.  Each round: the relaxed
    first-layer optimum against the current quantised second layer,
    oc_lpcd_left_project(Q2, W2, V1) with V1 = oc_qep_correct(W1, alpha = 1),
    projected by oc_gptq_quantize with the first layer's Hessian; then the
    second layer again by oc_quantize_layer with alpha = 1 on (Z, Zh).  Forward
    products are bf16 GEMMs (cuBLAS through torch), as in quantize_chain.
    W1 fp32 [d x n], W2 fp32 [m x d]; X, Xhat bf16 [N x n].  Returns a dict
    with the final layers' (codes, scales, zeros, perm) as q1 and q2, their
    dequantised weights Q1, Q2, the relaxed first-layer weights of each round
    (W1_star) with the quantised second layer each was solved against
    (Q2_used), the first layer's Hessian H1 and QEP weights V1 and, with track_error, the submodule's squared output error
    after the start and each round (errors) and the reference's squared norm.
    """
    import torch
    d, n = W1.shape
    m = W2.shape[0]
    X = X.to(torch.bfloat16).contiguous()
    Xhat = Xhat.to(torch.bfloat16).contiguous()
    H1, _, c1, s1, z1, p1 = oc_quantize_layer(W1, X, Xhat, alpha, damp, wbits, groupsize, act_order, stream=stream)
    Q1 = oc_dequantize(c1, s1, z1, n, wbits, groupsize, stream=stream)
    Z = (X @ W1.to(torch.bfloat16).t()).contiguous()

    def second(Q1, a):
        Zh = (Xhat @ Q1.to(torch.bfloat16).t()).contiguous()
        _, _, c2, s2, z2, p2 = oc_quantize_layer(W2, Z, Zh, a, damp, wbits, groupsize, act_order, stream=stream)
        return (c2, s2, z2, p2), oc_dequantize(c2, s2, z2, d, wbits, groupsize, stream=stream)

    def error(Q1, Q2):
        y = (X.float() @ W1.t()) @ W2.t()
        yh = (Xhat.float() @ Q1.t()) @ Q2.t()
        return float(((y - yh).double() ** 2).sum()), float((y.double() ** 2).sum())

    q2, Q2 = second(Q1, alpha)
    q1 = (c1, s1, z1, p1)
    out = {"W1_star": [], "Q2_used": [], "errors": []}
    if track_error:
        e, out["ref"] = error(Q1, Q2)
        out["errors"].append(e)
    V1 = oc_qep_correct(W1, X, Xhat, 1.0, damp, H_opt=H1, stream=stream)
    for _ in range(rounds):
        W1s = oc_lpcd_left_project(Q2, W2, V1, damp, stream=stream)
        out["W1_star"].append(W1s)
        out["Q2_used"].append(Q2)
        perm = torch.empty(n, dtype=torch.int32, device=W1.device)
        c1, s1, z1, _ = oc_gptq_quantize(W1s, H1, wbits, groupsize, damp, act_order, perm_out=perm, stream=stream)
        q1 = (c1, s1, z1, perm)
        Q1 = oc_dequantize(c1, s1, z1, n, wbits, groupsize, stream=stream)
        q2, Q2 = second(Q1, 1.0)
        if track_error:
            out["errors"].append(error(Q1, Q2)[0])
    out.update(q1=q1, q2=q2, Q1=Q1, Q2=Q2, H1=H1, V1=V1)
    return out


def oc_hadamard_rotate(X, block, out=None, stream=None):
    """X (I (x) H_block) / sqrt(block) along the last axis of a 2-D bf16 or fp32
    tensor (out may be X)."""
    import torch
    rows, n = X.shape
    if X.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("X must be bf16 or fp32")
    if out is None:
        out = torch.empty_like(X)
    st = _lib().oc_hadamard_rotate(_dev_ptr(X, X.dtype, "X", (rows, n)) if rows else None, rows, n, int(block),
                                   _dev_ptr(out, X.dtype, "out", (rows, n)) if rows else None,
                                   1 if X.dtype == torch.bfloat16 else 0, _stream_handle(stream))
    _check(st, "oc_hadamard_rotate")
    return out
