"""Seeded synthetic layer workloads (weights W, calibration inputs X and X-hat).

This module holds only random-number recipes: it computes none of the
quantisation method's arithmetic, so both the CUDA path and the float64 oracle
may take their inputs from it without sharing any of the method's code.

Workload recipes
----------------
Every workload is one linear layer ``y = W x`` with ``W`` of shape
``d_out x d_in`` and calibration activations stored token-major, ``X`` of shape
``n_tok x d_in`` (the PyTorch activation layout). ``X-hat`` is the input the
quantised layer sees: the full-precision input plus a small channel-wise
perturbation standing in for the quantisation error of earlier layers.

* ``layer_512``        512 x 512, W fp32 ~ N(0, 1/512); X: 2048 tokens, N(0,1) with 4
                       random channels x10; X-hat = X + N(0, 0.05^2); 4-bit, g128.
* ``q_proj_4096``      Llama-2-7B q_proj, 4096 x 4096, W bf16 ~ N(0, 0.02^2); X: 262144
                       tokens of Student-t(4) with 1% of channels x20; 4-bit g128.
* ``down_proj_11008``  Llama-2-7B down_proj, d_in 11008, d_out 4096; X: 262144 tokens of
                       SiLU(z1)*z2 with 0.5% of channels x50; 3-bit g128, act_order.
* ``llama7b_layers``   224 layers of a 32-block Llama-2-7B-shaped model, 131072 tokens
                       per layer, Student-t(4) with 1% of channels x20; attention 4-bit,
                       MLP 3-bit, g128.
* ``down_proj_28672``  Llama-3-70B down_proj, d_in 28672, d_out 8192; X: 65536 tokens of
                       Student-t(3) with 1% of channels x30; 2-bit g64, act_order.

Readings where the workload description leaves a knob open: outlier channel count is ``max(1, floor(frac * d_in))``, chosen
without replacement; Student-t is the standard t_nu (no rescaling); X-hat for
the large workloads is ``X + N(0, (0.02 * sigma_c)^2)`` with ``sigma_c`` the
theoretical standard deviation of channel ``c`` after outlier scaling; X and
X-hat are rounded to bf16 once and both sides use the rounded values; W of the
bf16 workloads is drawn in fp32, rounded to bf16 and handed to the library as
fp32 (exact upcast).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

__all__ = ["LayerSpec", "CONFIGS", "llama7b_layers", "make_layer_host",
           "make_layer_device", "random_layer_host", "bf16_round"]


@dataclass(frozen=True)
class LayerSpec:
    name: str
    d_in: int
    d_out: int
    n_tok: int
    w_std: float
    w_bf16: bool            # W drawn then rounded to bf16 (handed over as fp32)
    x_kind: str             # "normal" | "t" | "swiglu"
    nu: float = 0.0         # Student-t degrees of freedom
    outlier_frac: float = 0.0
    n_outliers: int = 0     # used when outlier_frac == 0
    outlier_scale: float = 1.0
    noise_abs: float = 0.0  # X-hat = X + N(0, noise_abs^2)          (c1)
    noise_rel: float = 0.0  # X-hat = X + N(0, (noise_rel*sigma_c)^2)  (the large workloads)
    wbits: int = 4
    groupsize: int = 128
    act_order: bool = False
    alpha: float = 0.5
    damp: float = 0.01
    seed: int = 0

    def outlier_count(self) -> int:
        if self.outlier_frac > 0:
            return max(1, int(math.floor(self.outlier_frac * self.d_in)))
        return self.n_outliers

    def with_(self, **kw) -> "LayerSpec":
        return replace(self, **kw)


CONFIGS = {
    "layer_512": LayerSpec("layer_512", d_in=512, d_out=512, n_tok=2048,
                        w_std=math.sqrt(1.0 / 512), w_bf16=False, x_kind="normal",
                        n_outliers=4, outlier_scale=10.0, noise_abs=0.05,
                        wbits=4, groupsize=128, act_order=False, seed=1),
    "q_proj_4096": LayerSpec("q_proj_4096", d_in=4096, d_out=4096, n_tok=262144,
                           w_std=0.02, w_bf16=True, x_kind="t", nu=4.0,
                           outlier_frac=0.01, outlier_scale=20.0, noise_rel=0.02,
                           wbits=4, groupsize=128, act_order=False, seed=2),
    "down_proj_11008": LayerSpec("down_proj_11008", d_in=11008, d_out=4096, n_tok=262144,
                              w_std=0.02, w_bf16=True, x_kind="swiglu",
                              outlier_frac=0.005, outlier_scale=50.0, noise_rel=0.02,
                              wbits=3, groupsize=128, act_order=True, seed=3),
    "down_proj_28672": LayerSpec("down_proj_28672", d_in=28672, d_out=8192, n_tok=65536,
                             w_std=0.015, w_bf16=True, x_kind="t", nu=3.0,
                             outlier_frac=0.01, outlier_scale=30.0, noise_rel=0.02,
                             wbits=2, groupsize=64, act_order=True, seed=5),
}


def llama7b_layers(n_tok: int = 131072):
    """The 224 layer specs of a 32-block Llama-2-7B-shaped model (per block:
    q/k/v/o 4096x4096 at 4 bits, gate/up 4096->11008 and down 11008->4096 at
    3 bits, g128, QEP alpha 0.5, damp 0.01, act_order off), one seed per layer."""
    shapes = [("q", 4096, 4096, 4), ("k", 4096, 4096, 4), ("v", 4096, 4096, 4),
              ("o", 4096, 4096, 4), ("gate", 4096, 11008, 3), ("up", 4096, 11008, 3),
              ("down", 11008, 4096, 3)]
    out = []
    for blk in range(32):
        for j, (nm, d_in, d_out, bits) in enumerate(shapes):
            idx = blk * len(shapes) + j
            out.append(LayerSpec(f"l7b_b{blk}_{nm}", d_in=d_in, d_out=d_out, n_tok=n_tok,
                                 w_std=0.02, w_bf16=True, x_kind="t", nu=4.0,
                                 outlier_frac=0.01, outlier_scale=20.0, noise_rel=0.02,
                                 wbits=bits, groupsize=128, act_order=False,
                                 seed=4_000_000 + idx))
    return out


def _silu_times_normal_std() -> float:
    # std of SiLU(z1) * z2 for independent standard normals = sqrt(E[SiLU(z)^2]),
    # by trapezoid quadrature on a fine grid (a property of the distribution only).
    z = np.linspace(-12.0, 12.0, 240001)
    pdf = np.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    silu = z / (1.0 + np.exp(-z))
    return math.sqrt(float(np.trapezoid(silu * silu * pdf, z)))


def _base_std(spec: LayerSpec) -> float:
    if spec.x_kind == "normal":
        return 1.0
    if spec.x_kind == "t":
        return math.sqrt(spec.nu / (spec.nu - 2.0))
    if spec.x_kind == "swiglu":
        return _silu_times_normal_std()
    raise ValueError(spec.x_kind)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32/float64 values to the nearest bf16 (ties to even), returned as float32."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    u = a32.view(np.uint32)
    # For finite inputs the sum stays below 2^32 (the largest finite pattern is
    # 0xFF7FFFFF), so 32-bit arithmetic cannot wrap.
    rounded = (u >> 16) & np.uint32(1)
    rounded += u
    rounded += np.uint32(0x7FFF)
    rounded &= np.uint32(0xFFFF0000)
    out = rounded.view(np.float32)
    # NaN/Inf are not produced by these recipes; keep them untouched if present.
    bad = ~np.isfinite(a32)
    if bad.any():
        out = out.copy()
        out[bad] = a32[bad]
    return out


# ----------------------------------------------------------------------------- host (numpy)

def _draw_x_host(rng: np.random.Generator, spec: LayerSpec, n_tok: int) -> np.ndarray:
    shape = (n_tok, spec.d_in)
    if spec.x_kind == "normal":
        x = rng.standard_normal(shape)
    elif spec.x_kind == "t":
        x = rng.standard_t(spec.nu, size=shape)
    elif spec.x_kind == "swiglu":
        z1 = rng.standard_normal(shape)
        z2 = rng.standard_normal(shape)
        x = z1 / (1.0 + np.exp(-z1)) * z2
    else:
        raise ValueError(spec.x_kind)
    return x


def make_layer_host(spec: LayerSpec, n_tok: Optional[int] = None):
    """Draw (W fp32, X, X-hat as bf16-valued float32 arrays) with numpy PCG64.

    Returns a dict with keys ``W`` (d_out x d_in float32), ``X`` and ``Xhat``
    (n_tok x d_in float32 holding bf16-representable values), ``outliers``.
    Intended for workloads that fit comfortably in host memory.
    """
    n_tok = spec.n_tok if n_tok is None else n_tok
    rng = np.random.default_rng(spec.seed)
    W = rng.standard_normal((spec.d_out, spec.d_in)) * spec.w_std
    W = bf16_round(W) if spec.w_bf16 else W.astype(np.float32)
    outliers = np.sort(rng.choice(spec.d_in, size=spec.outlier_count(), replace=False))
    x = _draw_x_host(rng, spec, n_tok)
    ch_scale = np.ones(spec.d_in)
    ch_scale[outliers] = spec.outlier_scale
    x *= ch_scale[None, :]
    if spec.noise_abs > 0:
        noise = rng.standard_normal(x.shape) * spec.noise_abs
    else:
        sigma_c = _base_std(spec) * ch_scale
        noise = rng.standard_normal(x.shape) * (spec.noise_rel * sigma_c)[None, :]
    xhat = x + noise
    return {"W": np.ascontiguousarray(W, dtype=np.float32),
            "X": bf16_round(x), "Xhat": bf16_round(xhat), "outliers": outliers}


def random_layer_host(d_out: int, d_in: int, n_tok: int, seed: int, *, w_std: float = 0.02,
                      x_kind: str = "t", nu: float = 4.0, outlier_frac: float = 0.01,
                      outlier_scale: float = 20.0, noise_rel: float = 0.02):
    """A small layer of the large workloads' distribution at arbitrary sizes."""
    spec = LayerSpec("random", d_in=d_in, d_out=d_out, n_tok=n_tok, w_std=w_std,
                     w_bf16=True, x_kind=x_kind, nu=nu, outlier_frac=outlier_frac,
                     outlier_scale=outlier_scale, noise_rel=noise_rel, seed=seed)
    return make_layer_host(spec)


# ----------------------------------------------------------------------------- device (torch)

def make_layer_device(spec: LayerSpec, device, n_tok: Optional[int] = None,
                      chunk: int = 8192, want_x: bool = True):
    """Draw the workload directly in device memory with a seeded torch generator.

    Returns ``W`` (fp32, bf16-valued when ``spec.w_bf16``), ``X`` and ``Xhat``
    (bf16, n_tok x d_in, contiguous).  Generation runs chunk by chunk over
    tokens so that temporaries stay small.  The same seed on the same device
    type reproduces the same tensors.
    """
    import torch

    n_tok = spec.n_tok if n_tok is None else n_tok
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed)
    W = torch.randn(spec.d_out, spec.d_in, generator=g, device=device, dtype=torch.float32)
    W.mul_(spec.w_std)
    if spec.w_bf16:
        W = W.to(torch.bfloat16).to(torch.float32)
    perm = torch.randperm(spec.d_in, generator=g, device=device)
    outliers = torch.sort(perm[: spec.outlier_count()]).values
    ch_scale = torch.ones(spec.d_in, device=device, dtype=torch.float32)
    ch_scale[outliers] = spec.outlier_scale
    if spec.noise_abs > 0:
        noise_std = torch.full_like(ch_scale, spec.noise_abs)
    else:
        noise_std = spec.noise_rel * _base_std(spec) * ch_scale
    X = torch.empty(n_tok, spec.d_in, device=device, dtype=torch.bfloat16) if want_x else None
    Xhat = torch.empty(n_tok, spec.d_in, device=device, dtype=torch.bfloat16)
    for t0 in range(0, n_tok, chunk):
        t1 = min(n_tok, t0 + chunk)
        shape = (t1 - t0, spec.d_in)
        if spec.x_kind == "normal":
            x = torch.randn(shape, generator=g, device=device)
        elif spec.x_kind == "t":
            # t_nu = z / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared normals (integer nu)
            k = int(round(spec.nu))
            z = torch.randn(shape, generator=g, device=device)
            chi2 = torch.zeros(shape, device=device)
            for _ in range(k):
                e = torch.randn(shape, generator=g, device=device)
                chi2.addcmul_(e, e)
            x = z * torch.rsqrt(chi2 / k)
        elif spec.x_kind == "swiglu":
            z1 = torch.randn(shape, generator=g, device=device)
            z2 = torch.randn(shape, generator=g, device=device)
            x = torch.nn.functional.silu(z1) * z2
        else:
            raise ValueError(spec.x_kind)
        x.mul_(ch_scale)
        noise = torch.randn(shape, generator=g, device=device).mul_(noise_std)
        Xhat[t0:t1] = (x + noise).to(torch.bfloat16)
        if X is not None:
            X[t0:t1] = x.to(torch.bfloat16)
    return {"W": W.contiguous(), "X": X, "Xhat": Xhat, "outliers": outliers}
