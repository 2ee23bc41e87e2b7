"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare it with the float64 oracle on the same seeded inputs.

Tolerance (stated for bf16 inputs with fp32 accumulation): max |O - O_ref| <=
1e-2 and max |LSE - LSE_ref| <= 1e-3.  The same bars apply to fp16 and fp32
inputs.  Where rounding O_ref itself to the output dtype already moves it by
more than 1e-2 (|O| >= 4 in bf16), the O bar is widened by half an output ulp
of O_ref; the helper reports when that happens.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import attention_batched, attention_rows, resolve_scale
from tiled_attention_13_b200 import fa_get_device_status, forward
from tiled_attention_13_b200.inputs import Workload, make_qkv

O_TOL = 1e-2
LSE_TOL = 1e-3

_TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "fp32":
        return np.zeros_like(x)
    mant = 7 if dtype == "bf16" else 10
    ax = np.maximum(np.abs(x), 1e-30)
    e = np.floor(np.log2(ax))
    return 0.5 * np.exp2(e - mant)


def o_bar(o_ref: np.ndarray, dtype: str) -> np.ndarray:
    """1e-2, widened by half an ulp of the output dtype where rounding O_ref to
    that dtype already costs more than 1e-2."""
    t = torch.from_numpy(o_ref).to(_TORCH_DT[dtype]).to(torch.float64).numpy()
    floor = np.max(np.abs(t - o_ref)) if o_ref.size else 0.0
    if floor > O_TOL:
        return O_TOL + half_ulp(o_ref, dtype)
    return np.full_like(o_ref, O_TOL)


def run_gpu(wl: Workload, q, k, v, scale=None):
    o, lse = forward(q, k, v, causal=wl.causal, scale=scale, layout=wl.layout)
    torch.cuda.synchronize()
    rc = fa_get_device_status(None)
    assert rc == 0, f"device status {rc}: a bounded wait expired"
    return o, lse


def compare_full(wl: Workload, scale=None, device="cuda"):
    """Full element-by-element comparison (small problems)."""
    q, k, v = make_qkv(wl, device="cpu")
    o, lse = run_gpu(wl, q.to(device), k.to(device), v.to(device), scale)
    o_ref, lse_ref = attention_batched(q, k, v, scale=scale, causal=wl.causal, layout=wl.layout)
    o_gpu = o.double().cpu().numpy()
    l_gpu = lse.double().cpu().numpy()
    err_o = np.abs(o_gpu - o_ref)
    err_l = np.abs(l_gpu - lse_ref)
    bar = o_bar(o_ref, wl.dtype)
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu)), "non-finite output"
    assert np.all(err_o <= bar), f"{wl}: max|dO| = {err_o.max():.3e}"
    assert err_l.max() <= LSE_TOL, f"{wl}: max|dLSE| = {err_l.max():.3e}"
    return float(err_o.max()), float(err_l.max())


def sample_rows(n: int, rng: np.random.Generator, extra: int = 48):
    fixed = {0, 1, 2, 63, 64, 127, 128, 129, 255, 256, 257, n // 2, n - 129, n - 128, n - 127, n - 2, n - 1}
    rows = {r for r in fixed if 0 <= r < n}
    rows |= set(rng.integers(0, n, size=min(extra, n)).tolist())
    return sorted(rows)


def compare_sampled(wl: Workload, heads, rows_per_head: int = 48, seed: int = 0, o=None, lse=None, qkv=None):
    """Generate on the GPU, run the kernel once, check sampled rows of the
    chosen (b, h) pairs against the oracle evaluated row by row."""
    q, k, v = qkv if qkv is not None else make_qkv(wl, device="cuda")
    if o is None:
        o, lse = run_gpu(wl, q, k, v)
    rng = np.random.default_rng(seed)
    worst_o = worst_l = 0.0
    group = wl.H // wl.kv_heads  # query heads per K/V head (contiguous groups, as the oracle reads GQA)
    for (b, h) in heads:
        hk = h // group
        if wl.layout == "BHND":
            qh, kh, vh, oh = q[b, h], k[b, hk], v[b, hk], o[b, h]
        else:
            qh, kh, vh, oh = q[b, :, h], k[b, :, hk], v[b, :, hk], o[b, :, h]
        rows = sample_rows(wl.Nq, rng, rows_per_head)
        idx = torch.tensor(rows, device=q.device)
        o_ref, l_ref = attention_rows(qh.index_select(0, idx).cpu(), kh.cpu(), vh.cpu(), rows,
                                      scale=None, causal=wl.causal)
        o_gpu = oh.index_select(0, idx).double().cpu().numpy()
        l_gpu = lse[b, h].index_select(0, idx).double().cpu().numpy()
        bar = o_bar(o_ref, wl.dtype)
        err_o = np.abs(o_gpu - o_ref)
        err_l = np.abs(l_gpu - l_ref)
        assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu))
        assert np.all(err_o <= bar), f"{wl.name} b={b} h={h}: max|dO| = {err_o.max():.3e}"
        assert err_l.max() <= LSE_TOL, f"{wl.name} b={b} h={h}: max|dLSE| = {err_l.max():.3e}"
        worst_o = max(worst_o, float(err_o.max()))
        worst_l = max(worst_l, float(err_l.max()))
    return worst_o, worst_l


def default_scale(d):
    return resolve_scale(None, d)


def tflops(wl: Workload, ms: float) -> float:
    return wl.flops / (ms * 1e-3) / 1e12


def isclose(a, b):
    return math.isclose(a, b, rel_tol=1e-9)
