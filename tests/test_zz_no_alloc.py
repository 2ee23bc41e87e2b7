"""fa_fwd_noalloc: the entry point for callers that must not allocate device
memory (code inside a memory pool or arena it does not own, services that
reserve all device memory when they start, hosts that forbid cudaMalloc after
start-up).  It must give the same results as fa_fwd, call after call, while
keeping its scheduler counter in a fixed static array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes alone in a fresh
process too (the library fixture builds and loads what it needs).
"""

import numpy as np
import pytest
import torch

import tiled_attention_13_b200 as fa
from tiled_attention_13_b200.inputs import Workload, make_qkv

O_TOL = 1e-2    # the parity tests' bars for O and LSE
LSE_TOL = 1e-3

_DT = {"bf16": fa.FA_DTYPE_BF16, "fp16": fa.FA_DTYPE_FP16, "fp32": fa.FA_DTYPE_FP32}


def _call(entry, wl, q, k, v):
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.H, wl.Nq), dtype=torch.float32, device=q.device)
    rc = entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), wl.B, wl.H, wl.Nq,
               wl.Nkv, wl.d, -1.0, int(wl.causal), fa.FA_LAYOUT_BHND if wl.layout == "BHND" else fa.FA_LAYOUT_BSND,
               _DT[wl.dtype], torch.cuda.current_stream().cuda_stream)
    assert rc == fa.FA_OK, fa.fa_status_string(rc)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == fa.FA_OK
    return o, lse


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [
    Workload("na", B=2, H=3, Nq=700, Nkv=900, d=128, dtype="bf16", layout="BSND", causal=True, seed=31),
    Workload("na", B=1, H=4, Nq=513, Nkv=333, d=64, dtype="fp16", layout="BHND", causal=False, seed=32),
    Workload("na", B=2, H=8, Nq=1024, Nkv=77, d=64, dtype="bf16", layout="BHND", causal=False, seed=33),
], ids=["bf16-d128-causal", "fp16-d64", "cross-like"])
def test_noalloc_matches_fa_fwd_on_two_calls_in_a_row(fa_lib, wl):
    q, k, v = (t.cuda() for t in make_qkv(wl))
    o_ref, lse_ref = _call(fa.fa_fwd, wl, q, k, v)
    for _ in range(2):  # the shared scratch must be ready again for the next call
        o, lse = _call(fa.fa_fwd_noalloc, wl, q, k, v)
        assert np.all(np.isfinite(o.float().cpu().numpy()))
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL
        assert (lse - lse_ref).abs().max().item() <= LSE_TOL


def test_noalloc_rejects_work_beyond_its_fixed_scratch(fa_lib):
    """The counter in the fixed scratch numbers at most 2^31 - 1025 work units;
    a larger call is refused before any CUDA work (fake, never-dereferenced
    16-byte aligned pointers)."""
    a = 1 << 20
    # B*H = 2^20 (b, h) pairs x 2^13 tile pairs (Nq = 2^21) = 2^33 units
    rc = fa.fa_fwd_noalloc(a, a, a, a, a, 1 << 10, 1 << 10, 1 << 21, 64, 64, -1.0, 0, fa.FA_LAYOUT_BHND,
                           fa.FA_DTYPE_BF16, None)
    assert rc == 7 and fa.fa_status_string(rc).startswith("FA_ERR_TOO_LARGE")
