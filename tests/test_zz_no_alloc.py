"""fa_fwd_noalloc: the entry point for callers that must not allocate device
memory (code inside a memory pool or arena it does not own, services that
reserve all device memory when they start, hosts that forbid cudaMalloc after
start-up).  It must give fa_fwd's results, call after call, while keeping its
scheduler counters in a fixed static array, and it must allocate nothing.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes alone in a fresh
process too (the library fixture builds and loads what it needs).
"""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import tiled_attention_13_b200 as fa
from oracle import attention_batched
from tiled_attention_13_b200.inputs import Workload, make_qkv

O_TOL = 1e-2    # the parity tests' bars for O and LSE against the oracle
LSE_TOL = 1e-3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
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
    Workload("na", B=1, H=2, Nq=70, Nkv=90, d=64, dtype="fp32", layout="BHND", causal=True, seed=34),
], ids=["bf16-d128-causal", "fp16-d64", "cross-like", "fp32"])
def test_noalloc_matches_fa_fwd_on_two_calls_in_a_row(fa_lib, wl):
    q, k, v = make_qkv(wl)
    o_or, lse_or = attention_batched(q, k, v, causal=wl.causal, layout=wl.layout)
    q, k, v = (t.cuda() for t in (q, k, v))
    o_ref, lse_ref = _call(fa.fa_fwd, wl, q, k, v)
    for _ in range(2):  # the shared scratch must be ready again for the next call
        o, lse = _call(fa.fa_fwd_noalloc, wl, q, k, v)
        # the same kernel on the same inputs: bit for bit the same results
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        assert np.abs(o.double().cpu().numpy() - o_or).max() <= O_TOL
        assert np.abs(lse.double().cpu().numpy() - lse_or).max() <= LSE_TOL


_NO_ALLOC_CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    import tiled_attention_13_b200 as fa
    from tiled_attention_13_b200.inputs import Workload, make_qkv
    torch.cuda.set_device(0)
    DT = {{"bf16": fa.FA_DTYPE_BF16, "fp16": fa.FA_DTYPE_FP16, "fp32": fa.FA_DTYPE_FP32}}
    def case(B, H, Nq, Nkv, d, dt, lay, causal, seed):
        wl = Workload("c", B=B, H=H, Nq=Nq, Nkv=Nkv, d=d, dtype=dt, layout=lay, causal=causal, seed=seed)
        q, k, v = (t.cuda() for t in make_qkv(wl))
        return wl, q, k, v, torch.empty_like(q), torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    def run(c):
        wl, q, k, v, o, lse = c
        rc = fa.fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), wl.B, wl.H,
                               wl.Nq, wl.Nkv, wl.d, -1.0, int(wl.causal), 0 if wl.layout == "BHND" else 1,
                               DT[wl.dtype], torch.cuda.current_stream().cuda_stream)
        assert rc == 0, fa.fa_status_string(rc)
    kinds = [(128, "bf16"), (64, "bf16"), (128, "fp16"), (64, "fp16"), (64, "fp32"), (128, "fp32")]
    warm = [case(1, 2, 200, 300, d, dt, "BHND", False, 1) for d, dt in kinds]
    later = [case(2, 3, 700, 900, 128, "bf16", "BSND", True, 2), case(1, 5, 1300, 77, 64, "fp16", "BHND", False, 3),
             case(3, 2, 129, 4000, 128, "fp16", "BSND", False, 4), case(1, 1, 5, 7, 64, "bf16", "BHND", True, 5),
             case(2, 2, 300, 300, 64, "fp32", "BSND", True, 6), case(1, 3, 90, 60, 128, "fp32", "BHND", False, 7)]
    torch.cuda.synchronize()
    for c in warm:  # first use of every kernel this test runs (loads its code)
        run(c)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        for c in later:
            run(c)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    free1, _ = torch.cuda.mem_get_info()
    print("free before", free0, "after", free1)
    assert free1 >= free0, (free0, free1)
    print("NO_ALLOC_OK")
""")


@pytest.mark.gpu
def test_noalloc_allocates_nothing_in_a_fresh_process(fa_lib):
    """In a process that never calls fa_fwd (whose first call allocates 8 KB
    of scheduler counters), calls of fa_fwd_noalloc on new shapes, both head
    dims and all three dtypes leave the device's free memory where it was: an
    allocation of any size would take at least one 2 MB granule.  Every
    kernel the test runs is used once before the free memory is read, so its
    code is already resident on the device."""
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _NO_ALLOC_CHILD.format(root=ROOT)], capture_output=True, text=True,
                       timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0 and "NO_ALLOC_OK" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])


def test_noalloc_rejects_work_beyond_its_fixed_scratch(fa_lib):
    """The counter in the fixed scratch numbers at most 2^31 - 1025 work units;
    a larger call is refused before any CUDA work (fake, never-dereferenced
    16-byte aligned pointers)."""
    a = 1 << 20
    # B*H = 2^20 (b, h) pairs x 2^13 tile pairs (Nq = 2^21) = 2^33 units
    rc = fa.fa_fwd_noalloc(a, a, a, a, a, 1 << 10, 1 << 10, 1 << 21, 64, 64, -1.0, 0, fa.FA_LAYOUT_BHND,
                           fa.FA_DTYPE_BF16, None)
    assert rc == 7 and fa.fa_status_string(rc).startswith("FA_ERR_TOO_LARGE")
