"""GPU parity of the backward pass (fa_bwd through the C ABI) against the
float64 oracle ``attention_backward_batched`` (page 1, "CANN ops-transformer
FlashAttentionScore", section 反向传播的重算策略及其合理性).

The stated tolerances are the forward's; the pages give none for the
gradients, so their bar is derived from the arithmetic: P and dS are rounded
to 16 bits before their products (2^-9 relative each), D comes from the
forward's rounded O, and the outputs are rounded to the input dtype.
Each gradient X must satisfy max|X - X_ref| <= 2^-6 max|X_ref| + 1e-3 and
||X - X_ref||_F <= 2^-7 ||X_ref||_F (+ 1e-3 for all-zero references).
"""

import numpy as np
import pytest
import torch

import tiled_attention_13_b200 as fa
from oracle import attention_backward_batched
from tiled_attention_13_b200.inputs import Workload, make_dout, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(fa_lib):
    return fa_lib


def _grad_out(wl: Workload):
    return make_dout(wl)


def _check(name, got, ref):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    mx = float(np.abs(ref).max()) if ref.size else 0.0
    assert np.all(np.isfinite(got)), f"{name}: non-finite"
    assert err.max() <= 2.0 ** -6 * mx + 1e-3, f"{name}: max err {err.max():.3e} vs max|ref| {mx:.3e}"
    fro = float(np.linalg.norm(ref))
    assert float(np.linalg.norm(got - ref)) <= 2.0 ** -7 * fro + 1e-3, f"{name}: Frobenius"


def compare_bwd(wl: Workload):
    q, k, v = make_qkv(wl)
    do = _grad_out(wl)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, causal=wl.causal, layout=wl.layout)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, causal=wl.causal, layout=wl.layout)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    rq, rk, rv = attention_backward_batched(q, k, v, do, causal=wl.causal, layout=wl.layout)
    _check("dQ", dq, rq)
    _check("dK", dk, rk)
    _check("dV", dv, rv)


SHAPES = [  # (B, H, Hkv, Nq, Nkv)
    (1, 1, 1, 1, 1),
    (1, 2, 2, 77, 77),
    (1, 1, 1, 129, 127),
    (2, 3, 3, 300, 333),
    (1, 2, 2, 513, 1000),
    (1, 1, 1, 384, 40),
    (1, 4, 2, 300, 260),
    (1, 3, 1, 200, 450),
]


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bwd_bf16(shape, d, causal, layout):
    B, H, Hkv, Nq, Nkv = shape
    compare_bwd(Workload("bwd", B=B, H=H, Hkv=Hkv, Nq=Nq, Nkv=Nkv, d=d, dtype="bf16", layout=layout, causal=causal,
                         seed=Nq * 5 + Nkv + d))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_bwd_fp16(d, causal):
    compare_bwd(Workload("bwd16", B=2, H=2, Nq=260, Nkv=300, d=d, dtype="fp16", layout="BSND", causal=causal, seed=9))


def test_bwd_workspace_contents_do_not_matter():
    """The call clears the fp32 dQ accumulator itself (in its first kernel):
    a workspace whose bytes are all 0xFF (NaN as fp32) gives the same
    gradients as a fresh one, dK and dV bit for bit (no atomics) and dQ
    within the bound of the determinism test below (its fp32 additions
    come in no fixed order)."""
    wl = Workload("bwdws", B=1, H=2, Nq=400, Nkv=300, d=128, dtype="bf16", layout="BHND", causal=True, seed=5)
    q, k, v = (t.cuda() for t in make_qkv(wl))
    do = _grad_out(wl).cuda()
    o, lse = fa.forward(q, k, v, causal=True)
    ref = fa.backward(q, k, v, o, lse, do, causal=True)
    rc, need = fa.fa_bwd_workspace_size(1, 2, 400, 128)
    assert rc == 0
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr()]
    tail = [1, 2, 2, 400, 300, 128, -1.0, 1, fa.FA_LAYOUT_BHND, fa.FA_DTYPE_BF16, None]
    torch.cuda.synchronize()
    assert fa.fa_bwd(*args, ws.data_ptr(), need, *tail) == 0
    torch.cuda.synchronize()
    assert torch.isfinite(dq.float()).all()
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert (dq.float() - ref[0].float()).abs().max().item() <= 2.0 ** -6 * ref[0].float().abs().max().item()


def test_bwd_deterministic_dk_dv_and_workspace_checks():
    """dK and dV come from one CTA per key tile without atomics: two calls give
    the same bits (dQ is summed with fp32 atomics, so only its value is
    checked).  A missing or short workspace is refused before any launch."""
    wl = Workload("bwddet", B=1, H=2, Nq=400, Nkv=300, d=128, dtype="bf16", layout="BHND", causal=True, seed=3)
    q, k, v = (t.cuda() for t in make_qkv(wl))
    do = _grad_out(wl).cuda()
    o, lse = fa.forward(q, k, v, causal=True)
    a = fa.backward(q, k, v, o, lse, do, causal=True)
    b = fa.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2.0 ** -6 * a[0].float().abs().max().item()
    rc, need = fa.fa_bwd_workspace_size(1, 2, 400, 128)
    assert rc == 0 and need > 1 * 2 * 400 * 128 * 4
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), a[0].data_ptr(),
            a[1].data_ptr(), a[2].data_ptr()]
    tail = [1, 2, 2, 400, 300, 128, -1.0, 1, fa.FA_LAYOUT_BHND, fa.FA_DTYPE_BF16, None]
    assert fa.fa_bwd(*args, None, 0, *tail) == 1           # no workspace
    assert fa.fa_bwd(*args, ws.data_ptr(), need - 1, *tail) == 1  # too small
    assert fa.fa_bwd(*args, ws.data_ptr() + 16, need, *tail) == 3  # not 256-byte aligned
