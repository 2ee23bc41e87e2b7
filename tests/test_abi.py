"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/fa.h, and rejects bad arguments before touching CUDA."""

import os
import re
import subprocess

import pytest

import tiled_attention_13_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(fa_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_entry_points():
    assert declared_symbols() == sorted(fa.EXPORTED)


def test_library_exports_every_declared_symbol(fa_lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    for s in declared_symbols():
        assert s in exported, s
        assert getattr(fa_lib, s) is not None


def test_status_strings_and_version(fa_lib):
    for code in range(9):
        assert fa.fa_status_string(code).startswith("FA_")
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_abi_version() == (1 << 16) | 7


def test_host_settings_roundtrip(fa_lib):
    prev = fa.fa_set_wait_timeout_us(12345)
    assert fa.fa_set_wait_timeout_us(0) == 12345
    assert fa.fa_set_wait_timeout_us(prev) == 2000000
    assert fa.fa_debug_set_fault(1) == 0
    assert fa.fa_debug_set_fault(0) == 1


A16 = 1 << 20  # a 16-byte aligned fake address (never dereferenced)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), 1), (dict(H=-2), 1), (dict(Nq=-1), 1), (dict(Nkv=-5), 1), (dict(d=0), 1),
    (dict(layout=2), 1), (dict(dtype=3), 1), (dict(causal=2), 1),
    (dict(d=96), 2), (dict(d=512), 2), (dict(d=256, dtype=2), 2),
    (dict(Nkv=0), 1),
    (dict(q=None), 1), (dict(o=None), 1),
    (dict(q=A16 + 8), 3), (dict(v=A16 + 4), 3), (dict(lse=A16 + 2), 3),
    (dict(Nq=0, q=None, k=None, v=None, o=None), 0), (dict(B=0), 0), (dict(H=0), 0),
    (dict(B=1 << 31), 2), (dict(Nq=1 << 31), 2),
])
def test_validation_before_any_cuda_call(fa_lib, kw, code):
    args = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=2, Nq=10, Nkv=10, d=64, scale=-1.0, causal=0,
                layout=0, dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"], args["Nq"],
                   args["Nkv"], args["d"], args["scale"], args["causal"], args["layout"], args["dtype"],
                   args["stream"])
    assert rc == code, fa.fa_status_string(rc)


@pytest.mark.parametrize("kw,code", [
    (dict(Hkv=0), 1), (dict(Hkv=-1), 1), (dict(Hkv=3), 1), (dict(Hkv=5), 1), (dict(Hkv=12), 1),
    (dict(H=0, Hkv=0), 0), (dict(d=96), 2), (dict(q=A16 + 8), 3),
])
def test_gqa_validation_before_any_cuda_call(fa_lib, kw, code):
    """fa_fwd_gqa: Hkv must be >= 1 and divide H (here H = 4); the other checks
    are fa_fwd's, in the same order."""
    args = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=4, Hkv=2, Nq=10, Nkv=10, d=64, scale=-1.0, causal=0,
                layout=0, dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd_gqa(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                       args["Hkv"], args["Nq"], args["Nkv"], args["d"], args["scale"], args["causal"],
                       args["layout"], args["dtype"], args["stream"])
    assert rc == code, fa.fa_status_string(rc)


@pytest.mark.parametrize("kw,code", [
    (dict(block_size=24), 1), (dict(block_size=8), 1), (dict(block_size=0), 1),
    (dict(max_blocks=2), 1), (dict(num_blocks=0), 1), (dict(Hkv=3), 1), (dict(bt=None), 1),
    (dict(dtype=2), 2), (dict(d=96), 2),
    (dict(bt=A16 + 2), 3), (dict(kc=A16 + 8), 3),
    (dict(Nq=0), 0), (dict(B=0), 0),
])
def test_paged_validation_before_any_cuda_call(fa_lib, kw, code):
    """fa_fwd_paged: block size a power of two >= 16, a table row long enough
    for Nkv (here 100 keys in blocks of 32 need 4 entries), at least one
    physical block, bf16/fp16 only, a 4-byte aligned table."""
    args = dict(q=A16, kc=A16, vc=A16, bt=A16, o=A16, lse=A16, B=1, H=4, Hkv=2, Nq=10, Nkv=100, d=64,
                block_size=32, num_blocks=8, max_blocks=4, scale=-1.0, causal=0, layout=1, dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd_paged(args["q"], args["kc"], args["vc"], args["bt"], args["o"], args["lse"], args["B"],
                         args["H"], args["Hkv"], args["Nq"], args["Nkv"], args["d"], args["block_size"],
                         args["num_blocks"], args["max_blocks"], args["scale"], args["causal"], args["layout"],
                         args["dtype"], args["stream"])
    assert rc == code, fa.fa_status_string(rc)


@pytest.mark.parametrize("kw,code", [
    (dict(pre=-1), 1), (dict(nxt=-1), 1), (dict(Nq=200, Nkv=100, pre=50), 1), (dict(Hkv=3), 1),
    (dict(dtype=2), 2), (dict(d=96), 2), (dict(q=A16 + 8), 3),
    (dict(B=0), 0), (dict(Nq=0), 0),
])
def test_band_validation_before_any_cuda_call(fa_lib, kw, code):
    """fa_fwd_band: non-negative widths, and pre_tokens >= Nq - Nkv so that the
    last query rows still see a key; bf16/fp16 only."""
    args = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=4, Hkv=2, Nq=10, Nkv=10, d=64, scale=-1.0, pre=3,
                nxt=1, layout=0, dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd_band(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"], args["Hkv"],
                        args["Nq"], args["Nkv"], args["d"], args["scale"], args["pre"], args["nxt"], args["layout"],
                        args["dtype"], args["stream"])
    assert rc == code, fa.fa_status_string(rc)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), 1), (dict(Hkv=3), 1), (dict(layout=2), 1), (dict(dtype=3), 1), (dict(ws_bytes=-1), 1),
    (dict(Nkv=0), 1), (dict(q=None), 1),
    (dict(dtype=2), 2), (dict(d=96), 2), (dict(B=1 << 31), 2),
    (dict(q=A16 + 8), 3), (dict(lse=A16 + 2), 3),
    (dict(B=0), 0), (dict(Nq=0), 0),
])
def test_splitkv_validation_before_any_cuda_call(fa_lib, kw, code):
    """fa_fwd_splitkv: fa_fwd_gqa's checks (no causal flag), bf16/fp16 only,
    a non-negative workspace size; the workspace itself is checked against
    the plan, which needs the device."""
    args = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=4, Hkv=2, Nq=1, Nkv=1000, d=128, scale=-1.0, S=0,
                ws=A16, ws_bytes=1 << 20, layout=1, dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd_splitkv(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                           args["Hkv"], args["Nq"], args["Nkv"], args["d"], args["scale"], args["S"], args["ws"],
                           args["ws_bytes"], args["layout"], args["dtype"], args["stream"])
    assert rc == code, fa.fa_status_string(rc)


@pytest.mark.parametrize("kw,code", [
    (dict(block_size=24), 1), (dict(max_blocks=7), 1), (dict(num_blocks=0), 1), (dict(bt=None), 1),
    (dict(dtype=2), 2), (dict(bt=A16 + 2), 3), (dict(Nq=0), 0),
])
def test_paged_splitkv_validation_before_any_cuda_call(fa_lib, kw, code):
    """fa_fwd_paged_splitkv: fa_fwd_paged's table and block checks (1000 keys
    in blocks of 128 need 8 table entries)."""
    args = dict(q=A16, kc=A16, vc=A16, bt=A16, o=A16, lse=A16, B=1, H=4, Hkv=2, Nq=1, Nkv=1000, d=128,
                block_size=128, num_blocks=9, max_blocks=8, scale=-1.0, S=0, ws=A16, ws_bytes=1 << 20, layout=1,
                dtype=0, stream=None)
    args.update(kw)
    rc = fa.fa_fwd_paged_splitkv(args["q"], args["kc"], args["vc"], args["bt"], args["o"], args["lse"], args["B"],
                                 args["H"], args["Hkv"], args["Nq"], args["Nkv"], args["d"], args["block_size"],
                                 args["num_blocks"], args["max_blocks"], args["scale"], args["S"], args["ws"],
                                 args["ws_bytes"], args["layout"], args["dtype"], args["stream"])
    assert rc == code, fa.fa_status_string(rc)


def _plan_cost(base, nt, s, sms):
    """The plan's wave model, written out: slices of ceil(nt / s) tiles."""
    t = -(-nt // s)
    sc = -(-nt // t)
    return -(-base * sc // sms) * (t + 1), sc


@pytest.mark.parametrize("B,H,Nq,Nkv", [(1, 40, 1, 8192), (8, 32, 1, 32768), (1, 8, 7, 129), (2, 8, 4096, 77),
                                        (1, 40, 8192, 8192), (1, 1, 1, 1), (1, 2, 300, 100000)])
def test_splitkv_plan_follows_its_wave_model(fa_lib, B, H, Nq, Nkv):
    """fa_splitkv_plan with an explicit SM count (no GPU needed): the chosen
    slice count has the least modelled cost of every count up to about four
    units per CTA slot (two slots per SM for Nq <= 8, where the decoding
    kernel runs two CTAs on an SM), no slice is empty, and the workspace is
    splits * B*H*Nq * (d + 1) fp32 values (none for one slice)."""
    d = 128
    S, nbytes = fa.splitkv_plan(B, H, Nq, Nkv, d, 0, 148)
    sms = 2 * 148 if Nq <= 8 else 148
    nt = -(-Nkv // 128)
    base = B * H * (-(-(-(-Nq // 128)) // 2))
    smax = min(nt, -(-4 * sms // base), 4096)
    costs = [_plan_cost(base, nt, s, sms) for s in range(1, smax + 1)]
    best = min(c for c, _ in costs)
    assert _plan_cost(base, nt, S, sms)[0] == best
    t = -(-nt // S)
    assert (S - 1) * t < nt <= S * t  # every slice holds at least one tile
    assert nbytes == (S * B * H * Nq * (d + 1) * 4 if S > 1 else 0)


def test_splitkv_plan_explicit_counts(fa_lib):
    """An explicit count is capped at one slice per key tile and rounded so
    that no slice is empty: 64 tiles in 5 asked slices are 5 slices of 13
    (the last 12); 3 tiles in 9 asked slices are 3."""
    assert fa.splitkv_plan(1, 40, 1, 8192, 128, 5, 148) == (5, 5 * 40 * 129 * 4)
    assert fa.splitkv_plan(1, 40, 1, 300, 128, 9, 148) == (3, 3 * 40 * 129 * 4)
    assert fa.splitkv_plan(1, 40, 1, 8192, 64, 1, 148) == (1, 0)
    assert fa.splitkv_plan(1, 40, 1, 8192, 64, 64, 148) == (64, 64 * 40 * 65 * 4)
    # 7 tiles in 4 asked slices: slices of 2 tiles, so 4 slices (2, 2, 2, 1)
    assert fa.splitkv_plan(1, 1, 1, 7 * 128, 128, 4, 148)[0] == 4
    # 9 tiles in 4 asked slices: slices of 3 tiles, so 3 slices
    assert fa.splitkv_plan(1, 1, 1, 9 * 128, 128, 4, 148)[0] == 3
    rc, _, _ = fa.fa_splitkv_plan(1, 1, 1, 100, 96, 0, 148)
    assert rc == 1


def test_product_path_has_no_cpu_fallback(monkeypatch, tmp_path):
    """With the library absent, the binding raises instead of computing."""
    import importlib

    mod = importlib.reload(fa)
    monkeypatch.setattr(mod, "lib_path", lambda: str(tmp_path / "missing.so"))
    mod._LIB = None
    with pytest.raises(RuntimeError):
        mod.lib()
    importlib.reload(fa)


def test_binding_does_not_import_oracle():
    src = open(os.path.join(ROOT, "tiled_attention_13_b200", "__init__.py")).read()
    for f in os.listdir(os.path.join(ROOT, "tiled_attention_13_b200", "csrc")):
        src += open(os.path.join(ROOT, "tiled_attention_13_b200", "csrc", f)).read()
    assert "oracle" not in src


def test_binding_rejects_host_tensors_and_bad_tables(fa_lib):
    """The Python wrappers check their tensors before calling the library:
    host (CPU) tensors raise ValueError for the contiguous and the paged form
    (without a GPU that check is the first one reached)."""
    import torch

    q = torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)
    kc = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16)
    table = torch.zeros((1, 4), dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.forward_paged(q, kc, kc, table, 40)
    with pytest.raises(ValueError):
        fa.forward(q, q.float(), q)


def test_bwd_workspace_size_and_argument_checks(fa_lib):
    """fa_bwd_workspace_size needs no GPU: an fp32 dQ accumulator plus two
    padded fp32 row arrays, each part rounded up to 256 bytes.  fa_bwd
    refuses bad arguments before touching the device (fake, never
    dereferenced pointers)."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for B, H, Nq, d in [(1, 1, 1, 64), (2, 3, 300, 128), (1, 40, 8192, 128)]:
        rc, nb = fa.fa_bwd_workspace_size(B, H, Nq, d)
        pad = -(-Nq // 128) * 128
        assert rc == 0 and nb == up(B * H * Nq * d * 4) + 2 * up(B * H * pad * 4)
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == (0, 0)
    assert fa.fa_bwd_workspace_size(1, 1, 10, 96)[0] == 1
    assert fa.fa_bwd_workspace_size(-1, 1, 10, 64)[0] == 1
    a = A16
    base = [a] * 9 + [a, 1 << 30]  # q k v o dout lse dq dk dv, workspace, bytes

    def call(**kw):
        args = dict(B=1, H=2, Hkv=2, Nq=300, Nkv=300, d=64, scale=-1.0, causal=0, layout=0, dtype=0)
        args.update(kw)
        ptrs = list(base)
        for i, name in enumerate(["q", "k", "v", "o", "dout", "lse", "dq", "dk", "dv", "ws"]):
            if name in kw:
                ptrs[i] = kw.pop(name)
                args.pop(name, None)
        return fa.fa_bwd(*ptrs, args["B"], args["H"], args["Hkv"], args["Nq"], args["Nkv"], args["d"], args["scale"],
                         args["causal"], args["layout"], args["dtype"], None)

    assert call(d=256) == 2 and call(dtype=2) == 2            # unsupported head dim, fp32
    assert call(Hkv=3) == 1 and call(causal=2) == 1 and call(Nkv=0) == 1
    assert call(lse=None) == 1 and call(dout=None) == 1
    assert call(q=A16 + 8) == 3 and call(lse=A16 + 2) == 3
    assert call(ws=A16 + 16) == 3                             # workspace must be 256-byte aligned
    assert call(B=0) == 0
