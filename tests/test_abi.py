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
    for code in range(8):
        assert fa.fa_status_string(code).startswith("FA_")
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.fa_abi_version() == (1 << 16) | 3


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
    (dict(d=96), 2), (dict(d=256), 2),
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
