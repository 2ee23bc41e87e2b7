"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small ragged problems are compared element by element; they span several
128-row Q tiles and 128-key KV tiles with ragged tails, both layouts, both
masks, both head dims and all three input dtypes.  The named full-size
workloads are run in the launch configuration the bench uses and checked on
sampled rows (first and last rows, tile boundaries and random rows of a few
heads) that the oracle evaluates one at a time.
"""

import numpy as np
import pytest
import torch

import tiled_attention_13_b200 as fa
from tiled_attention_13_b200.inputs import WORKLOADS, Workload, make_qkv

from .parity import compare_full, compare_sampled, half_ulp, run_gpu

pytestmark = pytest.mark.gpu

SHAPES = [  # (B, H, Nq, Nkv)
    (1, 1, 1, 1),
    (1, 2, 77, 77),
    (1, 1, 128, 128),
    (1, 1, 129, 127),
    (2, 3, 300, 333),
    (2, 1, 255, 257),
    (1, 2, 513, 1000),
    (1, 1, 384, 40),
]


@pytest.fixture(scope="module", autouse=True)
def _lib(fa_lib):
    return fa_lib


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_small_bf16(shape, d, causal, layout):
    B, H, Nq, Nkv = shape
    wl = Workload("small", B=B, H=H, Nq=Nq, Nkv=Nkv, d=d, dtype="bf16", layout=layout, causal=causal,
                  seed=sum(shape) + d)
    compare_full(wl)


def _random_tiny_cases(n=24, seed=20261202):
    """Seeded random tiny problems: Nq, Nkv in [1, 300] (every tail length of
    a 128-row tile is reachable), B in {1, 2}, H in {1, 2, 3}, with head dim,
    layout and mask cycling so that every combination appears."""
    import random

    rng = random.Random(seed)
    cases = []
    for i in range(n):
        cases.append((rng.randint(1, 2), rng.randint(1, 3), rng.randint(1, 300), rng.randint(1, 300),
                      (64, 128)[i % 2], ("BHND", "BSND")[(i // 2) % 2], bool((i // 4) % 2)))
    return cases


@pytest.mark.parametrize("case", _random_tiny_cases(), ids=lambda c: "x".join(map(str, c[:5])) + c[5] + "c" * c[6])
def test_random_tiny_shapes(case):
    """Randomized tiny shapes against the oracle, every element."""
    B, H, nq, nkv, d, layout, causal = case
    compare_full(Workload("rand", B=B, H=H, Nq=nq, Nkv=nkv, d=d, dtype="bf16", layout=layout, causal=causal,
                          seed=nq * 301 + nkv))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", [(2, 3, 300, 333), (1, 2, 513, 1000)], ids=lambda s: "x".join(map(str, s)))
def test_small_fp16(shape, d, causal):
    B, H, Nq, Nkv = shape
    wl = Workload("small16", B=B, H=H, Nq=Nq, Nkv=Nkv, d=d, dtype="fp16", layout="BSND", causal=causal, seed=5)
    compare_full(wl)


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (2, 3, 300, 333), (1, 1, 40, 70)], ids=lambda s: "x".join(map(str, s)))
def test_small_fp32(shape, d, causal, layout):
    B, H, Nq, Nkv = shape
    wl = Workload("small32", B=B, H=H, Nq=Nq, Nkv=Nkv, d=d, dtype="fp32", layout=layout, causal=causal, seed=9)
    compare_full(wl)


def test_explicit_scale_and_regression_inputs():
    """Explicit scale, and page 1's regression families: all-ones, large random
    values and alternating extremes (section 数值安全的边界条件)."""
    wl = Workload("s", B=1, H=2, Nq=200, Nkv=300, d=128, dtype="bf16", layout="BHND", causal=False, seed=3)
    compare_full(wl, scale=0.05)
    from oracle import attention_batched

    shape_q, shape_kv = wl.q_shape(), wl.kv_shape()
    g = torch.Generator().manual_seed(11)
    cases = {
        "ones": (torch.ones(shape_q), torch.ones(shape_kv), torch.randn(shape_kv, generator=g)),
        "large": (torch.randn(shape_q, generator=g) * 8, torch.randn(shape_kv, generator=g) * 8,
                  torch.randn(shape_kv, generator=g)),
        "alternating": (torch.ones(shape_q) * 6 * (1 - 2 * (torch.arange(200) % 2)).view(1, 1, -1, 1),
                        torch.ones(shape_kv) * 6 * (1 - 2 * (torch.arange(300) % 2)).view(1, 1, -1, 1),
                        torch.randn(shape_kv, generator=g)),
    }
    # These inputs are far from N(0, 1): scores spread over hundreds of units,
    # so P is nearly one-hot and O nearly a single row of V.  The bound follows
    # from the arithmetic: rounding O to bf16 costs half an ulp of O, rounding
    # P to bf16 before P V costs at most 2^-9 relative per weight, i.e.
    # 2^-9 max|V| on O; 1e-3 covers the fp32 accumulation.
    for name, (q, k, v) in cases.items():
        q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
        vmax = float(v.float().abs().max())
        for causal in (False, True):
            o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=causal)
            o_ref, l_ref = attention_batched(q, k, v, causal=causal)
            err = np.abs(o.double().cpu().numpy() - o_ref)
            bar = half_ulp(o_ref, "bf16") + 2.0 ** -9 * vmax + 1e-3
            el = np.abs(lse.double().cpu().numpy() - l_ref).max()
            assert np.all(err <= bar), (name, causal, err.max())
            assert el <= 1e-3, (name, causal, el)


def test_deterministic_and_lse_optional():
    wl = Workload("det", B=2, H=4, Nq=700, Nkv=900, d=128, dtype="bf16", layout="BSND", causal=True, seed=21)
    q, k, v = (t.cuda() for t in make_qkv(wl))
    o1, l1 = run_gpu(wl, q, k, v)
    o2, l2 = run_gpu(wl, q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3 = torch.empty_like(q)
    rc = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o3.data_ptr(), None, 2, 4, 700, 900, 128, -1.0, 1,
                   fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o3)
    assert fa.fa_get_device_status(None) == 0


def test_empty_problem_is_a_noop():
    q = torch.zeros((1, 2, 0, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.randn((1, 2, 5, 64), device="cuda").to(torch.bfloat16)
    o, lse = fa.forward(q, k, k)
    assert o.shape == q.shape and lse.shape == (1, 2, 0)


def test_host_pipeline_matches_device_calls():
    """HostPipeline (overlapped host<->device copies across calls) returns, for
    every call, exactly what the device-side call returns on the same inputs,
    including when calls reuse a device buffer set (more calls than slots)."""
    wls = [Workload("pipe", B=1, H=3, Nq=300, Nkv=333, d=128, dtype="bf16", layout="BSND", causal=c, seed=40 + i)
           for i, c in enumerate([True, True, True, True, True])]
    host_in = [tuple(t.cpu().pin_memory() for t in make_qkv(w)) for w in wls]
    outs = [(torch.empty_like(qh).pin_memory(), torch.empty((1, 3, 300), dtype=torch.float32).pin_memory())
            for qh, _, _ in host_in]
    hp = fa.HostPipeline(host_in[0][0], host_in[0][1], causal=True, layout="BSND")
    for (qh, kh, vh), (oh, lh) in zip(host_in, outs):
        hp.submit(qh, kh, vh, oh, lh)
    hp.synchronize()
    for w, (qh, kh, vh), (oh, lh) in zip(wls, host_in, outs):
        od, ld = run_gpu(w, qh.cuda(), kh.cuda(), vh.cuda())
        assert torch.equal(oh, od.cpu()) and torch.equal(lh, ld.cpu())
    o1, l1 = fa.forward_host(*host_in[0], causal=True, layout="BSND")
    assert torch.equal(o1, outs[0][0]) and torch.equal(l1, outs[0][1])


def test_polynomial_exp_option(tmp_path):
    """The kernel built with FA_POLY_EVERY=4 (one exp pair in four on the FMA
    pipe, polynomial 2^x) meets the same bars against the oracle, in a process
    of its own that loads that build."""
    import os
    import subprocess
    import sys

    from tiled_attention_13_b200.build import build_variant

    lib = build_variant(str(tmp_path / "libfa_poly4.so"), {"FA_POLY_EVERY": 4})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("from tests.parity import compare_full\n"
            "from tiled_attention_13_b200.inputs import Workload\n"
            "for c in (False, True):\n"
            "    compare_full(Workload('poly', B=2, H=3, Nq=600, Nkv=700, d=128, dtype='bf16', layout='BSND',"
            " causal=c, seed=77))\n"
            "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env={**os.environ, "FA_B200_LIB": lib},
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]


def test_index_checks_build(tmp_path):
    """The debug build (FA_CHECKS: every computed global index checked on the
    device, a violation reported as FA_ERR_CHECK) runs the contiguous, fp32,
    paged, paged split-KV, band and split-KV paths, the short-key kernels
    (d = 64 and 128), the decoding kernel (contiguous and paged), d = 256,
    block-sparse masks and the backward on ragged shapes with a clean status
    and the usual parity, in a process of its own."""
    import os
    import subprocess
    import sys

    from tiled_attention_13_b200.build import build_variant

    lib = build_variant(str(tmp_path / "libfa_checks.so"), {"FA_CHECKS": 1})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import tiled_attention_13_b200 as fa\n"
            "from tests.parity import compare_full\n"
            "from tests import test_gpu_parity as t\n"
            "from tiled_attention_13_b200.inputs import Workload\n"
            "for c in (False, True):\n"
            "    compare_full(Workload('chk', B=2, H=3, Nq=300, Nkv=333, d=128, dtype='bf16', layout='BSND',"
            " causal=c, seed=7))\n"
            "compare_full(Workload('chk32', B=1, H=2, Nq=70, Nkv=90, d=64, dtype='fp32', layout='BHND', seed=8))\n"
            "pw = Workload('chkp', B=2, H=8, Hkv=2, Nq=7, Nkv=4097, d=128, dtype='bf16', layout='BSND', seed=3,"
            " block_size=16)\n"
            "t._paged_parity(pw)\n"
            "t._paged_parity(pw, num_splits=3)\n"
            "t.test_band_bf16(t.BAND_CASES[1])\n"
            "t.test_splitkv(t.SPLIT_CASES[1])\n"
            "for d, c in ((64, True), (128, False)):\n"
            "    compare_full(Workload('chks', B=2, H=3, Nq=300, Nkv=77, d=d, dtype='bf16', layout='BSND', causal=c,"
            " seed=11))\n"
            "t.test_paged_decode_kernel(t.PAGED_DECODE_CASES[0])\n"
            "from tests import test_gpu_tile1 as t1, test_gpu_bwd as tb\n"
            "t1.test_d256_bf16(t1.D256_SHAPES[2], True, 'BSND')\n"
            "t1.test_block_sparse(t1.BSP_CASES[0])\n"
            "tb.test_bwd_bf16(tb.SHAPES[3], 128, True, 'BSND')\n"
            "tb.test_bwd_bf16(tb.SHAPES[6], 64, False, 'BHND')\n"
            "assert fa.fa_get_device_status(None) == 0\n"
            "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env={**os.environ, "FA_B200_LIB": lib},
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]


# ----------------------------------------------------------------- grouped-query attention
GQA_SHAPES = [  # (B, H, Hkv, Nq, Nkv)
    (1, 8, 1, 300, 333),
    (2, 8, 2, 255, 257),
    (1, 8, 4, 129, 1000),
    (1, 6, 3, 77, 77),
]


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("shape", GQA_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gqa_bf16(shape, d, causal, layout):
    B, H, hkv, Nq, Nkv = shape
    wl = Workload("gqa", B=B, H=H, Hkv=hkv, Nq=Nq, Nkv=Nkv, d=d, dtype="bf16", layout=layout, causal=causal,
                  seed=sum(shape) + d + 7)
    compare_full(wl)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_fp16_and_fp32(causal):
    for dt in ("fp16", "fp32"):
        wl = Workload("gqa-" + dt, B=2, H=6, Hkv=2, Nq=200, Nkv=230, d=64, dtype=dt, layout="BSND", causal=causal,
                      seed=91)
        compare_full(wl)


def test_gqa_llama13b_8k_sampled():
    """The grouped-query bench workload (40 query heads over 8 K/V heads), in
    the launch configuration the bench uses, on sampled rows of heads at both
    ends of several groups."""
    wl = WORKLOADS["llama13b-8k-gqa8"]
    compare_sampled(wl, heads=[(0, 0), (0, 4), (0, 5), (0, 22), (0, 39)], rows_per_head=40, seed=3)


# ----------------------------------------------------------------- paged K/V cache
def _paged_parity(wl, num_splits=None):
    """forward_paged on a cache built from the seeded K/V (shuffled physical
    blocks, NaN in every element the table does not point at) against the
    oracle's gather-then-attend on the same cache and table; with num_splits,
    the split-KV form of the same call."""
    from oracle import attention_paged
    from tiled_attention_13_b200.inputs import make_paged_kv

    from .parity import LSE_TOL, o_bar

    q, k, v = make_qkv(wl)
    kc, vc, table = make_paged_kv(wl, k, v)
    o, lse = fa.forward_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), wl.Nkv, causal=wl.causal,
                              layout=wl.layout, num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    o_ref, l_ref = attention_paged(q, kc, vc, table.numpy(), wl.Nkv, causal=wl.causal, layout=wl.layout)
    o_gpu, l_gpu = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu))
    assert np.all(np.abs(o_gpu - o_ref) <= o_bar(o_ref, wl.dtype)), float(np.abs(o_gpu - o_ref).max())
    assert np.abs(l_gpu - l_ref).max() <= LSE_TOL


@pytest.mark.parametrize("block_size", [16, 64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_paged_bf16(block_size, d, causal):
    wl = Workload("paged", B=2, H=8, Hkv=2, Nq=300, Nkv=300, d=d, dtype="bf16", layout="BSND", causal=causal,
                  block_size=block_size, seed=block_size + d)
    _paged_parity(wl)


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
def test_paged_ragged_mha_and_fp16(layout):
    """Nkv neither a multiple of the block size nor of 128 (the tail rows of
    the last block are NaN in the cache), one K/V head per query head, and
    fp16; query layout BHND and BSND."""
    for dt, hkv in (("bf16", 3), ("fp16", 1)):
        wl = Workload("paged-r", B=2, H=3, Hkv=hkv, Nq=129, Nkv=1000, d=128, dtype=dt, layout=layout,
                      causal=False, block_size=32, seed=17)
        _paged_parity(wl)


def test_paged_llama13b_8k_sampled():
    """The paged bench workload (16-key blocks, 40 query heads over 8 K/V
    heads) on sampled rows: the contiguous K/V it was built from is the
    reference input for the oracle, row by row."""
    from tiled_attention_13_b200.inputs import make_paged_kv

    wl = WORKLOADS["llama13b-8k-gqa8-paged16"]
    q, k, v = make_qkv(wl, device="cuda")
    kc, vc, table = make_paged_kv(wl, k, v)
    o, lse = fa.forward_paged(q, kc, vc, table, wl.Nkv, causal=wl.causal, layout=wl.layout)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    compare_sampled(wl, heads=[(0, 0), (0, 7), (0, 21), (0, 39)], rows_per_head=32, seed=5, o=o, lse=lse,
                    qkv=(q, k, v))


# ----------------------------------------------------------------- decode-shaped calls
@pytest.mark.parametrize("nkv", [1, 129, 4097])
@pytest.mark.parametrize("nq", [1, 7])
def test_decode_shapes_contiguous_and_paged(nq, nkv):
    """A few query rows (one partly filled Q tile) against short to long,
    ragged K/V with grouped heads: contiguous, and through a paged cache of
    16-key blocks (the decode use of a paged cache)."""
    wl = Workload("decode", B=2, H=8, Hkv=2, Nq=nq, Nkv=nkv, d=128, dtype="bf16", layout="BSND", causal=False,
                  seed=nq * 7 + nkv)
    compare_full(wl)
    _paged_parity(wl.with_(block_size=16))


# ----------------------------------------------------------------- band masks
BAND_CASES = [  # (B, H, Hkv, Nq, Nkv, pre_tokens, next_tokens, d, layout)
    (1, 2, 2, 300, 300, 64, 0, 128, "BSND"),     # sliding window of 65 keys
    (2, 2, 1, 300, 333, 100, 50, 64, "BHND"),    # two-sided band, MQA
    (1, 2, 2, 257, 257, 0, 0, 128, "BSND"),      # each row sees only its own key
    (1, 2, 2, 129, 1000, 1000, 1000, 128, "BHND"),  # wider than the sequences: full attention
    (1, 2, 2, 300, 300, 300, 0, 64, "BSND"),     # page 2's causal call
    (1, 8, 2, 513, 513, 200, 17, 128, "BSND"),   # grouped heads, band across tile edges
    (1, 2, 2, 700, 500, 200, 3, 128, "BHND"),    # Nq > Nkv: pre >= Nq - Nkv
]


@pytest.mark.parametrize("case", BAND_CASES, ids=lambda c: "x".join(map(str, c[:7])) + c[8])
def test_band_bf16(case):
    """fa_fwd_band against the oracle's explicit-mask attention on the band."""
    from oracle import attention_masked, band_mask

    from .parity import LSE_TOL, o_bar

    B, H, hkv, nq, nkv, pre, nxt, d, layout = case
    wl = Workload("band", B=B, H=H, Hkv=hkv, Nq=nq, Nkv=nkv, d=d, dtype="bf16", layout=layout, seed=nq + pre + nxt)
    q, k, v = make_qkv(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), layout=layout, band=(pre, nxt))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    if layout == "BSND":
        q, k, v, o = (t.transpose(1, 2) for t in (q, k, v, o))
    mask = band_mask(nq, nkv, pre, nxt)
    g = H // hkv
    for b in range(B):
        for h in range(H):
            o_ref, l_ref = attention_masked(q[b, h], k[b, h // g], v[b, h // g], mask)
            o_gpu, l_gpu = o[b, h].double().cpu().numpy(), lse[b, h].double().cpu().numpy()
            assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu))
            assert np.all(np.abs(o_gpu - o_ref) <= o_bar(o_ref, "bf16")), (b, h, float(np.abs(o_gpu - o_ref).max()))
            assert np.abs(l_gpu - l_ref).max() <= LSE_TOL


# ----------------------------------------------------------------- named workloads
def test_tiny_full():
    for name in ("tiny", "tiny-causal"):
        compare_full(WORKLOADS[name])


def test_cross_attention_full():
    compare_full(WORKLOADS["cross"])


def test_llama13b_2k_full():
    compare_full(WORKLOADS["llama13b-2k"])


@pytest.mark.parametrize("name", ["llama13b-4k", "llama13b-8k", "b4-2k", "b4-2k-causal", "b4-8k",
                                  "b4-8k-causal", "b4-32k", "b4-32k-causal"])
def test_named_sampled(name):
    wl = WORKLOADS[name]
    heads = [(0, 0), (wl.B - 1, wl.H - 1), (wl.B // 2, wl.H // 2)]
    compare_sampled(wl, heads, rows_per_head=40)


def test_long_context_sampled():
    wl = WORKLOADS["long"]
    heads = [(0, 0), (0, wl.H - 1)]
    compare_sampled(wl, heads, rows_per_head=24)
    torch.cuda.empty_cache()


# ----------------------------------------------------------------- split-KV
SPLIT_CASES = [  # (B, H, Hkv, Nq, Nkv, d, layout, dtype, num_splits); 0 = the library's count
    (1, 8, 2, 1, 4097, 128, "BSND", "bf16", 0),     # decode-shaped, ragged last key tile
    (2, 4, 4, 7, 1000, 64, "BHND", "bf16", 3),      # ragged last slice and tile
    (1, 4, 1, 300, 2000, 128, "BSND", "bf16", 5),   # three Q tiles: a pair with an inactive second tile; MQA
    (1, 2, 2, 1, 128, 128, "BSND", "bf16", 4),      # one key tile: one slice, the unsplit kernel
    (1, 2, 2, 129, 9000, 64, "BHND", "bf16", 71),   # one key tile per slice, two Q tiles
    (1, 6, 3, 5, 3000, 128, "BHND", "fp16", 0),     # fp16
    (1, 40, 40, 1, 8192, 128, "BSND", "bf16", 0),   # the LLaMA-13B decode step's shape
    (2, 8, 2, 2, 3001, 64, "BSND", "bf16", 0),      # decode-shaped with 8 rows per K/V head (the most)
    (1, 8, 1, 1, 2000, 128, "BHND", "fp16", 2),     # multi-query decode, fp16, two slices
    (3, 4, 4, 3, 77, 64, "BHND", "bf16", 1),        # decode-shaped, one short slice, final O written directly
    (1, 2, 2, 1, 100000, 128, "BSND", "bf16", 0),   # a long cache: many chunks per warp, ring wrap-around
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=lambda c: "x".join(map(str, c[:6])) + c[6] + c[7] + f"s{c[8]}")
def test_splitkv(case):
    """fa_fwd_splitkv (slices of the key tiles, fp32 partials, LSE merge)
    against the oracle's attention over all keys."""
    from oracle import attention_batched

    from .parity import LSE_TOL, o_bar

    B, H, hkv, nq, nkv, d, layout, dtype, S = case
    wl = Workload("splitkv", B=B, H=H, Hkv=hkv, Nq=nq, Nkv=nkv, d=d, dtype=dtype, layout=layout, causal=False,
                  seed=nq + nkv + S)
    q, k, v = make_qkv(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), layout=layout, num_splits=S)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    o_ref, l_ref = attention_batched(q, k, v, causal=False, layout=layout)
    o_gpu, l_gpu = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu))
    err_o = np.abs(o_gpu - o_ref)
    assert np.all(err_o <= o_bar(o_ref, dtype)), float(err_o.max())
    assert np.abs(l_gpu - l_ref).max() <= LSE_TOL, float(np.abs(l_gpu - l_ref).max())


@pytest.mark.parametrize("num_splits", [0, 3])
@pytest.mark.parametrize("block_size", [16, 128])
def test_paged_splitkv(block_size, num_splits):
    """fa_fwd_paged_splitkv on decode shapes: one and seven query rows per head
    against 4097 keys in a shuffled paged cache (NaN wherever the table does
    not point)."""
    for nq in (1, 7):
        wl = Workload("decode", B=2, H=8, Hkv=2, Nq=nq, Nkv=4097, d=128, dtype="bf16", layout="BSND", causal=False,
                      seed=nq + block_size + num_splits, block_size=block_size)
        _paged_parity(wl, num_splits=num_splits)


PAGED_DECODE_CASES = [  # (B, H, Hkv, Nq, Nkv, d, layout, dtype, block_size, num_splits)
    (3, 4, 4, 1, 1000, 64, "BHND", "bf16", 32, 0),      # d = 64, q and O in BHND
    (1, 8, 1, 1, 70000, 128, "BSND", "fp16", 16, 2),    # multi-query, long slices: table read in many batches
    (2, 6, 3, 4, 2049, 128, "BSND", "bf16", 256, 0),    # 8 rows per K/V head, large blocks, ragged tail
    (1, 2, 2, 1, 17, 64, "BSND", "bf16", 16, 1),        # one slice: O written directly
]


@pytest.mark.parametrize("case", PAGED_DECODE_CASES,
                         ids=lambda c: "x".join(map(str, c[:6])) + c[6] + c[7] + f"bs{c[8]}s{c[9]}")
def test_paged_decode_kernel(case):
    """Decoding-shaped paged split-KV calls (at most 8 query rows per K/V
    head) run on the CUDA-core decode kernel, which reads each 16-key chunk
    through the block table; against the oracle's gather-then-attend."""
    B, H, hkv, nq, nkv, d, layout, dtype, bs, S = case
    wl = Workload("decode-paged", B=B, H=H, Hkv=hkv, Nq=nq, Nkv=nkv, d=d, dtype=dtype, layout=layout, causal=False,
                  seed=nkv + bs + S, block_size=bs)
    _paged_parity(wl, num_splits=S)


def test_splitkv_rejects_a_short_workspace():
    """The workspace is checked against the plan before anything is launched."""
    B, H, nq, nkv, d = 1, 4, 1, 4096, 128
    S, nbytes = fa.splitkv_plan(B, H, nq, nkv, d, 4)
    assert S == 4 and nbytes > 0
    x = torch.zeros((B, nkv, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((B, nq, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, nq), dtype=torch.float32, device="cuda")
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    args = (x.data_ptr(), x.data_ptr(), x.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, H, nq, nkv, d, -1.0, 4)
    assert fa.fa_fwd_splitkv(*args, ws.data_ptr(), nbytes - 16, fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16, None) == 1
    assert fa.fa_fwd_splitkv(*args, None, 0, fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16, None) == 1
    assert fa.fa_fwd_splitkv(*args, ws.data_ptr() + 4, nbytes - 16, fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16, None) == 1
    assert fa.fa_fwd_splitkv(*args, ws.data_ptr() + 4, nbytes, fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16, None) == 3


# ----------------------------------------------------------------- short keys (Nkv <= 128)
# Calls whose keys fit one KV tile run the short-key kernel: one softmax pass
# per query tile, a static contiguous schedule of query tiles per CTA, K/V
# loaded again only when the (batch, K/V head) changes, O written by TMA
# stores from the tile's own Q stage.
SHORT_CASES = [  # (B, H, Hkv, Nq, Nkv, d, layout, causal, dtype)
    (1, 1, 1, 1, 1, 64, "BHND", False, "bf16"),
    (1, 1, 1, 1, 1, 128, "BSND", True, "bf16"),
    (1, 2, 2, 300, 16, 64, "BHND", False, "bf16"),
    (1, 2, 2, 300, 17, 128, "BSND", True, "bf16"),
    (2, 3, 3, 257, 33, 64, "BSND", False, "fp16"),
    (1, 2, 1, 129, 64, 128, "BHND", True, "fp16"),
    (2, 4, 2, 500, 96, 64, "BSND", True, "bf16"),
    (1, 3, 3, 1000, 127, 128, "BHND", False, "bf16"),
    (2, 2, 2, 640, 128, 64, "BHND", True, "bf16"),
    (1, 4, 4, 90, 128, 128, "BSND", False, "fp16"),
    (2, 8, 8, 1024, 77, 64, "BHND", False, "bf16"),
    (1, 8, 2, 2000, 77, 128, "BSND", False, "bf16"),
    (1, 4, 1, 700, 97, 64, "BHND", True, "bf16"),
    (3, 2, 2, 384, 80, 64, "BSND", False, "fp16"),
    (1, 2, 2, 77, 77, 64, "BHND", True, "bf16"),
    (1, 6, 3, 130, 112, 64, "BSND", False, "bf16"),
    (1, 1, 1, 5000, 48, 64, "BHND", True, "fp16"),
]


@pytest.mark.parametrize("case", SHORT_CASES, ids=lambda c: "x".join(map(str, c[:6])) + c[6] + "c" * c[7] + c[8])
def test_short_keys(case):
    B, H, Hkv, Nq, Nkv, d, layout, causal, dtype = case
    compare_full(Workload("short", B=B, H=H, Hkv=Hkv, Nq=Nq, Nkv=Nkv, d=d, dtype=dtype, layout=layout,
                          causal=causal, seed=Nq * 7 + Nkv))


@pytest.mark.parametrize("d", [64, 128])
def test_short_keys_many_tiles_per_cta_and_head_switches(d):
    """Enough query tiles that every CTA wraps its Q ring several times
    (B4 H32 Nq4096: 4096 tiles on <= 148 CTAs), and single-tile heads so that
    a CTA changes K/V head on every tile and reuses both K/V slots; checked on
    sampled rows of several heads."""
    wl = Workload("short-many", B=4, H=32, Nq=4096, Nkv=77, d=d, dtype="bf16", layout="BHND", causal=False, seed=9)
    compare_sampled(wl, [(0, 0), (3, 31), (1, 17), (2, 5)], rows_per_head=40)
    wl = Workload("short-heads", B=5, H=200, Hkv=100, Nq=100, Nkv=120, d=d, dtype="fp16", layout="BSND",
                  causal=True, seed=10)
    compare_sampled(wl, [(0, 0), (4, 199), (2, 101), (3, 50), (1, 1)], rows_per_head=20)


def test_dependent_launches_keep_stream_order():
    """The short-key (d = 64), decode and merge kernels are dependent
    launches: they may start while the previous kernel drains and wait for it
    before touching memory.  Chains where each call reads the previous call's
    output, with no synchronisation in between, must equal the same chains
    synchronised after every call (the kernels are deterministic)."""
    g = torch.Generator().manual_seed(5)
    # cross-attention shape: O of one call is Q of the next
    q = torch.randn(2, 8, 1024, 64, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(2, 8, 77, 64, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(2, 8, 77, 64, generator=g).to(torch.bfloat16).cuda()
    def chain(x, sync):
        outs = []
        for _ in range(4):
            x, _ = fa.forward(x, k, v)  # reads the previous call's output directly
            outs.append(x)
            if sync:
                torch.cuda.synchronize()
        return outs
    a, b = chain(q, False), chain(q, True)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    # decoding shape (split-KV decode kernel and merge): the query of the next
    # step is this step's output
    kd = torch.randn(1, 4096, 8, 128, generator=g).to(torch.bfloat16).cuda()
    vd = torch.randn(1, 4096, 8, 128, generator=g).to(torch.bfloat16).cuda()
    qd = torch.randn(1, 1, 8, 128, generator=g).to(torch.bfloat16).cuda()
    def dchain(x, sync):
        outs = []
        for _ in range(4):
            x, _ = fa.forward(x, kd, vd, layout="BSND", num_splits=0)
            outs.append(x)
            if sync:
                torch.cuda.synchronize()
        return outs
    a, b = dchain(qd, False), dchain(qd, True)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert fa.fa_get_device_status(None) == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
def test_short_keys_reference_max_raised(causal, dtype):
    """The d = 64 short-key kernel takes its reference max from a row's first
    32 keys and raises it when a later 32-key chunk's max passes it by more
    than 2^8, rescaling the P already written.  Keys whose scale grows chunk by
    chunk (x0.1, x1, x4, x8) make that happen two or three times in most
    rows; the result must still be the softmax of the scores.  Bound as for
    page 1's regression inputs: half an output ulp, 2^-9 max|V| for rounding
    P to 16 bits, 1e-3 for the fp32 accumulation."""
    from oracle import attention_batched

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    g = torch.Generator().manual_seed(31)
    B, H, Nq, Nkv, d = 1, 2, 300, 120, 64
    q = torch.randn(B, H, Nq, d, generator=g)
    k = torch.randn(B, H, Nkv, d, generator=g)
    k *= torch.tensor([0.1] * 32 + [1.0] * 32 + [4.0] * 32 + [8.0] * 24).view(1, 1, -1, 1)
    v = torch.randn(B, H, Nkv, d, generator=g)
    q, k, v = (t.to(tdt) for t in (q, k, v))
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    o_ref, l_ref = attention_batched(q, k, v, causal=causal)
    err = np.abs(o.double().cpu().numpy() - o_ref)
    bar = half_ulp(o_ref, dtype) + 2.0 ** -9 * float(v.float().abs().max()) + 1e-3
    assert np.all(err <= bar), err.max()
    assert np.abs(lse.double().cpu().numpy() - l_ref).max() <= 1e-3


@pytest.mark.parametrize("d", [64, 128])
def test_short_keys_bounded_wait_expires_and_context_survives(d):
    """The failure hook on the short-key kernels (d = 64: four tile pipelines
    per CTA; d = 128: two warpgroups): P is never signalled, the MMA issuer's
    bounded wait expires, every role leaves its loop and the status word
    reads FA_ERR_TIMEOUT; the next normal call is correct."""
    wl = Workload("short-fault", B=2, H=8, Nq=1024, Nkv=77, d=d, dtype="bf16", layout="BHND", causal=False, seed=4)
    q, k, v = (t.cuda() for t in make_qkv(wl))
    assert fa.fa_get_device_status(None) == 0
    prev_t = fa.fa_set_wait_timeout_us(50_000)
    prev_f = fa.fa_debug_set_fault(1)
    try:
        fa.forward(q, k, v)
        rc = fa.fa_get_device_status(None)
    finally:
        fa.fa_debug_set_fault(prev_f)
        fa.fa_set_wait_timeout_us(prev_t)
    assert rc == 5, fa.fa_status_string(rc)  # FA_ERR_TIMEOUT
    assert fa.fa_get_device_status(None) == 0
    compare_full(wl)
