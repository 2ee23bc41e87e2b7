"""GPU parity of the one-tile kernel: head dim 256 and block-sparse masks,
through the C ABI, against the float64 oracle.

d = 256 (page 1, section 分块 Tiling 的计算骨架: head dims of 64-256) is
compared element by element on ragged shapes over both layouts, both masks,
grouped K/V heads and fp16, and on sampled rows of the full-size workload.
Block-sparse masks (page 1, section 总结: SparseFlashAttention) are compared
with ``attention_masked`` over the expanded element mask (intersected with the
causal mask when causal is set), for every head dim, shared and per-head
masks; a query tile that sees no key block returns O = 0 and LSE = -inf.
"""

import numpy as np
import pytest
import torch

import tiled_attention_13_b200 as fa
from oracle import attention_masked, block_sparse_mask
from tiled_attention_13_b200.inputs import WORKLOADS, Workload, make_block_mask, make_qkv

from .parity import LSE_TOL, compare_full, compare_sampled, o_bar

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(fa_lib):
    return fa_lib


D256_SHAPES = [  # (B, H, Hkv, Nq, Nkv)
    (1, 1, 1, 1, 1),
    (1, 2, 2, 77, 77),
    (1, 1, 1, 129, 127),
    (2, 3, 3, 300, 333),
    (1, 2, 2, 513, 1000),
    (1, 4, 2, 384, 640),
    (1, 2, 1, 200, 40),
]


@pytest.mark.parametrize("layout", ["BHND", "BSND"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", D256_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_d256_bf16(shape, causal, layout):
    B, H, Hkv, Nq, Nkv = shape
    compare_full(Workload("d256", B=B, H=H, Hkv=Hkv, Nq=Nq, Nkv=Nkv, d=256, dtype="bf16", layout=layout,
                          causal=causal, seed=Nq + 3 * Nkv))


@pytest.mark.parametrize("causal", [False, True])
def test_d256_fp16(causal):
    compare_full(Workload("d256h", B=2, H=2, Nq=300, Nkv=500, d=256, dtype="fp16", layout="BSND", causal=causal,
                          seed=17))


def test_d256_full_size_sampled():
    wl = WORKLOADS["d256-8k"]
    compare_sampled(wl, [(0, 0), (0, wl.H - 1), (0, wl.H // 2)], rows_per_head=32)


def test_d256_deterministic_and_noalloc_identical():
    """Two calls give the same bits, and fa_fwd_noalloc (ticket counter in its
    fixed scratch) gives the same bits as fa_fwd."""
    wl = Workload("d256det", B=1, H=3, Nq=700, Nkv=900, d=256, dtype="bf16", layout="BHND", causal=True, seed=2)
    q, k, v = (t.cuda() for t in make_qkv(wl))
    o1, l1 = fa.forward(q, k, v, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    o3, l3 = torch.empty_like(q), torch.empty_like(l1)
    rc = fa.fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o3.data_ptr(), l3.data_ptr(), 1, 3, 700, 900,
                           256, -1.0, 1, fa.FA_LAYOUT_BHND, fa.FA_DTYPE_BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3) and torch.equal(l1, l3)


def _heads(x, b, h, layout):
    return x[b, h] if layout == "BHND" else x[b, :, h]


def _check_block_sparse(wl: Workload, mask: torch.Tensor):
    """Run fa_fwd_block_sparse with ``mask`` ([B or 1, H or 1, QT, KT]) and
    compare every row with the oracle over the expanded element mask; rows
    that see no key must come back as O = 0, LSE = -inf."""
    q, k, v = make_qkv(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=wl.causal, layout=wl.layout, block_mask=mask.cuda())
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    group = wl.H // wl.kv_heads
    tril = np.tril(np.ones((wl.Nq, wl.Nkv), dtype=bool))
    n_empty = 0
    for b in range(wl.B):
        for h in range(wl.H):
            bm = mask[b if mask.shape[0] > 1 else 0, h if mask.shape[1] > 1 else 0].numpy()
            em = block_sparse_mask(bm, 128, 128, wl.Nq, wl.Nkv)
            if wl.causal:
                em &= tril
            seen = em.any(axis=1)
            og = _heads(o, b, h, wl.layout).double().cpu().numpy()
            lg = lse[b, h].double().cpu().numpy()
            if seen.any():
                o_ref, l_ref = attention_masked(_heads(q, b, h, wl.layout)[torch.from_numpy(seen)],
                                                _heads(k, b, h // group, wl.layout), _heads(v, b, h // group, wl.layout),
                                                em[seen])
                err_o = np.abs(og[seen] - o_ref)
                assert np.all(err_o <= o_bar(o_ref, wl.dtype)), (b, h, err_o.max())
                assert np.abs(lg[seen] - l_ref).max() <= LSE_TOL, (b, h)
            if (~seen).any():
                n_empty += int((~seen).sum())
                assert np.all(og[~seen] == 0.0) and np.all(np.isneginf(lg[~seen])), (b, h)
    return n_empty


BSP_CASES = [  # (B, H, Hkv, Nq, Nkv, d, layout, causal, dtype, density, shared)
    (1, 2, 2, 300, 333, 64, "BHND", False, "bf16", 0.5, False),
    (2, 2, 1, 513, 1000, 128, "BSND", True, "bf16", 0.4, False),
    (1, 3, 3, 700, 700, 128, "BHND", True, "fp16", 0.3, True),
    (1, 2, 2, 384, 900, 256, "BSND", False, "bf16", 0.5, False),
    (1, 2, 2, 260, 260, 256, "BHND", True, "bf16", 0.6, True),
    (2, 4, 2, 640, 1536, 64, "BSND", False, "fp16", 0.25, False),
]


@pytest.mark.parametrize("case", BSP_CASES, ids=lambda c: "x".join(map(str, c[:6])) + c[6] + "c" * c[7] + c[8])
def test_block_sparse(case):
    B, H, Hkv, Nq, Nkv, d, layout, causal, dtype, density, shared = case
    wl = Workload("bsp", B=B, H=H, Hkv=Hkv, Nq=Nq, Nkv=Nkv, d=d, dtype=dtype, layout=layout, causal=causal,
                  seed=Nq + Nkv + d, block_density=density)
    mask = make_block_mask(wl)
    if shared:
        mask = mask[:1, :1].contiguous()
    _check_block_sparse(wl, mask)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_block_sparse_full_mask_is_plain_attention_and_empty_tiles(d):
    """An all-ones mask gives fa_fwd's result on the same inputs (causal and
    not); a query tile whose mask row is all zero returns O = 0 and
    LSE = -inf while the other tiles stay correct."""
    for causal in (False, True):
        wl = Workload("bspfull", B=1, H=2, Nq=400, Nkv=500, d=d, dtype="bf16", layout="BHND", causal=causal, seed=3)
        compare_full(wl)
        ones = torch.ones((1, 1, 4, 4), dtype=torch.uint8)
        assert _check_block_sparse(wl, ones) == 0
        holes = torch.ones((1, 2, 4, 4), dtype=torch.uint8)
        holes[0, 1, 2, :] = 0  # head 1, query tile 2: no key block
        assert _check_block_sparse(wl, holes) == 128


def test_block_sparse_full_size_sampled():
    """The bench's block-sparse workload (LLaMA-13B 8K causal, half of each
    head's blocks plus the diagonal), sampled rows checked against the oracle
    over each row's visible keys."""
    wl = WORKLOADS["llama13b-8k-bsp50"]
    q, k, v = make_qkv(wl, device="cuda")
    mask = make_block_mask(wl)
    o, lse = fa.forward(q, k, v, causal=True, layout=wl.layout, block_mask=mask.cuda())
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(None) == 0
    rng = np.random.default_rng(0)
    for h in (0, 17, wl.H - 1):
        rows = sorted(set([0, 127, 128, 4095, 8191] + rng.integers(0, wl.Nq, 27).tolist()))
        bm = mask[0, h].numpy()
        qh, kh, vh = q[0, :, h].cpu(), k[0, :, h].cpu(), v[0, :, h].cpu()
        for r in rows:
            vis = np.repeat(bm[r // 128], 128)[: wl.Nkv].astype(bool) & (np.arange(wl.Nkv) <= r)
            o_ref, l_ref = attention_masked(qh[r:r + 1], kh, vh, vis[None, :])
            og = o[0, r, h].double().cpu().numpy()
            assert np.all(np.abs(og - o_ref[0]) <= o_bar(o_ref, "bf16")[0]), (h, r)
            assert abs(float(lse[0, h, r]) - l_ref[0]) <= LSE_TOL, (h, r)


def test_block_sparse_rejects_bad_masks():
    q = torch.zeros((1, 2, 300, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fa.forward(q, q, q, block_mask=torch.ones((1, 2, 3, 2), dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        fa.forward(q, q, q, block_mask=torch.ones((1, 2, 3, 3), dtype=torch.int32, device="cuda"))
    rc = fa.fa_fwd_block_sparse(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), None, None, 0, 0, 1, 2, 2,
                                300, 300, 64, -1.0, 0, fa.FA_LAYOUT_BHND, fa.FA_DTYPE_BF16, None)
    assert rc == 1  # FA_ERR_INVALID_ARG: no mask
