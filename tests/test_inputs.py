"""Seeded input generator: determinism, shapes, dtypes and the outlier recipe."""

import torch

from tiled_attention_13_b200.inputs import WORKLOADS, Workload, make_qkv, outlier_positions


def test_deterministic_and_shaped():
    wl = Workload("t", B=2, H=3, Nq=17, Nkv=9, d=64, dtype="bf16", layout="BSND", seed=7)
    q, k, v = make_qkv(wl)
    q2, k2, v2 = make_qkv(wl)
    assert q.shape == (2, 17, 3, 64) and k.shape == (2, 9, 3, 64) and v.shape == (2, 9, 3, 64)
    assert q.dtype == torch.bfloat16
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    assert not torch.equal(k.float()[:, :9], v.float()[:, :9])  # independent streams


def test_outliers_recipe():
    wl = Workload("t", B=1, H=2, Nq=1000, Nkv=1000, d=8, dtype="fp32", layout="BSND", seed=3,
                  k_outlier=3.0, outlier_frac=0.01)
    pos = outlier_positions(wl)
    assert len(pos) == 10 and len(set(pos.tolist())) == 10
    q, k, v = make_qkv(wl)
    base = make_qkv(wl.with_(k_outlier=0.0, outlier_frac=0.0))[1]
    diff = (k - base)
    mask = torch.zeros(1000, dtype=torch.bool)
    mask[pos] = True
    assert torch.allclose(diff[:, mask], torch.full_like(diff[:, mask], 3.0), atol=1e-6)
    assert torch.count_nonzero(diff[:, ~mask]) == 0


def test_named_workloads():
    assert WORKLOADS["long"].outlier_frac == 0.01 and WORKLOADS["long"].k_outlier == 3.0
    assert round(0.01 * 131072) == 1311
    w = WORKLOADS["llama13b-8k"]
    assert w.flops == 4 * 40 * 8192 * 8192 * 128 / 2
    assert WORKLOADS["cross"].bytes_min == 2 * 2 * 8 * 64 * (2 * 4096 + 2 * 77) + 4 * 2 * 8 * 4096


def test_block_mask_recipe_and_visible_pairs():
    """The block-sparse workloads' mask: seeded, diagonal always visible, and
    the FLOP count's visible-pair total equals a brute-force count over the
    element mask (block mask expanded, intersected with the causal mask)."""
    import numpy as np

    from oracle import block_sparse_mask
    from tiled_attention_13_b200.inputs import Workload, make_block_mask, visible_pairs_block

    for causal in (False, True):
        wl = Workload("bsp", B=2, H=3, Nq=300, Nkv=260, d=64, causal=causal, block_density=0.4, seed=5)
        m = make_block_mask(wl)
        assert m.dtype == torch.uint8 and tuple(m.shape) == (2, 3, 3, 3)
        assert torch.equal(m, make_block_mask(wl))
        assert all(int(m[b, h, i, i]) == 1 for b in range(2) for h in range(3) for i in range(3))
        total = 0
        for b in range(2):
            for h in range(3):
                em = block_sparse_mask(m[b, h].numpy(), 128, 128, wl.Nq, wl.Nkv)
                if causal:
                    em &= np.tril(np.ones((wl.Nq, wl.Nkv), dtype=bool))
                total += int(em.sum())
        assert visible_pairs_block(wl) == total
        assert wl.flops == 4.0 * wl.d * total
