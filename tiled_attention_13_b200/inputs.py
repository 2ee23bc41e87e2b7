"""Seeded synthetic inputs for the attention forward (shared by tests and bench).

This module holds no attention arithmetic: it only draws Q, K and V.  It is the
one module that both the CUDA-side tests and the CPU oracle checks read.

Recipe:

* Q, K, V are i.i.d. N(0, 1) drawn in float32 by ``torch.randn`` from three
  independent generators seeded ``4*seed + 0/1/2`` (Q, K, V), then rounded to
  the storage dtype (bf16, fp16 or fp32) with round-to-nearest-even.
* Long-context K outliers: ``round(frac * N)`` sequence positions chosen by
  ``torch.randperm`` on a CPU generator seeded ``4*seed + 3`` (the same
  positions for every batch and head); ``+3.0`` is added to all d entries of K
  at those positions before the rounding.
* Paged K/V (``block_size > 0``): the keys and values above are placed into
  a cache of ``B * ceil(Nkv / block_size) + 3`` physical blocks in an order
  drawn by ``torch.randperm`` on a CPU generator seeded ``10**9 + seed``;
  every cache element no block-table entry points at (spare blocks, rows past
  Nkv in each sequence's last block) is NaN, so that any read of them shows.
* Block-sparse masks (``block_density > 0``): a uint8 mask [B, H, ceil(Nq/128),
  ceil(Nkv/128)] of 128 x 128 blocks, each entry 1 with probability
  ``block_density`` (``torch.rand`` on a CPU generator seeded
  ``2 * 10**9 + seed``), and the diagonal blocks (kt == qt) always 1, so that
  every row of a causal call sees a key.
* The named workloads are the shapes the surveyed pages benchmark (LLaMA-13B
  self-attention, B=4/H=32/D=128 batched attention, a diffusion cross-attention
  block, 128K long context), plus variants of the LLaMA-13B shape that the
  pages name without sizes: grouped-query (8 K/V heads for its 40 query
  heads), the same through a paged cache, a 2048-key sliding window (band
  mask), one decoding step (one query row per head against an 8192-key
  cache), a block-sparse mask over it, and head dim 256 at the same model
  width (20 heads of 256).  The pages give head dims up to 256 and name
  SparseFlashAttention without a pattern or density.  No dataset, weights or benchmark items are used: every tensor is
  random and only the shapes follow the pages.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

BASE_SEED = 20261202

_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nkv: int
    d: int
    dtype: str = "bf16"
    layout: str = "BHND"
    causal: bool = False
    seed: int = BASE_SEED
    k_outlier: float = 0.0
    outlier_frac: float = 0.0
    Hkv: int = 0  # K/V heads (grouped-query attention); 0 means H
    block_size: int = 0  # > 0: K/V read through a paged cache with blocks of this many keys
    band: tuple = ()  # (pre_tokens, next_tokens): key j visible to query i iff i - pre <= j <= i + next
    num_splits: int = -1  # >= 0: split-KV with that many slices of the key tiles (0: the library's count)
    block_density: float = 0.0  # > 0: block-sparse mask of 128 x 128 blocks with this density (plus the diagonal)
    backward: bool = False  # the step is the backward pass (dQ, dK, dV for a seeded dO), not the forward

    @property
    def kv_heads(self) -> int:
        return self.Hkv if self.Hkv > 0 else self.H

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*B*H*Nq*Nkv*d, halved when causal; with a band
        or a block-sparse mask, 4*d times the number of visible (query, key)
        pairs.  The backward's five products (S, dP, dV, dK, dQ) against the
        forward's two count 2.5 times the forward's."""
        if self.backward:
            return 2.5 * self.with_(backward=False).flops
        if self.block_density > 0:
            return 4.0 * self.d * float(visible_pairs_block(self))
        if self.band:
            pre, nxt = self.band
            i = torch.arange(self.Nq, dtype=torch.float64)
            lo = torch.clamp(i - pre, min=0)
            hi = torch.clamp(i + nxt, max=self.Nkv - 1)
            pairs = float(torch.clamp(hi - lo + 1, min=0).sum())
            return 4.0 * self.B * self.H * self.d * pairs
        f = 4.0 * self.B * self.H * self.Nq * self.Nkv * self.d
        return f / 2 if self.causal else f

    @property
    def bytes_min(self) -> int:
        """Compulsory HBM bytes: read Q, K, V once, write O and the fp32 LSE
        (backward: read Q, K, V, O, dO and the LSE, write dQ, dK, dV)."""
        es = 4 if self.dtype == "fp32" else 2
        if self.backward:
            return (es * self.B * self.d * (4 * self.H * self.Nq + 4 * self.kv_heads * self.Nkv)
                    + 4 * self.B * self.H * self.Nq)
        return (es * self.B * self.d * (2 * self.H * self.Nq + 2 * self.kv_heads * self.Nkv)
                + 4 * self.B * self.H * self.Nq)

    def q_shape(self):
        return (self.B, self.H, self.Nq, self.d) if self.layout == "BHND" else (self.B, self.Nq, self.H, self.d)

    def kv_shape(self):
        hk = self.kv_heads
        return (self.B, hk, self.Nkv, self.d) if self.layout == "BHND" else (self.B, self.Nkv, hk, self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _wl(name, idx, **kw):
    return Workload(name=name, seed=BASE_SEED + idx, **kw)


# The five workload families; idx fixes the seed (BASE_SEED + idx).
WORKLOADS = {
    "tiny": _wl("tiny", 0, B=1, H=2, Nq=256, Nkv=256, d=64, dtype="fp32", layout="BHND"),
    "tiny-causal": _wl("tiny-causal", 0, B=1, H=2, Nq=256, Nkv=256, d=64, dtype="fp32", layout="BHND", causal=True),
    "llama13b-2k": _wl("llama13b-2k", 1, B=1, H=40, Nq=2048, Nkv=2048, d=128, layout="BSND", causal=True),
    "llama13b-4k": _wl("llama13b-4k", 1, B=1, H=40, Nq=4096, Nkv=4096, d=128, layout="BSND", causal=True),
    "llama13b-8k": _wl("llama13b-8k", 1, B=1, H=40, Nq=8192, Nkv=8192, d=128, layout="BSND", causal=True),
    "b4-2k": _wl("b4-2k", 2, B=4, H=32, Nq=2048, Nkv=2048, d=128),
    "b4-2k-causal": _wl("b4-2k-causal", 2, B=4, H=32, Nq=2048, Nkv=2048, d=128, causal=True),
    "b4-8k": _wl("b4-8k", 2, B=4, H=32, Nq=8192, Nkv=8192, d=128),
    "b4-8k-causal": _wl("b4-8k-causal", 2, B=4, H=32, Nq=8192, Nkv=8192, d=128, causal=True),
    "b4-32k": _wl("b4-32k", 2, B=4, H=32, Nq=32768, Nkv=32768, d=128),
    "b4-32k-causal": _wl("b4-32k-causal", 2, B=4, H=32, Nq=32768, Nkv=32768, d=128, causal=True),
    "cross": _wl("cross", 3, B=2, H=8, Nq=4096, Nkv=77, d=64),
    "long": _wl("long", 4, B=1, H=32, Nq=131072, Nkv=131072, d=128, layout="BSND", causal=True,
                k_outlier=3.0, outlier_frac=0.01),
    "llama13b-8k-gqa8": _wl("llama13b-8k-gqa8", 5, B=1, H=40, Hkv=8, Nq=8192, Nkv=8192, d=128, layout="BSND",
                            causal=True),
    "llama13b-8k-swa2k": _wl("llama13b-8k-swa2k", 1, B=1, H=40, Nq=8192, Nkv=8192, d=128, layout="BSND",
                             band=(2047, 0)),
    "llama13b-8k-gqa8-paged16": _wl("llama13b-8k-gqa8-paged16", 5, B=1, H=40, Hkv=8, Nq=8192, Nkv=8192, d=128,
                                    layout="BSND", causal=True, block_size=16),
    # one decoding step of the LLaMA-13B shape: the new token's query rows
    # against an 8192-key cache, batch 1 (online inference), split-KV
    "llama13b-decode-8k": _wl("llama13b-decode-8k", 6, B=1, H=40, Nq=1, Nkv=8192, d=128, layout="BSND",
                              num_splits=0),
    "llama13b-decode-8k-paged16": _wl("llama13b-decode-8k-paged16", 6, B=1, H=40, Nq=1, Nkv=8192, d=128,
                                      layout="BSND", block_size=16, num_splits=0),
    # the LLaMA-13B 8K causal shape with a block-sparse mask: half of the
    # 128 x 128 blocks of each head (plus the diagonal) visible
    "llama13b-8k-bsp50": _wl("llama13b-8k-bsp50", 7, B=1, H=40, Nq=8192, Nkv=8192, d=128, layout="BSND",
                             causal=True, block_density=0.5),
    # head dim 256 at the LLaMA-13B model width (20 heads x 256 = 5120), 8K causal
    "d256-8k": _wl("d256-8k", 8, B=1, H=20, Nq=8192, Nkv=8192, d=256, layout="BSND", causal=True),
    # the backward pass of the LLaMA-13B 8K causal forward, for a seeded N(0, 1) dO
    "llama13b-8k-bwd": _wl("llama13b-8k-bwd", 1, B=1, H=40, Nq=8192, Nkv=8192, d=128, layout="BSND", causal=True,
                           backward=True),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_positions(wl: Workload) -> torch.Tensor:
    """Sequence positions of K that receive +k_outlier (sorted, int64, CPU)."""
    n = int(round(wl.outlier_frac * wl.Nkv))
    if n == 0:
        return torch.zeros((0,), dtype=torch.int64)
    perm = torch.randperm(wl.Nkv, generator=_gen(4 * wl.seed + 3, "cpu"))
    return torch.sort(perm[:n]).values


def make_block_mask(wl: Workload, device="cpu") -> torch.Tensor:
    """The block-sparse mask of ``wl``: uint8 [B, H, ceil(Nq/128), ceil(Nkv/128)]."""
    qt, kt = -(-wl.Nq // 128), -(-wl.Nkv // 128)
    m = torch.rand((wl.B, wl.H, qt, kt), generator=_gen(2 * 10**9 + wl.seed, "cpu")) < wl.block_density
    d = torch.arange(min(qt, kt))
    m[:, :, d, d] = True
    return m.to(torch.uint8).to(device)


def visible_pairs_block(wl: Workload) -> int:
    """(query, key) pairs a block-sparse workload's mask leaves visible
    (intersected with the causal mask when the workload is causal)."""
    m = make_block_mask(wl).to(torch.int64)
    qt, kt = m.shape[2], m.shape[3]
    rows = torch.clamp(wl.Nq - torch.arange(qt) * 128, max=128)
    if not wl.causal:
        cols = torch.clamp(wl.Nkv - torch.arange(kt) * 128, max=128)
        per = rows.view(-1, 1) * cols.view(1, -1)
    else:  # pairs (i, j) with j <= i inside each block, summed exactly
        i = torch.arange(wl.Nq).view(-1, 1)
        lim = torch.clamp(i + 1, max=wl.Nkv)  # keys [0, lim) per row
        k0 = (torch.arange(kt) * 128).view(1, -1)
        cnt = torch.clamp(torch.minimum(lim, k0 + 128) - k0, min=0)  # [Nq, kt]
        per = torch.zeros((qt, kt), dtype=torch.int64).index_add_(0, torch.arange(wl.Nq) // 128, cnt)
    return int((m * per.view(1, 1, qt, kt)).sum())


def make_dout(wl: Workload, device="cpu"):
    """The upstream gradient dO of a backward workload: i.i.d. N(0, 1) in q's
    shape, drawn in fp32 from a generator seeded 7 * seed + 1, rounded to the
    storage dtype."""
    dev = torch.device(device)
    gdev = "cuda" if dev.type == "cuda" else "cpu"
    with torch.cuda.device(dev) if dev.type == "cuda" else _null():
        g = torch.randn(wl.q_shape(), generator=_gen(7 * wl.seed + 1, gdev), device=dev, dtype=torch.float32)
    return g.to(_DTYPES[wl.dtype])


def make_qkv(wl: Workload, device="cpu"):
    """Draw (q, k, v) for ``wl`` on ``device`` in its layout and storage dtype."""
    dev = torch.device(device)
    dt = _DTYPES[wl.dtype]
    gdev = "cuda" if dev.type == "cuda" else "cpu"
    with torch.cuda.device(dev) if dev.type == "cuda" else _null():
        q = torch.randn(wl.q_shape(), generator=_gen(4 * wl.seed + 0, gdev), device=dev, dtype=torch.float32)
        q = q.to(dt)
        k = torch.randn(wl.kv_shape(), generator=_gen(4 * wl.seed + 1, gdev), device=dev, dtype=torch.float32)
        if wl.k_outlier != 0.0 and wl.outlier_frac > 0.0:
            pos = outlier_positions(wl).to(dev)
            axis = 2 if wl.layout == "BHND" else 1
            k.index_add_(axis, pos, torch.full_like(k.index_select(axis, pos), wl.k_outlier))
        k = k.to(dt)
        v = torch.randn(wl.kv_shape(), generator=_gen(4 * wl.seed + 2, gdev), device=dev, dtype=torch.float32)
        v = v.to(dt)
    return q, k, v


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def storage_dtype(name: str) -> torch.dtype:
    return _DTYPES[name]


def make_paged_kv(wl: Workload, k, v, spare: int = 3):
    """Place contiguous k, v (``wl``'s layout) into a paged cache.

    Returns (k_cache, v_cache, block_table): caches [num_blocks, block_size,
    Hkv, d] in k's dtype and device, NaN wherever the table does not point;
    block_table int32 [B, ceil(Nkv / block_size)], logical block i of batch
    entry b -> physical block.  Layout only: no attention arithmetic.
    """
    bs = wl.block_size
    if bs <= 0:
        raise ValueError("workload has no block size")
    kk = k if wl.layout == "BSND" else k.transpose(1, 2)  # [B, Nkv, Hkv, d]
    vv = v if wl.layout == "BSND" else v.transpose(1, 2)
    B, n, hk, d = kk.shape
    nb = -(-n // bs)
    num_blocks = B * nb + spare
    order = torch.randperm(num_blocks, generator=_gen(10**9 + wl.seed, "cpu"))
    table = order[:B * nb].reshape(B, nb).to(torch.int32)
    kc = torch.full((num_blocks, bs, hk, d), float("nan"), dtype=k.dtype, device=k.device)
    vc = torch.full_like(kc, float("nan"))
    for b in range(B):
        for i in range(nb):
            rows = min(bs, n - i * bs)
            phys = int(table[b, i])
            kc[phys, :rows] = kk[b, i * bs:i * bs + rows]
            vc[phys, :rows] = vv[b, i * bs:i * bs + rows]
    return kc, vc, table.to(k.device)

