"""Plain, slow, obviously-correct float64 attention forward (the oracle).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  No blocking, fusion or
reordering beyond what the definition states, except that query rows are
processed in independent row blocks so that the full score matrix never has to
be held at once (each row's result depends on that row alone).

Sources (the three surveyed web pages):

* Page 1 -- "CANN ops-transformer FlashAttentionScore" (nanhubrain.csdn.net),
  section 平方级显存的精确来源: the three-step definition
  S = Q K^T / sqrt(d_k), P = softmax(S), O = P V; section 在线 Softmax 的数学
  原理拆解: softmax(x)_i = exp(x_i - max x) / sum_j exp(x_j - max x) and the
  one-block online update of (m, l); section 分块 Tiling 的计算骨架: the
  Q-tile-outer / KV-tile-inner loop that writes O, row_max and row_sum.
* Page 2 -- "FlashAttention on Ascend via ops-transformer" (pwwt.cn), section
  标准 vs IO-Aware 实现: naive_attention (scores / sqrt(d_k), softmax, @ V).
* Page 3 -- "ops-nn efficient attention for AIGC" (ascendai.csdn.net), section
  2.2 在线 Softmax 算法: the accumulator form
  new_output = prev_output * correction + exp(S - new_max) @ V; section 6.1
  完整示例代码: causal mask = triu(ones(Nq, Nkv), diagonal=1) -> -inf, i.e.
  key j is visible to query i iff j <= i; scale = d ** -0.5 by default
  (section 3.1 Config: softmax_scale = -1 means 1/sqrt(d)).

Readings where the pages are silent or garbled:

* The page-1 tiling listing divides the block's P by its own sum l_ij inside
  the loop and again by l_prev at the end; the page-2 update divides new_out by
  new_sum every step.  Both contradict page 1's own claim (same section) that
  the tiled result equals the global softmax exactly.  The reading taken is
  page 3's unnormalised accumulator, divided by l once at the end.
* The pages return row_max and row_sum; this oracle returns one per-row
  log-sum-exp LSE = m + ln(l) in natural-log units of the *scaled* scores.
* Causal alignment for Nq != Nkv is not stated; the reading is page 3's
  triu(diagonal=1) applied to the [Nq, Nkv] score matrix (top-left aligned):
  key j visible to query i iff j <= i.
* scale <= 0 or NaN means "auto" = 1/sqrt(d) (page 3, Config softmax_scale=-1).
* The page-1 numerical-safety clamp/reset of the rescale factor is NOT applied
  (it would change the exact result); underflow to 0 is the correct limit.
"""

from __future__ import annotations

import math

import numpy as np

ROW_BLOCK = 1024  # query rows per independent block (memory bound only)


def resolve_scale(scale, d: int) -> float:
    """Softmax scale: the given value, or 1/sqrt(d) when it is None, <= 0 or NaN.

    Page 3, section 3.1 (Config.softmax_scale = -1 -> 1/sqrt(d)) and section 3.3
    (attribute table: softmax_scale defaults to "auto").
    """
    if scale is None:
        return 1.0 / math.sqrt(d)
    s = float(scale)
    if not (s > 0.0):  # catches <= 0 and NaN
        return 1.0 / math.sqrt(d)
    return s


def allowed_keys(i: int, nkv: int, causal: bool) -> np.ndarray:
    """Indices of the keys query row ``i`` attends to.

    Non-causal: all keys 0..Nkv-1.  Causal: page 3 section 6.1,
    triu(ones(Nq, Nkv), diagonal=1) is masked, so key j is visible iff j <= i.
    """
    if not causal:
        return np.arange(nkv)
    return np.arange(min(i + 1, nkv))


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor (bf16/fp16/fp32 -> f64 is exact)
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attention(q, k, v, scale=None, causal: bool = False, row_offset: int = 0):
    """Naive attention for one (batch, head): returns (O [Nq, d], LSE [Nq]).

    ``row_offset`` is the sequence position of q's first row (it only moves the
    causal mask), so a block of query rows can be evaluated on its own.

    Page 1 section 平方级显存的精确来源 and page 2 naive_attention:
      s_ij = scale * sum_c q_ic k_jc            (j in the allowed set A_i)
      m_i  = max_j s_ij
      l_i  = sum_j exp(s_ij - m_i)               (page 1 softmax definition)
      O_i  = sum_j exp(s_ij - m_i) v_j / l_i
      LSE_i = m_i + ln l_i
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    nq, d = q.shape
    nkv = k.shape[0]
    if nq == 0:
        return np.zeros((0, v.shape[1])), np.zeros((0,))
    if nkv == 0:
        raise ValueError("attention over an empty key set is undefined")
    sc = resolve_scale(scale, d)
    o = np.empty((nq, v.shape[1]), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    for r0 in range(0, nq, ROW_BLOCK):
        r1 = min(nq, r0 + ROW_BLOCK)
        s = sc * (q[r0:r1] @ k.T)  # [r, Nkv]
        if causal:
            rows = np.arange(r0, r1)[:, None] + row_offset
            cols = np.arange(nkv)[None, :]
            s = np.where(cols > rows, -np.inf, s)
        m = s.max(axis=1)
        e = np.exp(s - m[:, None])
        l = e.sum(axis=1)
        o[r0:r1] = (e @ v) / l[:, None]
        lse[r0:r1] = m + np.log(l)
    return o, lse


def attention_rows(q_rows, k, v, rows, scale=None, causal: bool = False):
    """The same definition evaluated only at the query positions ``rows``.

    ``q_rows[t]`` is the query vector of global row ``rows[t]`` (the row index
    matters only for the causal mask).  Used to check sampled outputs of
    full-size problems one row at a time.
    """
    q_rows = _as_f64(q_rows)
    k = _as_f64(k)
    v = _as_f64(v)
    d = q_rows.shape[1]
    sc = resolve_scale(scale, d)
    nkv = k.shape[0]
    o = np.empty((len(rows), v.shape[1]))
    lse = np.empty((len(rows),))
    for t, i in enumerate(rows):
        a = allowed_keys(int(i), nkv, causal)
        s = sc * (k[a] @ q_rows[t])
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        o[t] = (e @ v[a]) / l
        lse[t] = m + math.log(l)
    return o, lse


def attention_batched(q, k, v, scale=None, causal: bool = False, layout: str = "BHND"):
    """Apply ``attention`` to every (b, h).  Layouts (page 2 input_layout):

    * "BHND": q [B, H, Nq, d], k/v [B, Hkv, Nkv, d]
    * "BSND": q [B, Nq, H, d], k/v [B, Nkv, Hkv, d]

    Hkv < H is grouped-query attention (page 1, section GatherPAKVCache 的显存
    管理逻辑: under GQA/MQA there are fewer K/V heads than query heads, and the
    needed head is selected; page 3, section 7.3 names GQA and MQA).  The pages
    do not fix which query heads share a K/V head; the reading taken is
    contiguous groups: query head h uses K/V head h // (H // Hkv).  Hkv must
    divide H; Hkv == H is ordinary multi-head attention.

    Returns O in the input layout and LSE [B, H, Nq] (head-major for both).
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    if layout == "BSND":
        q = q.transpose(0, 2, 1, 3)
        k = k.transpose(0, 2, 1, 3)
        v = v.transpose(0, 2, 1, 3)
    elif layout != "BHND":
        raise ValueError(f"unknown layout {layout!r}")
    B, H, nq, _ = q.shape
    hkv = k.shape[1]
    if hkv < 1 or H % hkv != 0 or v.shape[1] != hkv:
        raise ValueError(f"K/V heads ({hkv}) must divide the query heads ({H})")
    group = H // hkv
    o = np.empty((B, H, nq, v.shape[3]))
    lse = np.empty((B, H, nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention(q[b, h], k[b, h // group], v[b, h // group], scale, causal)
    if layout == "BSND":
        o = o.transpose(0, 2, 1, 3)
    return o, lse


def online_softmax_step(m_prev, l_prev, x_t):
    """One block of the online softmax statistics (page 1, section 在线 Softmax
    的数学原理拆解): m_t = max x_t, s_t = sum exp(x_t - m_t),
    m_cur = max(m_prev, m_t), l_cur = l_prev e^(m_prev - m_cur) + s_t e^(m_t - m_cur).
    """
    m_t = float(np.max(x_t))
    s_t = float(np.sum(np.exp(x_t - m_t)))
    m_cur = max(m_prev, m_t)
    prev = 0.0 if l_prev == 0.0 else l_prev * math.exp(m_prev - m_cur)
    l_cur = prev + s_t * math.exp(m_t - m_cur)
    return m_cur, l_cur


def attention_tiled_online(q, k, v, block_r: int, block_c: int, scale=None, causal: bool = False):
    """The tiled online-softmax form (page 1 section 分块 Tiling 的计算骨架, loop
    order Q tile outer / KV tile inner, with page 3 section 2.2's unnormalised
    accumulator), in float64, for any tile sizes.  Returns (O, LSE).

    For Q tile i and KV tile j:
      S      = scale * q_i k_j^T  (masked entries -> -inf)
      m_new  = max(m_prev, rowmax S)
      corr   = exp(m_prev - m_new)
      l      = l * corr + rowsum exp(S - m_new)
      o      = o * corr + exp(S - m_new) @ v_j
    and after the last KV tile O_i = o / l, LSE_i = m + ln l.  This exists only
    to pin the claim (page 1, same section) that tiling changes nothing.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    nq, d = q.shape
    nkv = k.shape[0]
    sc = resolve_scale(scale, d)
    O = np.empty((nq, v.shape[1]))
    LSE = np.empty((nq,))
    for r0 in range(0, nq, block_r):
        r1 = min(nq, r0 + block_r)
        m = np.full((r1 - r0,), -np.inf)
        l = np.zeros((r1 - r0,))
        o = np.zeros((r1 - r0, v.shape[1]))
        for c0 in range(0, nkv, block_c):
            c1 = min(nkv, c0 + block_c)
            s = sc * (q[r0:r1] @ k[c0:c1].T)
            if causal:
                rows = np.arange(r0, r1)[:, None]
                cols = np.arange(c0, c1)[None, :]
                s = np.where(cols > rows, -np.inf, s)
            m_new = np.maximum(m, s.max(axis=1))
            # rows whose every key so far is masked keep m = -inf; use 0 as the
            # reference there so that exp(-inf - (-inf)) never appears
            ref = np.where(np.isneginf(m_new), 0.0, m_new)
            corr = np.exp(m - ref)
            e = np.exp(s - ref[:, None])
            l = l * corr + e.sum(axis=1)
            o = o * corr[:, None] + e @ v[c0:c1]
            m = m_new
        O[r0:r1] = o / l[:, None]
        LSE[r0:r1] = m + np.log(l)
    return O, LSE


def gather_paged_kv(cache, block_table, seq_len: int):
    """Contiguous keys (or values) of one sequence from a paged cache.

    Page 1, section GatherPAKVCache 的显存管理逻辑: the cache is stored in
    fixed-size physical blocks; a block table translates the sequence's
    logical block i (its keys [i*bs, (i+1)*bs)) to the physical block holding
    them, so the blocks of one sequence need not be adjacent.  Reading of the
    layout (the page's listing is inconsistent about which axis holds the
    heads): ``cache`` is [num_blocks, block_size, Hkv, d]; the result is
    [seq_len, Hkv, d], made of logical blocks 0 .. ceil(seq_len/bs) - 1 in
    order, cut to seq_len rows.  Table entries past those blocks are not read.
    """
    cache = _as_f64(cache)
    bs = cache.shape[1]
    n_blocks = -(-seq_len // bs)
    table = np.asarray(block_table).reshape(-1)
    if n_blocks > table.shape[0]:
        raise ValueError("block table shorter than the sequence")
    rows = []
    for i in range(n_blocks):
        phys = int(table[i])
        if not 0 <= phys < cache.shape[0]:
            raise ValueError(f"block table entry {i} = {phys} out of range")
        rows.append(cache[phys])
    out = np.concatenate(rows, axis=0) if rows else np.zeros((0,) + cache.shape[2:])
    return out[:seq_len]


def attention_paged(q, k_cache, v_cache, block_tables, seq_len: int, scale=None, causal: bool = False,
                    layout: str = "BSND"):
    """Attention with K/V read through a paged cache: for every batch entry b,
    K and V are ``gather_paged_kv`` of ``block_tables[b]`` (``seq_len`` keys,
    Hkv heads), then ``attention_batched`` as for contiguous K/V (grouped-query
    when Hkv < H).  q is [B, H, Nq, d] (BHND) or [B, Nq, H, d] (BSND); O comes
    back in q's layout, LSE as [B, H, Nq]."""
    tables = np.asarray(block_tables)
    k = np.stack([gather_paged_kv(k_cache, tables[b], seq_len) for b in range(tables.shape[0])])
    v = np.stack([gather_paged_kv(v_cache, tables[b], seq_len) for b in range(tables.shape[0])])
    if layout == "BHND":
        k = k.transpose(0, 2, 1, 3)
        v = v.transpose(0, 2, 1, 3)
    elif layout != "BSND":
        raise ValueError(f"unknown layout {layout!r}")
    return attention_batched(q, k, v, scale=scale, causal=causal, layout=layout)


def merge_partials(o_parts, lse_parts):
    """Attention over a key set split into parts, from each part's own result:
    with O_r, LSE_r the attention of the same query rows over key part r,
    LSE = log sum_r exp(LSE_r) and O = sum_r exp(LSE_r - LSE) O_r.  This is the
    online-softmax merge (page 1, section 在线 Softmax 的数学原理拆解) applied
    to whole parts, the step that splitting the keys across workers (page 1's
    Ring Attention, split-KV decoding) needs.  A part with no visible key for a
    row has LSE_r = -inf and weight 0.  o_parts [R, ..., d], lse_parts [R, ...].
    """
    o = _as_f64(o_parts)
    lse = _as_f64(lse_parts)
    m = np.max(lse, axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse - m_safe)
    tot = np.sum(w, axis=0)
    out_lse = m_safe + np.log(tot)
    out_o = np.sum(w[..., None] * o, axis=0) / tot[..., None]
    return out_o, out_lse


def band_mask(nq: int, nkv: int, pre_tokens: int, next_tokens: int) -> np.ndarray:
    """Visible (query, key) pairs of a band: key j is visible to query i iff
    i - pre_tokens <= j <= i + next_tokens.  Page 2's flash_attention_score
    takes pre_tokens / next_tokens and calls it with pre_tokens = seq_len,
    next_tokens = 0 for causal inference; that call's meaning (every earlier
    key, no later one) is the reading taken for other values."""
    i = np.arange(nq).reshape(-1, 1)
    j = np.arange(nkv).reshape(1, -1)
    return (j >= i - pre_tokens) & (j <= i + next_tokens)


def block_sparse_mask(block_mask, block_r: int, block_c: int, nq: int, nkv: int) -> np.ndarray:
    """Element mask of a block-sparse pattern (page 1, SparseFlashAttention:
    key blocks marked as not needed are skipped): query tile a (rows
    [a*block_r, ...)) sees key tile b (keys [b*block_c, ...)) iff
    block_mask[a, b]."""
    bm = np.asarray(block_mask, dtype=bool)
    rows = np.arange(nq) // block_r
    cols = np.arange(nkv) // block_c
    return bm[rows][:, cols]


def attention_masked(q, k, v, mask, scale=None):
    """The definition with an explicit boolean mask [Nq, Nkv] of visible
    (query, key) pairs: softmax over each row's visible keys only.  Every row
    must see at least one key."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    mask = np.asarray(mask, dtype=bool)
    if mask.shape != (q.shape[0], k.shape[0]):
        raise ValueError("mask must be [Nq, Nkv]")
    if q.shape[0] and not np.all(mask.any(axis=1)):
        raise ValueError("a query row sees no key")
    sc = resolve_scale(scale, q.shape[1])
    s = np.where(mask, sc * (q @ k.T), -np.inf)
    m = np.max(s, axis=1, keepdims=True) if q.shape[0] else np.zeros((0, 1))
    e = np.exp(s - m)
    z = np.sum(e, axis=1, keepdims=True)
    return (e @ v) / z, (m + np.log(z)).reshape(-1)

