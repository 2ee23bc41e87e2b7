"""B200 (sm_100a) fused scaled-dot-product attention forward.

Python side of the C ABI in ``include/fa.h``: the functions below have the
same names and arguments as the C entry points and only marshal arguments;
every step of the computation runs in the CUDA library ``libfa_b200.so``
(built in-tree by ``python -m tiled_attention_13_b200.build``).  There is no
CPU path: when the library is missing, every call raises.

``forward(q, k, v, ...)`` is the torch-facing convenience wrapper: it takes
CUDA tensors, allocates O and LSE with torch (PyTorch is used for device
memory and streams only) and launches on the current stream.
``forward_host(...)`` is the end-to-end form: pinned host tensors in, host
tensors out, with the copies on the same stream.  ``HostPipeline`` runs a
sequence of such calls with the host<->device copies of neighbouring calls
overlapping the computation (separate copy streams, two device buffer sets).
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "FA_LAYOUT_BHND", "FA_LAYOUT_BSND", "FA_DTYPE_BF16", "FA_DTYPE_FP16", "FA_DTYPE_FP32",
    "FaError", "lib", "lib_path", "fa_fwd", "fa_fwd_gqa", "fa_fwd_band", "fa_fwd_block_sparse", "fa_fwd_paged",
    "fa_fwd_noalloc", "fa_bwd_workspace_size", "fa_bwd", "backward",
    "fa_splitkv_plan", "fa_fwd_splitkv", "fa_fwd_paged_splitkv", "splitkv_plan", "fa_status_string",
    "fa_get_device_status", "fa_set_wait_timeout_us", "fa_debug_set_fault", "fa_abi_version", "forward",
    "forward_paged", "forward_host",
    "HostForward", "HostPipeline", "EXPORTED",
]

FA_LAYOUT_BHND, FA_LAYOUT_BSND = 0, 1
FA_DTYPE_BF16, FA_DTYPE_FP16, FA_DTYPE_FP32 = 0, 1, 2
FA_OK = 0

EXPORTED = ("fa_fwd", "fa_fwd_gqa", "fa_fwd_band", "fa_fwd_block_sparse", "fa_bwd_workspace_size", "fa_bwd",
            "fa_fwd_paged", "fa_fwd_noalloc", "fa_splitkv_plan",
            "fa_fwd_splitkv", "fa_fwd_paged_splitkv", "fa_status_string", "fa_get_device_status", "fa_set_wait_timeout_us", "fa_debug_set_fault", "fa_abi_version")

_LIB = None


def lib_path() -> str:
    """The in-tree library, or another build named by $FA_B200_LIB."""
    return os.environ.get("FA_B200_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")


class FaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {fa_status_string(code)} ({code})" if what else fa_status_string(code))


def lib() -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m tiled_attention_13_b200.build`")
    L = ctypes.CDLL(path)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_float, ctypes.c_int,
                         ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd.restype = ctypes.c_int
    L.fa_fwd_noalloc.argtypes = L.fa_fwd.argtypes
    L.fa_fwd_noalloc.restype = ctypes.c_int
    L.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, ctypes.c_int,
                             ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd_gqa.restype = ctypes.c_int
    L.fa_fwd_band.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, i64, i64, ctypes.c_int,
                              ctypes.c_int, vp]
    L.fa_fwd_band.restype = ctypes.c_int
    L.fa_fwd_block_sparse.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd_block_sparse.restype = ctypes.c_int
    L.fa_bwd_workspace_size.argtypes = [i64, i64, i64, i64, ctypes.POINTER(i64)]
    L.fa_bwd_workspace_size.restype = ctypes.c_int
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float,
                         ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    L.fa_bwd.restype = ctypes.c_int
    L.fa_fwd_paged.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, i64, ctypes.c_float,
                               ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd_paged.restype = ctypes.c_int
    L.fa_splitkv_plan.argtypes = [i64, i64, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                  ctypes.POINTER(i64)]
    L.fa_splitkv_plan.restype = ctypes.c_int
    L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, ctypes.c_float, ctypes.c_int, vp,
                                 i64, ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd_splitkv.restype = ctypes.c_int
    L.fa_fwd_paged_splitkv.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, i64,
                                       ctypes.c_float, ctypes.c_int, vp, i64, ctypes.c_int, ctypes.c_int, vp]
    L.fa_fwd_paged_splitkv.restype = ctypes.c_int
    L.fa_status_string.argtypes = [ctypes.c_int]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_get_device_status.argtypes = [vp]
    L.fa_get_device_status.restype = ctypes.c_int
    L.fa_set_wait_timeout_us.argtypes = [ctypes.c_uint32]
    L.fa_set_wait_timeout_us.restype = ctypes.c_uint32
    L.fa_debug_set_fault.argtypes = [ctypes.c_int]
    L.fa_debug_set_fault.restype = ctypes.c_int
    L.fa_abi_version.argtypes = []
    L.fa_abi_version.restype = ctypes.c_int
    _LIB = L
    return L


# ------------------------------------------------------------------ C ABI, 1:1
def fa_fwd(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, layout, dtype, stream) -> int:
    """int fa_fwd(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, layout, dtype, stream).

    Pointers are integers (device addresses) or None; returns the status code.
    """
    return lib().fa_fwd(q, k, v, o, lse, B, H, Nq, Nkv, d, float(scale), int(causal), int(layout),
                        int(dtype), stream)


def fa_fwd_gqa(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, scale, causal, layout, dtype, stream) -> int:
    """int fa_fwd_gqa(...): k and v hold Hkv heads (Hkv divides H); query head h
    reads K/V head h / (H / Hkv)."""
    return lib().fa_fwd_gqa(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, float(scale), int(causal), int(layout),
                            int(dtype), stream)


def fa_fwd_band(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, scale, pre_tokens, next_tokens, layout, dtype, stream) -> int:
    """int fa_fwd_band(...): key j visible to query i iff i - pre_tokens <= j <=
    i + next_tokens."""
    return lib().fa_fwd_band(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, float(scale), int(pre_tokens), int(next_tokens),
                             int(layout), int(dtype), stream)


def fa_fwd_block_sparse(q, k, v, o, lse, block_mask, mask_batch_stride, mask_head_stride, B, H, Hkv, Nq, Nkv, d,
                        scale, causal, layout, dtype, stream) -> int:
    """int fa_fwd_block_sparse(...): query tile qt of (b, h) sees key tile kt
    iff block_mask[b * mask_batch_stride + h * mask_head_stride + qt * KT + kt]
    != 0 (uint8, 128 x 128 blocks, KT = ceil(Nkv / 128))."""
    return lib().fa_fwd_block_sparse(q, k, v, o, lse, block_mask, int(mask_batch_stride), int(mask_head_stride), B,
                                     H, Hkv, Nq, Nkv, d, float(scale), int(causal), int(layout), int(dtype), stream)


def fa_bwd_workspace_size(B, H, Nq, d):
    """int fa_bwd_workspace_size(...) -> (status, workspace_bytes)."""
    wb = ctypes.c_int64(0)
    rc = lib().fa_bwd_workspace_size(B, H, Nq, d, ctypes.byref(wb))
    return rc, wb.value


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, Nq, Nkv, d, scale, causal, layout,
           dtype, stream) -> int:
    """int fa_bwd(...): dQ, dK, dV of the forward, recomputing P tile by tile
    from q, k and the forward's LSE."""
    return lib().fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, int(workspace_bytes), B, H, Hkv, Nq, Nkv, d,
                        float(scale), int(causal), int(layout), int(dtype), stream)


def backward(q, k, v, o, lse, dout, causal: bool = False, scale=None, layout: str = "BHND", stream=None):
    """(dq, dk, dv) of ``forward(q, k, v, causal, scale, layout)`` for the
    upstream gradient ``dout`` (o and lse are that forward's outputs).  The
    workspace comes from torch's caching allocator."""
    import torch

    for t in (q, k, v, o, dout, lse):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, o, dout and lse must be contiguous CUDA tensors")
    B, H, Nq, Nkv, d = _dims(q, k, layout)
    Hkv = _kv_heads(k, layout)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc, nbytes = fa_bwd_workspace_size(B, H, Nq, d)
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd_workspace_size")
    user_stream = stream is not None
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    if user_stream:
        ws.record_stream(torch.cuda.ExternalStream(stream, device=q.device))
    rc = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(), B, H, Hkv, Nq, Nkv, d,
                -1.0 if scale is None else float(scale), int(bool(causal)),
                FA_LAYOUT_BHND if layout == "BHND" else FA_LAYOUT_BSND, _dtype_code(q), stream)
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def fa_fwd_paged(q, k_cache, v_cache, block_table, o, lse, B, H, Hkv, Nq, Nkv, d, block_size, num_blocks,
                 max_blocks, scale, causal, layout, dtype, stream) -> int:
    """int fa_fwd_paged(...): K/V through a paged cache [num_blocks, block_size,
    Hkv, d] and an int32 block table [B, max_blocks]."""
    return lib().fa_fwd_paged(q, k_cache, v_cache, block_table, o, lse, B, H, Hkv, Nq, Nkv, d, block_size,
                              num_blocks, max_blocks, float(scale), int(causal), int(layout), int(dtype), stream)


def fa_splitkv_plan(B, H, Nq, Nkv, d, num_splits, num_sms):
    """int fa_splitkv_plan(...) -> (status, splits, workspace_bytes)."""
    sp, wb = ctypes.c_int(0), ctypes.c_int64(0)
    rc = lib().fa_splitkv_plan(B, H, Nq, Nkv, d, int(num_splits), int(num_sms), ctypes.byref(sp), ctypes.byref(wb))
    return rc, sp.value, wb.value


def fa_fwd_splitkv(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, scale, num_splits, workspace, workspace_bytes, layout,
                   dtype, stream) -> int:
    """int fa_fwd_splitkv(...): non-causal attention with the key tiles cut into
    slices, each slice's (O, LSE) in the fp32 workspace, then merged."""
    return lib().fa_fwd_splitkv(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, float(scale), int(num_splits), workspace,
                                int(workspace_bytes), int(layout), int(dtype), stream)


def fa_fwd_paged_splitkv(q, k_cache, v_cache, block_table, o, lse, B, H, Hkv, Nq, Nkv, d, block_size, num_blocks,
                         max_blocks, scale, num_splits, workspace, workspace_bytes, layout, dtype, stream) -> int:
    """int fa_fwd_paged_splitkv(...): fa_fwd_splitkv with K/V through a paged cache."""
    return lib().fa_fwd_paged_splitkv(q, k_cache, v_cache, block_table, o, lse, B, H, Hkv, Nq, Nkv, d, block_size,
                                      num_blocks, max_blocks, float(scale), int(num_splits), workspace,
                                      int(workspace_bytes), int(layout), int(dtype), stream)


def fa_fwd_noalloc(q, k, v, o, lse, B, H, Nq, Nkv, d, scale, causal, layout, dtype, stream) -> int:
    """int fa_fwd_noalloc(...): fa_fwd for callers that must not allocate device
    memory (fixed static scratch; calls must not overlap on the GPU)."""
    return lib().fa_fwd_noalloc(q, k, v, o, lse, B, H, Nq, Nkv, d, float(scale), int(causal), int(layout),
                                int(dtype), stream)


def fa_status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def fa_get_device_status(stream=None) -> int:
    return lib().fa_get_device_status(stream)


def fa_set_wait_timeout_us(us: int) -> int:
    return lib().fa_set_wait_timeout_us(int(us))


def fa_debug_set_fault(mode: int) -> int:
    return lib().fa_debug_set_fault(int(mode))


def fa_abi_version() -> int:
    return lib().fa_abi_version()


# ------------------------------------------------------------------ torch wrappers
def _dtype_code(t):
    import torch

    return {torch.bfloat16: FA_DTYPE_BF16, torch.float16: FA_DTYPE_FP16, torch.float32: FA_DTYPE_FP32}[t.dtype]


def _dims(q, k, layout):
    if layout == "BHND":
        B, H, Nq, d = q.shape
        Nkv = k.shape[2]
    elif layout == "BSND":
        B, Nq, H, d = q.shape
        Nkv = k.shape[1]
    else:
        raise ValueError(f"layout must be 'BHND' or 'BSND', got {layout!r}")
    return B, H, Nq, Nkv, d


def _kv_heads(k, layout):
    return k.shape[1] if layout == "BHND" else k.shape[2]


def splitkv_plan(B, H, Nq, Nkv, d, num_splits: int = 0, num_sms: int = 0):
    """(splits, workspace_bytes) of a split-KV call: num_splits <= 0 lets the
    library choose for num_sms SMs (<= 0: the current device's)."""
    rc, sp, wb = fa_splitkv_plan(B, H, Nq, Nkv, d, num_splits, num_sms)
    if rc != FA_OK:
        raise FaError(rc, "fa_splitkv_plan")
    return sp, wb


def _splitkv_workspace(B, H, Nq, Nkv, d, num_splits, device, stream, user_stream):
    """Device workspace for a split-KV call (None when the plan has one
    slice).  Taken from torch's caching allocator; when the call runs on a
    stream other than the current one, the block is tied to that stream so
    that it is not reused before the call's kernels finish."""
    import torch

    _, nbytes = splitkv_plan(B, H, Nq, Nkv, d, num_splits)
    if nbytes == 0:
        return None
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if user_stream:
        ws.record_stream(torch.cuda.ExternalStream(stream, device=device))
    return ws


def forward(q, k, v, causal: bool = False, scale=None, layout: str = "BHND", out=None, lse=None,
            stream=None, band=None, num_splits=None, block_mask=None):
    """O, LSE = softmax(scale Q K^T [+causal]) V on the GPU (returns (o, lse)).

    q: [B,H,Nq,d] (BHND) or [B,Nq,H,d] (BSND); k, v the same with Nkv and
    Hkv heads (Hkv dividing H: grouped-query attention when Hkv < H); all
    contiguous CUDA tensors of one dtype (bf16, fp16 or fp32); d in {64, 128},
    or 256 for bf16/fp16.
    scale None -> 1/sqrt(d).  LSE is fp32 [B, H, Nq].  band = (pre_tokens,
    next_tokens) replaces ``causal``: key j visible to query i iff
    i - pre_tokens <= j <= i + next_tokens (fa_fwd_band; bf16/fp16).
    num_splits (not None; bf16/fp16, no mask) runs split-KV (fa_fwd_splitkv):
    the key tiles cut into that many slices, or as many as the library
    chooses for this device when it is 0.  block_mask (a uint8 CUDA tensor of
    shape [B or 1, H or 1, ceil(Nq/128), ceil(Nkv/128)], bf16/fp16) runs
    fa_fwd_block_sparse: query tile qt sees key tile kt iff the entry is
    nonzero (and causal still applies when set); a size-1 batch or head
    dimension is shared.
    """
    import torch

    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share one dtype")
    B, H, Nq, Nkv, d = _dims(q, k, layout)
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    user_stream = stream is not None
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    sc = -1.0 if scale is None else float(scale)
    Hkv = _kv_heads(k, layout)
    lay = FA_LAYOUT_BHND if layout == "BHND" else FA_LAYOUT_BSND
    lp = lse.data_ptr() if lse.numel() else None
    if num_splits is not None:
        if causal or band is not None or block_mask is not None:
            raise ValueError("split-KV takes no mask (causal=False, band=None, block_mask=None)")
        ws = _splitkv_workspace(B, H, Nq, Nkv, d, int(num_splits), q.device, stream, user_stream)
        rc = fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, B, H, Hkv, Nq, Nkv, d, sc,
                            int(num_splits), None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel(),
                            lay, _dtype_code(q), stream)
        if rc != FA_OK:
            raise FaError(rc, "fa_fwd_splitkv")
        return out, lse
    if block_mask is not None:
        if band is not None:
            raise ValueError("give either band or block_mask")
        import torch as _t

        if block_mask.dtype != _t.uint8 or block_mask.dim() != 4 or not block_mask.is_cuda:
            raise ValueError("block_mask must be a 4-D uint8 CUDA tensor")
        qt, kt = -(-Nq // 128), -(-Nkv // 128)
        if tuple(block_mask.shape[2:]) != (qt, kt) or block_mask.shape[0] not in (1, B) or \
                block_mask.shape[1] not in (1, H) or block_mask.stride(3) != 1 or block_mask.stride(2) != kt:
            raise ValueError(f"block_mask must be [B or 1, H or 1, {qt}, {kt}] with dense last two dims")
        sb = 0 if block_mask.shape[0] == 1 else block_mask.stride(0)
        sh = 0 if block_mask.shape[1] == 1 else block_mask.stride(1)
        rc = fa_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, block_mask.data_ptr(),
                                 sb, sh, B, H, Hkv, Nq, Nkv, d, sc, int(bool(causal)), lay, _dtype_code(q), stream)
        if rc != FA_OK:
            raise FaError(rc, "fa_fwd_block_sparse")
        return out, lse
    if band is not None:
        if causal:
            raise ValueError("give either causal or band")
        pre, nxt = band
        rc = fa_fwd_band(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, B, H, Hkv, Nq, Nkv, d, sc,
                         int(pre), int(nxt), lay, _dtype_code(q), stream)
        if rc != FA_OK:
            raise FaError(rc, "fa_fwd_band")
        return out, lse
    if Hkv == H:
        rc = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, B, H, Nq, Nkv, d, sc,
                    int(bool(causal)), lay, _dtype_code(q), stream)
    else:
        rc = fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, B, H, Hkv, Nq, Nkv, d, sc,
                        int(bool(causal)), lay, _dtype_code(q), stream)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd" if Hkv == H else "fa_fwd_gqa")
    return out, lse


def forward_paged(q, k_cache, v_cache, block_table, seq_len: int, causal: bool = False, scale=None,
                  layout: str = "BSND", out=None, lse=None, stream=None, num_splits=None):
    """O, LSE with K and V gathered through a paged cache (returns (o, lse)).

    q: [B,H,Nq,d] (BHND) or [B,Nq,H,d] (BSND), bf16 or fp16; k_cache, v_cache:
    [num_blocks, block_size, Hkv, d] of q's dtype; block_table: int32
    [B, max_blocks] CUDA tensor; seq_len: keys per sequence.  All contiguous.
    num_splits (not None, causal False) runs split-KV (fa_fwd_paged_splitkv),
    as for forward().
    """
    import torch

    for t in (q, k_cache, v_cache, block_table):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, caches and block_table must be contiguous CUDA tensors")
    if not (q.dtype == k_cache.dtype == v_cache.dtype) or k_cache.shape != v_cache.shape:
        raise ValueError("q and the caches must share one dtype; the two caches one shape")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise ValueError("block_table must be an int32 [B, max_blocks] tensor")
    if layout == "BHND":
        B, H, Nq, d = q.shape
    elif layout == "BSND":
        B, Nq, H, d = q.shape
    else:
        raise ValueError(f"layout must be 'BHND' or 'BSND', got {layout!r}")
    num_blocks, block_size, Hkv, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    user_stream = stream is not None
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    sc = -1.0 if scale is None else float(scale)
    if num_splits is not None:
        if causal:
            raise ValueError("split-KV takes no mask (causal=False)")
        ws = _splitkv_workspace(B, H, Nq, int(seq_len), d, int(num_splits), q.device, stream, user_stream)
        rc = fa_fwd_paged_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                                  out.data_ptr(), lse.data_ptr() if lse.numel() else None, B, H, Hkv, Nq, int(seq_len),
                                  d, block_size, num_blocks, block_table.shape[1], sc, int(num_splits),
                                  None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel(),
                                  FA_LAYOUT_BHND if layout == "BHND" else FA_LAYOUT_BSND, _dtype_code(q), stream)
        if rc != FA_OK:
            raise FaError(rc, "fa_fwd_paged_splitkv")
        return out, lse
    rc = fa_fwd_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(), out.data_ptr(),
                      lse.data_ptr() if lse.numel() else None, B, H, Hkv, Nq, int(seq_len), d, block_size,
                      num_blocks, block_table.shape[1], sc, int(bool(causal)),
                      FA_LAYOUT_BHND if layout == "BHND" else FA_LAYOUT_BSND, _dtype_code(q), stream)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_paged")
    return out, lse


class HostForward:
    """End-to-end form over pinned host tensors with reusable device buffers.

    Each call copies q, k, v host->device, runs fa_fwd and copies O and LSE
    device->host, all on one stream; ``__call__`` returns the pinned host
    outputs (valid after ``torch.cuda.current_stream().synchronize()``).
    """

    def __init__(self, q_host, k_host, v_host, causal=False, scale=None, layout="BHND", device="cuda"):
        import torch

        self.causal, self.scale, self.layout = causal, scale, layout
        self.dev = torch.device(device)
        self.qd = torch.empty_like(q_host, device=self.dev)
        self.kd = torch.empty_like(k_host, device=self.dev)
        self.vd = torch.empty_like(v_host, device=self.dev)
        self.od = torch.empty_like(self.qd)
        B, H, Nq, _, _ = _dims(q_host, k_host, layout)
        self.lsed = torch.empty((B, H, Nq), dtype=torch.float32, device=self.dev)
        self.o_host = torch.empty_like(q_host).pin_memory()
        self.lse_host = torch.empty((B, H, Nq), dtype=torch.float32).pin_memory()
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in (q_host, k_host, v_host))
        self.d2h_bytes = self.o_host.numel() * self.o_host.element_size() + self.lse_host.numel() * 4

    def __call__(self, q_host, k_host, v_host):
        self.qd.copy_(q_host, non_blocking=True)
        self.kd.copy_(k_host, non_blocking=True)
        self.vd.copy_(v_host, non_blocking=True)
        forward(self.qd, self.kd, self.vd, causal=self.causal, scale=self.scale, layout=self.layout,
                out=self.od, lse=self.lsed)
        self.o_host.copy_(self.od, non_blocking=True)
        self.lse_host.copy_(self.lsed, non_blocking=True)
        return self.o_host, self.lse_host


class HostPipeline:
    """End-to-end calls over pinned host tensors, pipelined across calls.

    ``submit(q, k, v, o, lse)`` queues one call: the host->device copy of
    q, k, v (pinned host tensors) on an upload stream, fa_fwd on a compute
    stream, and the device->host copy of O and LSE into the pinned host
    tensors ``o`` and ``lse`` on a download stream.  Two device buffer sets
    alternate, and events order each set's reuse, so call i+1's upload and
    call i-1's download run while call i computes.  ``synchronize()`` waits
    for every queued call; a host output is valid once it has returned.
    """

    def __init__(self, q_host, k_host, causal=False, scale=None, layout="BHND", device="cuda", slots=2):
        import torch

        self.causal, self.scale, self.layout = causal, scale, layout
        self.dev = torch.device(device)
        B, H, Nq, _, _ = _dims(q_host, k_host, layout)
        self.bufs = []
        for _ in range(slots):
            qd = torch.empty_like(q_host, device=self.dev)
            kd = torch.empty_like(k_host, device=self.dev)
            vd = torch.empty_like(k_host, device=self.dev)
            od = torch.empty_like(qd)
            lsed = torch.empty((B, H, Nq), dtype=torch.float32, device=self.dev)
            self.bufs.append((qd, kd, vd, od, lsed))
        self.up = torch.cuda.Stream(self.dev)
        self.comp = torch.cuda.Stream(self.dev)
        self.down = torch.cuda.Stream(self.dev)
        ev = lambda: [torch.cuda.Event() for _ in range(slots)]  # noqa: E731
        self.uploaded, self.computed, self.downloaded = ev(), ev(), ev()
        self.used = [False] * slots
        self.i = 0
        self.h2d_bytes = (q_host.numel() + 2 * k_host.numel()) * q_host.element_size()
        self.d2h_bytes = q_host.numel() * q_host.element_size() + B * H * Nq * 4

    def submit(self, q_host, k_host, v_host, o_host, lse_host):
        import torch

        s = self.i % len(self.bufs)
        qd, kd, vd, od, lsed = self.bufs[s]
        with torch.cuda.stream(self.up):
            if self.used[s]:
                self.up.wait_event(self.computed[s])  # the slot's inputs were read
            qd.copy_(q_host, non_blocking=True)
            kd.copy_(k_host, non_blocking=True)
            vd.copy_(v_host, non_blocking=True)
            self.uploaded[s].record(self.up)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(self.uploaded[s])
            if self.used[s]:
                self.comp.wait_event(self.downloaded[s])  # the slot's outputs were read back
            forward(qd, kd, vd, causal=self.causal, scale=self.scale, layout=self.layout, out=od, lse=lsed,
                    stream=self.comp.cuda_stream)
            self.computed[s].record(self.comp)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.computed[s])
            o_host.copy_(od, non_blocking=True)
            lse_host.copy_(lsed, non_blocking=True)
            self.downloaded[s].record(self.down)
        self.used[s] = True
        self.i += 1

    def synchronize(self):
        for st in (self.up, self.comp, self.down):
            st.synchronize()


def forward_host(q_host, k_host, v_host, causal=False, scale=None, layout="BHND", device="cuda"):
    """One end-to-end call from host tensors; returns host (o, lse) after syncing."""
    import torch

    hf = HostForward(q_host, k_host, v_host, causal=causal, scale=scale, layout=layout, device=device)
    o, lse = hf(q_host, k_host, v_host)
    torch.cuda.current_stream(hf.dev).synchronize()
    return o.clone(), lse.clone()

