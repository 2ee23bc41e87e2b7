"""Failure detection on the GPU without a GPU fault.

The test hook fa_debug_set_fault(1) makes the softmax warps withhold their
"P ready" signal, so the MMA warp's bounded wait expires.  Every role then
leaves its loop, the CTA waits (bounded) for its own copies and MMAs, frees
its tensor memory and exits; fa_get_device_status() reports FA_ERR_TIMEOUT and
the context stays usable for the next, normal call.
"""

import pytest
import torch

import tiled_attention_13_b200 as fa
from tiled_attention_13_b200.inputs import Workload

from .parity import compare_full

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal,d", [(False, 128), (True, 128), (False, 64), (True, 256)],
                         ids=["one-row-kernel", "two-tile-kernel", "two-tile-kernel-d64", "one-tile-kernel-d256"])
def test_bounded_wait_expires_and_context_survives(fa_lib, causal, d):
    """Every kernel family behind fa_fwd: the non-causal d = 128 call runs the
    one-row-per-thread kernel, causal and d = 64 calls the two-tile kernel,
    d = 256 the one-tile kernel."""
    wl = Workload("fault", B=1, H=2, Nq=256, Nkv=300, d=d, dtype="bf16", layout="BHND", causal=causal, seed=4)
    q = torch.randn(wl.q_shape(), device="cuda").to(torch.bfloat16)
    k = torch.randn(wl.kv_shape(), device="cuda").to(torch.bfloat16)
    v = torch.randn(wl.kv_shape(), device="cuda").to(torch.bfloat16)
    assert fa.fa_get_device_status(None) == 0
    prev_t = fa.fa_set_wait_timeout_us(50_000)
    prev_f = fa.fa_debug_set_fault(1)
    try:
        fa.forward(q, k, v, causal=causal)
        rc = fa.fa_get_device_status(None)
    finally:
        fa.fa_debug_set_fault(prev_f)
        fa.fa_set_wait_timeout_us(prev_t)
    assert rc == fa.FA_OK + 5, fa.fa_status_string(rc)  # FA_ERR_TIMEOUT
    assert fa.fa_get_device_status(None) == 0            # read-and-clear
    # the context is intact: a normal call right after is correct
    compare_full(wl)
