"""Failure detection on the device: every wait of the tensor-core kernels is
bounded, and one that runs out must end the launch with a status the host can
read, leaving the context usable.

A one-nanosecond wait budget (misa_set_wait_limit_ns) makes the first wait that
is not already satisfied give up: the kernel raises its CTA-local abort flag,
records MISA_ERR_TIMEOUT in the device status word, lets its own copies and MMAs
land, frees its TMEM and returns.  Nothing here faults, traps or hangs the GPU:
the wait is made to run out, no flag is left unset for ever.  With the default
budget restored, the same launches must reproduce the results taken before.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import inputs_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import _lib
    return _lib


def _stages(lib, g, wl, cand=None):
    """pool, route, score (store mode) and, given candidates, the all-head rerank."""
    _, hl = lib.misa_pool_keys(g["K"], wl.B)
    heads, r = lib.misa_route_heads(g["Q"], g["w"], hl, wl.q_pos0, wl.n_k, wl.B, wl.h, want_r=True)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], wl.q_pos0)
    out = {"heads": heads, "r": r, "logits": logits}
    if cand is not None:
        out["rerank"] = lib.misa_rerank(g["Q"], g["w"], g["K"], cand, wl.q_pos0, wl.k,
                                        want_full=True)[1]
    return out


def test_expired_waits_report_timeout_and_leave_the_context_usable(lib):
    wl = W.small_workload("expiry", n_q=512, q_pos0=20000, n_k=20512, H=64, d=128, B=128, h=8,
                          k=64, seed=5, generator="clustered", kp=512)
    g = inputs_to_device(W.generate(wl))
    assert lib.misa_last_device_status() == lib.MISA_OK
    ref = _stages(lib, g, wl)
    cand = lib.misa_topk(ref["logits"], wl.q_pos0, wl.n_k, wl.kp)
    ref = _stages(lib, g, wl, cand)
    torch.cuda.synchronize()
    assert lib.misa_last_device_status() == lib.MISA_OK
    try:
        for name in ("route", "score", "rerank"):
            lib.misa_set_wait_limit_ns(1)
            if name == "route":
                _, hl = lib.misa_pool_keys(g["K"], wl.B)
                lib.misa_route_heads(g["Q"], g["w"], hl, wl.q_pos0, wl.n_k, wl.B, wl.h)
            elif name == "score":
                lib.misa_score_tokens(g["Q"], g["w"], ref["heads"], g["K"], wl.q_pos0)
            else:
                lib.misa_rerank(g["Q"], g["w"], g["K"], cand, wl.q_pos0, wl.k)
            st = lib.misa_last_device_status()       # synchronises the stream
            assert st == lib.MISA_ERR_TIMEOUT, f"{name}: status {st}"
            assert lib.misa_last_device_status() == lib.MISA_OK   # read once, then cleared
    finally:
        lib.misa_set_wait_limit_ns(0)                 # the default budget again
    again = _stages(lib, g, wl, cand)
    torch.cuda.synchronize()
    assert lib.misa_last_device_status() == lib.MISA_OK
    for key in ("heads", "r", "rerank"):
        assert np.array_equal(ref[key].cpu().numpy(), again[key].cpu().numpy()), key
    # logits: every causal entry (the rest of a row is not part of the result)
    causal = np.arange(wl.n_k)[None, :] <= (wl.q_pos0 + np.arange(wl.n_q))[:, None]
    a, b = ref["logits"].cpu().numpy(), again["logits"].cpu().numpy()
    assert np.array_equal(a[causal], b[causal])
