"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point its header declares, and rejects bad arguments before any
launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "misa.h")


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import build
    build.build()
    from long_context_sparse_block_b200 import _lib
    return _lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(misa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_stage_calls():
    names = declared_functions()
    for n in ("misa_pool_keys", "misa_route_heads", "misa_score_tokens", "misa_topk",
              "misa_rerank", "misa_workspace_size", "misa_status_string",
              "misa_last_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(so, name), name


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert lib.misa_status_string(st) != "unknown status"
    assert lib.misa_status_string(12345) == "unknown status"


def test_workspace_size(lib):
    assert lib.misa_workspace_size("rerank", 8192, 131072, 2048, 8192) == 8192 * 8192 * 4
    assert lib.misa_workspace_size("topk", 8192, 131072, 2048, 0) == 0
    assert lib.misa_workspace_size("rerank", 0, 10, 1, 1) == 0


def test_workspace_size_fused(lib):
    ws = lambda n_q, n_k, k: lib.misa_workspace_size("score_topk", n_q, n_k, k, 0)
    assert ws(8192, 131072, 2048) > 0
    assert ws(8192, 131072, 8192) > 0
    assert ws(8192, 4095, 64) == 0            # prefix shorter than the sample
    assert ws(8192, (1 << 18) + 1, 2048) == 0  # past the largest fused key count
    assert ws(8192, 131072, 8193) == 0         # k past the finish kernel's list
    assert ws(8192, 131072, 0) == 0
    assert ws(0, 131072, 2048) == 0
    # grows with the queries (per-row flags, thresholds, sample logits, masks)
    assert ws(2048, 131072, 2048) < ws(8192, 131072, 2048)


def _so(lib):
    return lib._lib


def test_invalid_arguments_rejected_before_launch(lib):
    so = _so(lib)
    p = ctypes.c_void_p(16 * 1024)          # aligned, never dereferenced
    odd = ctypes.c_void_p(16 * 1024 + 2)    # not 16-byte aligned
    INV, UNS = lib.MISA_ERR_INVALID_ARG, lib.MISA_ERR_UNSUPPORTED
    # pool: null K, bad d, B out of range, fp8 without scales, no outputs
    assert so.misa_pool_keys(None, None, 0, 128, 128, 64, p, p, None) == INV
    assert so.misa_pool_keys(p, None, 0, 128, 96, 64, p, p, None) == INV
    assert so.misa_pool_keys(p, None, 0, 128, 128, 0, p, p, None) == INV
    assert so.misa_pool_keys(p, None, 1, 128, 128, 64, p, p, None) == INV
    assert so.misa_pool_keys(p, None, 0, 128, 128, 64, None, None, None) == INV
    assert so.misa_pool_keys(odd, None, 0, 128, 128, 64, p, p, None) == INV
    # pool range: m1 past the blocks, m0 > m1, negative m0
    assert so.misa_pool_keys_range(p, None, 0, 256, 128, 64, 0, 5, p, p, None) == INV
    assert so.misa_pool_keys_range(p, None, 0, 256, 128, 64, 3, 2, p, p, None) == INV
    assert so.misa_pool_keys_range(p, None, 0, 256, 128, 64, -1, 2, p, p, None) == INV
    # route: queries past the keys, h > H, H not a power of two
    assert so.misa_route_heads(p, p, p, 10, 95, 100, 64, 128, 64, 8, p, None, None) == INV
    assert so.misa_route_heads(p, p, p, 10, 0, 100, 8, 128, 64, 9, p, None, None) == INV
    assert so.misa_route_heads(p, p, p, 10, 0, 100, 48, 128, 64, 8, p, None, None) == UNS
    assert so.misa_route_heads(p, p, p, 10, 0, 100, 64, 80, 64, 8, p, None, None) == UNS
    # score: ld < n_k, dense with h != H, h not a power of two
    assert so.misa_score_tokens(p, p, p, p, None, 0, 10, 0, 100, 64, 128, 8, p, 99, None) == INV
    assert so.misa_score_tokens(p, p, None, p, None, 0, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert so.misa_score_tokens(p, p, p, p, None, 0, 10, 0, 100, 64, 128, 6, p, 100, None) == UNS
    assert so.misa_score_tokens(odd, p, p, p, None, 0, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert so.misa_score_tokens(p, p, p, p, None, 0, 10, 0, 101, 64, 128, 8, p, 101, None) == INV
    # FP8 queries and keys: d = 32 unsupported, missing scales, misaligned codes,
    # ld < n_k, dense with h != H
    f8 = so.misa_score_tokens_fp8
    assert f8(p, p, p, p, p, p, 10, 0, 100, 64, 32, 8, p, 100, None) == UNS
    assert f8(p, None, p, p, p, p, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert f8(p, p, p, p, p, None, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert f8(odd, p, p, p, p, p, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert f8(p, p, p, p, p, p, 10, 0, 100, 64, 128, 8, p, 99, None) == INV
    assert f8(p, p, p, None, p, p, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert f8(p, p, p, p, p, p, 0, 0, 100, 64, 128, 8, p, 100, None) == 0
    # fused score + top-k: ld not a multiple of 4, k too large, missing workspace
    # where the sizes need one, d unsupported
    assert so.misa_score_topk(p, p, p, p, None, 0, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9001,
                              p, 1 << 30, None) == INV
    assert so.misa_score_topk(p, p, p, p, None, 0, 10, 8000, 9000, 64, 128, 8, 20000, p, p, 9000,
                              p, 1 << 30, None) == INV
    assert so.misa_score_topk(p, p, p, p, None, 0, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000,
                              None, 0, None) == lib.MISA_ERR_WORKSPACE
    assert so.misa_score_topk(p, p, p, p, None, 0, 10, 8000, 9000, 64, 96, 8, 64, p, p, 9000,
                              p, 1 << 30, None) == UNS
    # top-k: k too large, ld too small
    assert so.misa_topk(p, 100, 10, 0, 100, 20000, p, None, 0, None) == INV
    assert so.misa_topk(p, 5, 10, 0, 100, 4, p, None, 0, None) == INV
    # rerank: k > kp, missing workspace
    assert so.misa_rerank(p, p, p, None, 0, p, 16, 4, 0, 100, 64, 128, 32, p, None, p, 1 << 20,
                          None) == INV
    assert so.misa_rerank(p, p, p, None, 0, p, 16, 4, 0, 100, 64, 128, 8, p, None, None, 0,
                          None) == lib.MISA_ERR_WORKSPACE


def test_paged_arguments_rejected_before_launch(lib):
    so = _so(lib)
    p = ctypes.c_void_p(16 * 1024)
    odd = ctypes.c_void_p(16 * 1024 + 2)
    INV, UNS = lib.MISA_ERR_INVALID_ARG, lib.MISA_ERR_UNSUPPORTED
    # (pages, scales, kdtype, block table, page size, pages in the pool)
    good = (p, None, 0, p, 64, 100)
    # pool: no table, page size not 16/32/64/128, empty pool, pool rows past 2^31,
    # FP8 pages without scales, misaligned table
    pool = so.misa_pool_keys_paged
    assert pool(p, None, 0, None, 64, 100, 1000, 128, 64, 0, 16, p, p, None) == INV
    assert pool(p, None, 0, p, 48, 100, 1000, 128, 64, 0, 16, p, p, None) == UNS
    assert pool(p, None, 0, p, 8, 100, 1000, 128, 64, 0, 16, p, p, None) == UNS
    assert pool(p, None, 0, p, 64, 0, 1000, 128, 64, 0, 16, p, p, None) == INV
    assert pool(p, None, 0, p, 128, 1 << 24, 1000, 128, 64, 0, 16, p, p, None) == INV
    assert pool(p, None, 1, p, 64, 100, 1000, 128, 64, 0, 16, p, p, None) == INV
    assert pool(p, None, 0, odd, 64, 100, 1000, 128, 64, 0, 16, p, p, None) == INV
    assert pool(*good, 1000, 128, 64, 3, 3, p, p, None) == 0          # empty range
    # score, fused score + top-k and rerank refuse the same tables
    sc = so.misa_score_tokens_paged
    assert sc(p, p, p, p, None, 0, None, 64, 100, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert sc(p, p, p, p, None, 0, p, 24, 100, 10, 0, 100, 64, 128, 8, p, 100, None) == UNS
    assert sc(p, p, p, *good, 10, 0, 100, 64, 128, 8, p, 99, None) == INV
    assert sc(p, p, p, *good, 0, 0, 100, 64, 128, 8, p, 100, None) == 0
    st = so.misa_score_topk_paged
    assert st(p, p, p, p, None, 0, None, 64, 100, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000, p,
              1 << 30, None) == INV
    assert st(p, p, p, *good, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000, None, 0,
              None) == lib.MISA_ERR_WORKSPACE
    rr = so.misa_rerank_paged
    assert rr(p, p, p, None, 0, None, 64, 100, p, 16, 4, 0, 100, 64, 128, 8, p, p, None, 0,
              None) == INV
    assert rr(p, p, *good, p, 16, 4, 0, 100, 64, 128, 32, p, p, None, 0, None) == INV


def test_scaled_bf16_keys_and_their_decode_rejected_before_launch(lib):
    so = _so(lib)
    p = ctypes.c_void_p(16 * 1024)
    q = ctypes.c_void_p(64 * 1024 * 1024)    # far from p: no overlap
    odd = ctypes.c_void_p(16 * 1024 + 2)
    INV, UNS = lib.MISA_ERR_INVALID_ARG, lib.MISA_ERR_UNSUPPORTED
    SC = lib.MISA_K_BF16_SCALED
    # decode: null or misaligned buffers, overlapping buffers, d unsupported, n_k < 0
    dec = so.misa_keys_e4m3_to_bf16
    assert dec(None, 100, 128, q, None) == INV
    assert dec(p, 100, 128, None, None) == INV
    assert dec(odd, 100, 128, q, None) == INV
    assert dec(p, 100, 128, odd, None) == INV
    assert dec(p, 100, 128, ctypes.c_void_p(16 * 1024 + 4096), None) == INV
    assert dec(p, 100, 96, q, None) == UNS
    assert dec(p, -1, 128, q, None) == INV
    assert dec(p, 0, 128, q, None) == 0
    # scaled bf16 keys: the fused call needs their scales; paged caches and the
    # other calls refuse the key type
    assert so.misa_score_topk(p, p, p, p, None, SC, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000,
                              p, 1 << 30, None) == INV
    assert so.misa_score_topk(p, p, p, p, odd, SC, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000,
                              p, 1 << 30, None) == INV
    assert so.misa_score_topk(p, p, p, p, p, SC, 10, 8000, 9000, 64, 128, 8, 64, p, p, 9000,
                              None, 0, None) == lib.MISA_ERR_WORKSPACE
    assert so.misa_score_topk(p, p, p, p, p, SC, 0, 8000, 9000, 64, 128, 8, 64, p, p, 9000,
                              None, 0, None) == 0
    assert so.misa_score_topk_paged(p, p, p, p, p, SC, p, 64, 100, 10, 8000, 9000, 64, 128, 8, 64,
                                    p, p, 9000, p, 1 << 30, None) == INV
    assert so.misa_score_tokens(p, p, p, p, p, SC, 10, 0, 100, 64, 128, 8, p, 100, None) == INV
    assert so.misa_pool_keys(p, p, SC, 128, 128, 64, p, p, None) == INV
    assert so.misa_rerank(p, p, p, p, SC, p, 16, 4, 0, 100, 64, 128, 8, p, None, p, 1 << 20,
                          None) == INV


def test_empty_work_is_a_no_op(lib):
    so = _so(lib)
    p = ctypes.c_void_p(16 * 1024)
    assert so.misa_topk(p, 100, 0, 0, 100, 4, p, None, 0, None) == 0
    assert so.misa_topk(p, 100, 10, 0, 100, 0, None, None, 0, None) == 0
    assert so.misa_pool_keys_range(p, None, 0, 256, 128, 64, 2, 2, p, p, None) == 0
    assert so.misa_score_tokens(p, p, p, p, None, 0, 0, 0, 100, 64, 128, 8, p, 100, None) == 0


def test_host_pipeline_pieces(lib):
    # run_host's query pieces cover the chunk in order, none empty, with small
    # first and last pieces from three pieces on
    from long_context_sparse_block_b200.indexer import _piece_bounds
    for n, pieces in ((8192, 1), (8192, 2), (8192, 3), (8192, 4), (8192, 8), (600, 4), (5, 4), (1, 4)):
        b = _piece_bounds(n, pieces)
        assert b[0][0] == 0 and b[-1][1] == n
        assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
        assert all(y > x for x, y in b)
        assert len(b) <= pieces
    sizes = [y - x for x, y in _piece_bounds(8192, 4)]
    assert sizes == [1024, 3072, 3072, 1024]


def test_binding_refuses_undersized_buffers(lib):
    # the C ABI sees pointers only: the binding checks the element counts the
    # kernels will touch before anything is launched (CPU tensors: the size
    # check comes first, the device check after it)
    import torch
    n_q, H, d, n_k, h, k = 4, 8, 64, 256, 2, 16
    Q = torch.zeros((n_q, H, d), dtype=torch.int16)
    K = torch.zeros((n_k, d), dtype=torch.int16)
    w = torch.zeros((n_q, H), dtype=torch.float32)
    heads = torch.zeros((n_q, h), dtype=torch.int32)

    def size_error(fn, *a, **kw):
        with pytest.raises(ValueError, match="the call needs"):
            fn(*a, **kw)

    def device_error(fn, *a, **kw):
        with pytest.raises(ValueError, match="must be a CUDA tensor"):
            fn(*a, **kw)

    lg = torch.zeros((n_q, n_k), dtype=torch.float32)
    device_error(lib.misa_score_tokens, Q, w, heads, K, 0, logits=lg, h=h)
    size_error(lib.misa_score_tokens, Q, w[:3], heads, K, 0, logits=lg, h=h)
    size_error(lib.misa_score_tokens, Q, w, heads[:, :1], K, 0, logits=lg, h=h)
    size_error(lib.misa_score_tokens, Q, w, heads, K, 0, logits=lg[:, :n_k - 1], h=h)
    size_error(lib.misa_score_tokens, Q, w, heads, K.to(torch.uint8), 0,
               k_scale=torch.ones(n_k - 1), logits=lg, h=h)
    size_error(lib.misa_score_tokens_fp8, Q.to(torch.uint8), torch.ones((n_q, H - 1)), w, heads,
               K.to(torch.uint8), torch.ones(n_k), 0, logits=lg, h=h)
    size_error(lib.misa_topk, lg[:, :2], 0, n_k, k)                # rows see up to n_q keys
    device_error(lib.misa_topk, lg[:, :n_q], 0, n_k, k)
    size_error(lib.misa_topk, lg, 0, n_k, k, idx=torch.zeros((n_q, k - 1), dtype=torch.int32))
    size_error(lib.misa_route_heads, Q, w, torch.zeros((2, 3, d), dtype=torch.int16), 0, n_k, 64, h)
    size_error(lib.misa_pool_keys, K, 64, kbar=torch.zeros((3, d)))
    size_error(lib.misa_pool_keys_range, K[:100], 64, 0, 2, n_k=200)
    size_error(lib.misa_rerank, Q, w, K, torch.zeros((n_q - 1, 32), dtype=torch.int32), 0, k)
    size_error(lib.misa_score_topk, Q, w, heads, K, 0, k, h=h,
               idx=torch.zeros((n_q, k - 1), dtype=torch.int32), logits=lg)
    # decoded FP8 keys: bf16 codes that come with scales need one per key
    size_error(lib.misa_score_topk, Q, w, heads, K, 0, k, h=h, k_scale=torch.ones(n_k - 1),
               logits=lg)
    size_error(lib.misa_keys_e4m3_to_bf16, K.to(torch.uint8), out=torch.zeros((n_k - 1, d),
                                                                             dtype=torch.int16))
    device_error(lib.misa_keys_e4m3_to_bf16, K.to(torch.uint8),
                 out=torch.zeros((n_k, d), dtype=torch.int16))


def test_binding_checks_pass_for_well_sized_buffers(lib):
    # every wrapper runs all of its size checks on correctly sized (CPU) tensors
    # and stops only at the device check
    import torch
    n_q, H, d, n_k, h, k, kp, B = 4, 8, 64, 256, 2, 16, 32, 64
    M = n_k // B
    Q = torch.zeros((n_q, H, d), dtype=torch.int16)
    K = torch.zeros((n_k, d), dtype=torch.int16)
    K8 = torch.zeros((n_k, d), dtype=torch.uint8)
    w = torch.zeros((n_q, H), dtype=torch.float32)
    heads = torch.zeros((n_q, h), dtype=torch.int32)
    lg = torch.zeros((n_q, n_k), dtype=torch.float32)
    hl = torch.zeros((2, M, d), dtype=torch.int16)
    calls = [
        lambda: lib.misa_pool_keys(K, B, kbar=torch.zeros((M, d)), kbar_hl=hl),
        lambda: lib.misa_pool_keys_range(K, B, 0, M, kbar_hl=hl),
        lambda: lib.misa_route_heads(Q, w, hl, 0, n_k, B, h),
        lambda: lib.misa_score_tokens(Q, w, heads, K, 0, logits=lg, h=h),
        lambda: lib.misa_score_tokens_fp8(Q.to(torch.uint8), torch.ones((n_q, H)), w, heads, K8,
                                          torch.ones(n_k), 0, logits=lg, h=h),
        lambda: lib.misa_topk(lg, 0, n_k, k),
        lambda: lib.misa_score_topk(Q, w, heads, K, 0, k, h=h, logits=lg),
        lambda: lib.misa_rerank(Q, w, K, torch.zeros((n_q, kp), dtype=torch.int32), 0, k),
        lambda: lib.misa_rerank_noalloc(Q, w, K, torch.zeros((n_q, kp), dtype=torch.int32), 0, k),
    ]
    for fn in calls:
        with pytest.raises(ValueError, match="must be a CUDA tensor"):
            fn()
