"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, sizes its buffers, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from sparse_rank_approximation_b200 import binding as bd

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "elsaa.h")


def _declared():
    text = open(HEADER).read()
    return set(re.findall(r"ELSAA_API\s+[\w\s\*]+?\b(elsaa_\w+)\s*\(", text))


def test_header_declarations_are_all_exported():
    names = _declared()
    assert names == set(bd.EXPORTED)
    L = bd.lib()
    for n in names:
        assert hasattr(L, n), n


def test_sizes_for_valid_and_invalid_params():
    L = bd.lib()
    p = bd.make_params(1, 32, 16384, 128, rank_r=128, block_size=128, topk=16)
    assert L.elsaa_saved_bytes(ctypes.byref(p)) > 2 * 32 * 16384 * 128 * 2
    assert L.elsaa_workspace_bytes(ctypes.byref(p), 0) > 0
    assert L.elsaa_workspace_bytes(ctypes.byref(p), 1) > L.elsaa_workspace_bytes(ctypes.byref(p), 0)
    bad = [dict(d=96), dict(rank_r=24), dict(rank_r=512), dict(block_size=32), dict(topk=200),
           dict(hash_bits=3), dict(tau=0.0), dict(eps=-1.0),
           dict(N=0), dict(B=0), dict(H=0), dict(N=-5)]      # empty or negative problems are rejected
    for kw in bad:
        args = dict(B=1, H=2, N=1024, d=64, rank_r=64, block_size=64, topk=4)
        hb = kw.pop("hash_bits", 4)
        args.update(kw)
        q = bd.make_params(args.pop("B"), args.pop("H"), args.pop("N"), args.pop("d"), hash_bits=hb, **args)
        assert L.elsaa_saved_bytes(ctypes.byref(q)) == 0, kw
        assert L.elsaa_workspace_bytes(ctypes.byref(q), 1) == 0, kw
    assert L.elsaa_saved_bytes(None) == 0
    # the smallest problem (one row, one partial tile) is valid
    one = bd.make_params(1, 1, 1, 64, rank_r=16, block_size=64, topk=1)
    assert L.elsaa_saved_bytes(ctypes.byref(one)) > 0


def test_block_size_one_is_f32_only():
    L = bd.lib()
    p = bd.make_params(1, 1, 256, 64, dtype=bd.ELSAA_DTYPE_F32, causal=False, rank_r=16, block_size=1, topk=32)
    assert L.elsaa_saved_bytes(ctypes.byref(p)) > 0
    p.dtype = bd.ELSAA_DTYPE_BF16
    assert L.elsaa_saved_bytes(ctypes.byref(p)) == 0
    p.dtype = bd.ELSAA_DTYPE_F32
    p.N = 8192
    assert L.elsaa_saved_bytes(ctypes.byref(p)) == 0


def _fwd(L, p, Q=0x1000, K=0x1000, V=0x1000, W=0x1000, O=0x1000, saved=0x1000, ws=0x1000, wsb=1 << 40):
    return L.elsaa_forward(ctypes.byref(p), Q, K, V, W, None, None, None, O, saved, ws, wsb, None)


def test_argument_errors_return_before_any_launch():
    L = bd.lib()
    p = bd.make_params(1, 2, 1024, 64, rank_r=64, block_size=64, topk=4)
    assert _fwd(L, p, Q=None) == bd.ELSAA_ERR_INVALID_ARG
    assert b"Q is NULL" in L.elsaa_last_error_message()
    assert _fwd(L, p, V=0x1008) == bd.ELSAA_ERR_INVALID_ARG
    assert b"aligned" in L.elsaa_last_error_message()
    assert _fwd(L, p, W=None) == bd.ELSAA_ERR_INVALID_ARG
    assert _fwd(L, p, wsb=16) == bd.ELSAA_ERR_WORKSPACE
    q = bd.make_params(1, 2, 1024, 96, rank_r=64, block_size=64, topk=4)
    assert _fwd(L, q) == bd.ELSAA_ERR_UNSUPPORTED
    q = bd.make_params(1, 2, 1024, 64, rank_r=64, block_size=64, topk=17)
    assert _fwd(L, q) == bd.ELSAA_ERR_INVALID_ARG
    st = L.elsaa_backward(ctypes.byref(p), 0x1000, 0x1000, 0x1000, 0x1000, None, None, None, None, 0x1000,
                          0x1000, 0x1000, 0x1000, 0x1000, 1 << 40, None)
    assert st == bd.ELSAA_ERR_INVALID_ARG and b"dO" in L.elsaa_last_error_message()
    assert L.elsaa_check_device_flags(None, None) == bd.ELSAA_ERR_INVALID_ARG
    st = L.elsaa_fusion_grads(ctypes.byref(p), None, None, None, None, 0x1000, 0x1000, None, None, None)
    assert st == bd.ELSAA_ERR_INVALID_ARG and b"dO" in L.elsaa_last_error_message()
    # nothing requested: returns before any launch
    assert L.elsaa_fusion_grads(ctypes.byref(p), None, None, None, 0x1000, 0x1000, None, None, None, None) == 0


def test_status_strings():
    L = bd.lib()
    for s in range(6):
        assert L.elsaa_status_string(s)
    assert L.elsaa_status_string(99) == b"unknown status"


def test_sortlsh_shape_limits():
    """sortLSH: any length up to 1024 tiles (heads or halves past 16384 rows sort through
    global memory); the causal recursion needs bf16 and a power-of-two block count."""
    L = bd.lib()
    ok = dict(selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=6, topk=1)
    for n, d, t, causal in ((16384, 64, 64, False), (65536, 64, 64, False), (16384, 128, 128, True),
                            (32768, 64, 64, True), (65536, 128, 128, True), (131072, 128, 128, True)):
        p = bd.make_params(1, 2, n, d, block_size=t, rank_r=128 if t == 128 else 16, causal=causal, **ok)
        assert L.elsaa_saved_bytes(ctypes.byref(p)) > 0, (n, d, t, causal)
    bad = [dict(N=64 * 1025, d=64, block_size=64, causal=False),
           dict(N=64 * 6, d=64, block_size=64, causal=True),
           dict(N=128 * 6, d=128, block_size=128, causal=True),
           dict(N=1024, d=128, block_size=128, causal=True, dtype=bd.ELSAA_DTYPE_F32),
           dict(N=128 * 2048, d=128, block_size=128, causal=True)]
    for kw in bad:
        p = bd.make_params(1, 1, kw.pop("N"), kw.pop("d"), rank_r=128 if kw["block_size"] == 128 else 16, **kw, **ok)
        assert L.elsaa_saved_bytes(ctypes.byref(p)) == 0, kw
    p = bd.make_params(1, 1, 1024, 128, block_size=128, rank_r=128, causal=True, selector=bd.ELSAA_SEL_SORTLSH,
                       lsh_bits=17, topk=1)
    assert L.elsaa_saved_bytes(ctypes.byref(p)) == 0


def test_sortlsh_saved_buffer_holds_the_gathered_rows():
    """With sortLSH the forward keeps the rows it gathered (the sorted Q, K, V; with the causal
    recursion every level's future-half queries and past-half keys and values) in the saved
    buffer for the backward, so saved grows by 3 x levels x B H N d x element bytes."""
    L = bd.lib()
    B, H, N, d = 1, 2, 4096, 128
    base = dict(block_size=128, rank_r=128, topk=1)
    n_t = N // 128                             # 32 tiles: the sorted levels are 1 .. log2(32) - 1
    lv = n_t.bit_length() - 2
    for causal, n_levels in ((False, 1), (True, lv)):
        p = bd.make_params(B, H, N, d, causal=causal, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=5, **base)
        q = bd.make_params(B, H, N, d, causal=causal, **base)
        rows = 3 * n_levels * B * H * N * d * 2
        orders = (n_levels if causal else 1) * B * H * 2 * N * 4
        grown = L.elsaa_saved_bytes(ctypes.byref(p)) - L.elsaa_saved_bytes(ctypes.byref(q))
        assert grown >= rows + orders, (causal, grown, rows, orders)
        assert grown <= rows + orders + 4096, (causal, grown, rows, orders)


def test_step_host_argument_errors_return_before_any_copy():
    """The host-buffer step entry checks its arrays, inputs and events before it copies."""
    L = bd.lib()
    p = bd.make_params(1, 2, 1024, 64, rank_r=64, block_size=64, topk=4)
    arr = lambda *xs: (ctypes.c_void_p * len(xs))(*xs)
    hin, hout = arr(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None), arr(0x1000, 0x1000, 0x1000, 0x1000)
    din, dout = arr(0x1000, 0x1000, 0x1000, 0x1000, 0x1000), arr(0x1000, 0x1000, 0x1000, 0x1000)
    ev = arr(0x1000, 0x1000, 0x1000)
    call = lambda *a: L.elsaa_step_host(ctypes.byref(p), *a, 0x1000, 0x1000, 1 << 40, None, None, None, ev)
    assert call(None, hout, din, dout) == bd.ELSAA_ERR_INVALID_ARG
    assert call(hin, hout, din, None) == bd.ELSAA_ERR_INVALID_ARG
    assert call(arr(0x1000, None, 0x1000, 0x1000, 0x1000, None), hout, din, dout) == bd.ELSAA_ERR_INVALID_ARG
    assert b"host K" in L.elsaa_last_error_message()
    assert call(hin, arr(0x1000, 0x1000, None, 0x1000), din, dout) == bd.ELSAA_ERR_INVALID_ARG
    assert b"host dK" in L.elsaa_last_error_message()
    assert call(hin, hout, arr(0x1000, 0x1008, 0x1000, 0x1000, 0x1000), dout) == bd.ELSAA_ERR_INVALID_ARG
    assert b"aligned" in L.elsaa_last_error_message()
    assert L.elsaa_step_host(ctypes.byref(p), hin, hout, din, dout, 0x1000, 0x1000, 1 << 40, None, None, None,
                             arr(0x1000, None, 0x1000)) == bd.ELSAA_ERR_INVALID_ARG
    lsh = bd.make_params(1, 2, 1024, 64, rank_r=64, block_size=64, topk=1, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=4)
    assert L.elsaa_step_host(ctypes.byref(lsh), hin, hout, din, dout, 0x1000, 0x1000, 1 << 40, None, None, None,
                             ev) == bd.ELSAA_ERR_INVALID_ARG
    assert b"planes" in L.elsaa_last_error_message()
