"""Host-side checks of libps.so that need no GPU: it loads, it exports every function
include/ps.h declares, host validation returns the documented status codes before
touching the device, and the host tile-plan count matches the oracle's brute force."""
import ctypes
import os

import pytest

import oracle as O
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200 import build as BLD


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        BLD.build(quiet=True)
    return B.load()


def test_library_exports_every_header_function(lib):
    names = B.header_functions()
    assert "ps_kv_append_rope" in names and "ps_decode_attn" in names
    assert "ps_masked_prefill_attn" in names and "ps_full_attn_ref" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(B._SIGS), set(names) - set(B._SIGS)


def test_version_string(lib):
    assert "sm_100a" in B.ps_version()


def test_struct_layout_matches_header():
    assert ctypes.sizeof(B.PsParams) == 40
    assert B.PsParams.rope_theta.offset == 24
    assert ctypes.sizeof(B.PsKVCache) == 40


def _params(**kw):
    base = dict(n_q_heads=16, n_kv_heads=2, head_dim=128, l_prefix=100, window=512)
    base.update(kw)
    return B.make_params(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), B.PS_ERR_UNSUPPORTED),
    (dict(n_q_heads=15), B.PS_ERR_INVALID_ARG),
    (dict(window=0), B.PS_ERR_INVALID_ARG),
    (dict(l_prefix=-1), B.PS_ERR_INVALID_ARG),
    (dict(n_kv_heads=0), B.PS_ERR_INVALID_ARG),
    (dict(rope_theta=-1.0), B.PS_ERR_INVALID_ARG),
])
def test_bad_params_rejected_on_host(lib, kw, code):
    p = _params(**kw)
    cache = B.PsKVCache(None, None, None, None, 1)
    rc = lib.ps_decode_attn(ctypes.byref(p), ctypes.byref(cache), None, None, None, None, None, 0,
                            None, None)
    assert rc == code
    assert B.last_error() != ""


def test_group_above_eight_unsupported_for_decode(lib):
    p = _params(n_q_heads=32, n_kv_heads=2)
    cache = B.PsKVCache(16, 16, 16, 16, 1)
    rc = lib.ps_decode_attn(ctypes.byref(p), ctypes.byref(cache), 16, 16, 16, None, None, 0, None,
                            None)
    assert rc == B.PS_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected(lib):
    p = _params()
    cache = B.PsKVCache(16, 16, 16, 16, 2)
    # q misaligned
    rc = lib.ps_decode_attn(ctypes.byref(p), ctypes.byref(cache), 18, 16, 32, None, None, 0, None,
                            None)
    assert rc == B.PS_ERR_INVALID_ARG and "aligned" in B.last_error()
    # ring NULL
    cache2 = B.PsKVCache(16, 16, None, 16, 2)
    rc = lib.ps_decode_attn(ctypes.byref(p), ctypes.byref(cache2), 16, 16, 32, None, None, 0,
                            None, None)
    assert rc == B.PS_ERR_INVALID_ARG
    # pos misaligned (needs 8 bytes)
    rc = lib.ps_kv_append_rope(ctypes.byref(p), ctypes.byref(cache), 16, 16, None, 20, 1, None,
                               None)
    assert rc == B.PS_ERR_INVALID_ARG
    # T < 1
    rc = lib.ps_kv_append_rope(ctypes.byref(p), ctypes.byref(cache), 16, 16, None, 16, 0, None,
                               None)
    assert rc == B.PS_ERR_INVALID_ARG


def test_zero_batch_is_a_no_op(lib):
    p = _params()
    cache = B.PsKVCache(None, None, None, None, 0)
    rc = lib.ps_kv_append_rope(ctypes.byref(p), ctypes.byref(cache), None, None, None, None, 1,
                               None, None)
    assert rc == B.PS_OK


def test_tile_geometry(lib):
    assert B.ps_prefill_tile_geometry() == (128, 128)


@pytest.mark.parametrize("seq,lp,w", [(8192, 256, 2048), (300, 0, 300), (1000, 33, 100),
                                     (129, 5, 1), (4096, 4096, 1), (1, 0, 1), (777, 100, 4096)])
def test_host_plan_count_matches_oracle(lib, seq, lp, w):
    bq, bk = B.ps_prefill_tile_geometry()
    n = B.ps_prefill_plan_tiles(_params(l_prefix=lp, window=w), seq)
    want = O.tile_plan(seq, lp, w, bq, bk).shape[0]
    assert n == want


def test_prefill_plan_rejects_bad_seq(lib):
    with pytest.raises(B.PsError) as e:
        B.ps_prefill_plan_tiles(_params(), 0)
    assert e.value.code == B.PS_ERR_INVALID_ARG


def test_prefill_small_plan_capacity_rejected(lib):
    p = _params(l_prefix=256, window=2048)
    n_tiles = ctypes.c_int64(-1)
    rc = lib.ps_masked_prefill_attn(ctypes.byref(p), 16, 16, 16, 1, 8192, 16, None, 16, 10,
                                    ctypes.byref(n_tiles), None, 0, None, None)
    assert rc == B.PS_ERR_INVALID_ARG
    assert n_tiles.value == O.tile_plan(8192, 256, 2048, 128, 128).shape[0]


def test_workspace_too_small_rejected(lib):
    p = _params(l_prefix=256, window=2048)
    need = B.ps_prefill_workspace_bytes(p, 1, 8192)
    assert need > 0
    rc = lib.ps_masked_prefill_attn(ctypes.byref(p), 16, 16, 16, 1, 8192, 16, None, None, 0, None,
                                    16, need - 1, None, None)
    assert rc == B.PS_ERR_WORKSPACE


def test_prefill_bwd_host_validation(lib):
    """The backward checks pointers, alignment and workspace on the host, before any launch."""
    p = _params(n_q_heads=28, n_kv_heads=4, l_prefix=256, window=2048)
    need = B.ps_prefill_bwd_workspace_bytes(p, 4, 8192)
    # plan + two fp32 statistics per (batch, head, row) + the work counter
    plan = B.ps_prefill_workspace_bytes(p, 4, 8192)
    assert need >= plan + 2 * 4 * 28 * 8192 * 4 + 256
    f = lib.ps_masked_prefill_attn_bwd
    ok = [16] * 5
    args = lambda ptrs, lse=16, grads=(16, 16, 16), ws=256, wsb=need: (  # noqa: E731
        ctypes.byref(p), *ptrs, lse, 4, 8192, *grads, ws, wsb, None, None)
    assert f(*args(ok, lse=None)) == B.PS_ERR_INVALID_ARG          # lse is required
    assert f(*args([16, 16, 16, 16, None])) == B.PS_ERR_INVALID_ARG  # dout NULL
    assert f(*args([16, 16, 8, 16, 16])) == B.PS_ERR_INVALID_ARG     # v misaligned
    assert f(*args(ok, grads=(16, None, 16))) == B.PS_ERR_INVALID_ARG
    one = B.ps_prefill_bwd_workspace_bytes(p, 1, 8192)       # the minimum: one sequence
    assert f(*args(ok, wsb=one - 1)) == B.PS_ERR_WORKSPACE
    assert f(*args(ok, ws=None)) == B.PS_ERR_WORKSPACE
    assert f(*args(ok, ws=272)) == B.PS_ERR_INVALID_ARG              # workspace not 256-aligned
    assert f(ctypes.byref(p), *ok, 16, 4, 0, 16, 16, 16, 256, need, None, None) == \
        B.PS_ERR_INVALID_ARG                                          # seq < 1
    assert f(ctypes.byref(p), *ok, 16, 0, 8192, 16, 16, 16, None, 0, None, None) == B.PS_OK


def test_prefill_bwd_workspace_stops_growing_with_batch():
    """The dS^T store (32 KB per planned tile per head) of one pass stays within 4 GiB: at the
    truncated-backprop shape (28 heads, 8192 tokens, W 2048, 1045 planned tiles per head: 0.96
    GB per sequence) four sequences fit, so batch 32 takes the workspace of batch 4; below
    that the size grows with the batch."""
    p = _params(n_q_heads=28, n_kv_heads=4, l_prefix=256, window=2048)
    ws = [B.ps_prefill_bwd_workspace_bytes(p, n, 8192) for n in (1, 2, 4, 5, 32, 1000)]
    per_seq = 28 * 1045 * 128 * 128 * 2
    assert ws[1] - ws[0] >= per_seq
    assert ws[2] - ws[1] >= 2 * per_seq
    assert ws[2] <= 4 * per_seq + (64 << 20)
    assert ws[3] == ws[4] == ws[5] == ws[2]
    assert ws[2] - 4 * per_seq < (1 << 30) and 4 * per_seq <= 4 << 30 < 5 * per_seq


def test_shared_prefix_host_validation(lib):
    p = _params(l_prefix=2000, window=4096)
    need = B.ps_decode_shared_prefix_workspace_bytes(p, 256, 64)
    # prefix partials alone: >= one fp32 o + lse per (sequence, head)
    assert need >= 256 * 16 * (128 + 1) * 4
    assert B.ps_decode_shared_prefix_workspace_bytes(p, 256, 60) == 0   # not a multiple
    assert B.ps_decode_shared_prefix_workspace_bytes(p, 256, 0) == 0
    assert B.ps_decode_shared_prefix_workspace_bytes(_params(l_prefix=0), 256, 64) == 0
    f = lib.ps_decode_attn_shared_prefix
    cache = B.PsKVCache(16, 16, 16, 16, 256)
    args = lambda gs, ws=256, wsb=need, prm=p: (ctypes.byref(prm), ctypes.byref(cache), gs,  # noqa: E731
                                                 16, 16, 16, None, ws, wsb, None, None)
    assert f(*args(60)) == B.PS_ERR_INVALID_ARG          # batch not a multiple of the group
    assert f(*args(0)) == B.PS_ERR_INVALID_ARG
    assert f(*args(64, prm=_params(l_prefix=0, window=4096))) == B.PS_ERR_INVALID_ARG
    assert f(*args(64, wsb=need - 1)) == B.PS_ERR_WORKSPACE
    assert f(*args(64, ws=272)) == B.PS_ERR_INVALID_ARG  # workspace not 256-aligned
    assert f(*args(64, prm=_params(n_q_heads=32, n_kv_heads=2))) == B.PS_ERR_UNSUPPORTED


def test_reset_pe_host_validation(lib):
    p = _params()
    f = lib.ps_decode_attn_reset_pe
    cache = B.PsKVCache(16, 16, 16, 16, 4)
    assert f(ctypes.byref(p), ctypes.byref(cache), 16, None, 16, None, None, 0, None,
             None) == B.PS_ERR_INVALID_ARG                      # pos NULL
    assert f(ctypes.byref(p), ctypes.byref(cache), 16, 12, 16, None, None, 0, None,
             None) == B.PS_ERR_INVALID_ARG                      # pos not 8-byte aligned
    empty = B.PsKVCache(None, None, None, None, 0)
    assert f(ctypes.byref(p), ctypes.byref(empty), 16, 16, 16, None, None, 0, None,
             None) == B.PS_OK                                   # batch 0: nothing to do


def test_pin_host_validation(lib):
    p = _params(l_prefix=100, window=512)
    cache = B.PsKVCache(16, 16, 16, 16, 4)
    f = lib.ps_kv_pin
    ok = dict(cnt=16, pp=16, t0=16, t1=16, pos=16)
    call = lambda cap, **kw: f(ctypes.byref(p), ctypes.byref(cache), cap,  # noqa: E731
                               *[kw.get(k, v) for k, v in ok.items()], None, None)
    assert call(100) == B.PS_ERR_INVALID_ARG     # capacity must exceed l_prefix
    assert call(200, cnt=None) == B.PS_ERR_INVALID_ARG
    assert call(200, pp=12) == B.PS_ERR_INVALID_ARG   # pin positions not 8-byte aligned
    assert call(200, cnt=18) == B.PS_ERR_INVALID_ARG  # counts not 4-byte aligned
    assert B.ps_decode_pinned_workspace_bytes(p, 64, 99) == 0
    assert B.ps_decode_pinned_workspace_bytes(p, 64, 1124) >= \
        B.ps_decode_pinned_workspace_bytes(p, 64, 100)
    g = lib.ps_decode_attn_pinned
    assert g(ctypes.byref(p), ctypes.byref(cache), 100, 16, 16, 16, 16, 16, None, None, 0,
             None, None) == B.PS_ERR_INVALID_ARG    # capacity must exceed l_prefix
    assert g(ctypes.byref(p), ctypes.byref(cache), 200, None, 16, 16, 16, 16, None, None, 0,
             None, None) == B.PS_ERR_INVALID_ARG


def test_paged_host_validation(lib):
    """Window not a multiple of 64, a table too narrow for L_prefix + W, no blocks, and NULL
    or misaligned pointers are refused before any launch."""
    f, g = lib.ps_kv_append_rope_paged, lib.ps_decode_attn_paged
    p = _params(l_prefix=100, window=512)          # 2 prefix + 8 ring blocks per sequence

    def app(par=p, n_blocks=64, table=16, stride=10, k_pool=16, pos0=16, T=1):
        return f(ctypes.byref(par), k_pool, 16, n_blocks, table, stride, 4, 16, 16, None, pos0,
                 T, None, None)

    def dec(par=p, n_blocks=64, table=16, stride=10, k_pool=16):
        return g(ctypes.byref(par), k_pool, 16, n_blocks, table, stride, 4, 16, 16, 16, None,
                 None, 0, None, None)

    for call in (app, dec):
        assert call(par=_params(l_prefix=100, window=500)) == B.PS_ERR_UNSUPPORTED
        assert call(stride=9) == B.PS_ERR_INVALID_ARG
        assert call(n_blocks=0) == B.PS_ERR_INVALID_ARG
        assert call(table=None) == B.PS_ERR_INVALID_ARG
        assert call(table=18) == B.PS_ERR_INVALID_ARG   # not 4-byte aligned
        assert call(k_pool=None) == B.PS_ERR_INVALID_ARG
    assert app(T=0) == B.PS_ERR_INVALID_ARG
    assert app(pos0=None) == B.PS_ERR_INVALID_ARG
    assert app(pos0=12) == B.PS_ERR_INVALID_ARG         # not 8-byte aligned


def test_wait_timeout_diagnostic_host_validation(lib):
    """The wait diagnostic needs a status word: NULL or misaligned is refused before any
    launch."""
    assert lib.ps_check_wait_timeout(None, None) == B.PS_ERR_INVALID_ARG
    assert lib.ps_check_wait_timeout(2, None) == B.PS_ERR_INVALID_ARG
