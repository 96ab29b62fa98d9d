"""Thin ctypes binding of libps.so (include/ps.h).

Argument marshalling only: every function takes torch tensors (device memory allocated by
PyTorch), passes their data pointers, sizes and the current CUDA stream to the C entry
point of the same name, and raises PsError on a negative status.  All computation runs in
the library's CUDA kernels; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libps.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "ps.h")

PS_OK = 0
PS_ERR_INVALID_ARG = -1
PS_ERR_UNSUPPORTED = -2
PS_ERR_WORKSPACE = -3
PS_ERR_CUDA = -4

PS_DEV_BAD_POS = 1
PS_DEV_POS_RANGE = 2
PS_DEV_TIMEOUT = 4

PS_TILE_FULL = 1
PS_TILE_PARTIAL = 2


class PsError(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func} failed with status {code}: {msg}")
        self.code = code


class PsParams(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", c_int32),
        ("n_kv_heads", c_int32),
        ("head_dim", c_int32),
        ("l_prefix", c_int32),
        ("window", c_int32),
        ("reserved", c_int32),
        ("rope_theta", c_double),
        ("softmax_scale", c_float),
        ("reserved2", c_int32),
    ]


class PsKVCache(ctypes.Structure):
    _fields_ = [
        ("k_prefix", c_void_p),
        ("v_prefix", c_void_p),
        ("k_ring", c_void_p),
        ("v_ring", c_void_p),
        ("batch", c_int64),
    ]


_lib = None

_SIGS = {
    "ps_kv_append_rope": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    "ps_decode_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64]),
    "ps_decode_attn": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "ps_decode_attn_noalloc": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "ps_full_attn_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64, c_int64]),
    "ps_full_attn_ref": (c_int32, [POINTER(PsParams), c_void_p, c_void_p, c_int64, c_void_p,
                                   c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_size_t,
                                   c_void_p, c_void_p]),
    "ps_prefill_tile_geometry": (c_int32, [POINTER(c_int32), POINTER(c_int32)]),
    "ps_prefill_plan_tiles": (c_int64, [POINTER(PsParams), c_int64]),
    "ps_prefill_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64, c_int64]),
    "ps_masked_prefill_attn": (c_int32, [POINTER(PsParams), c_void_p, c_void_p, c_void_p, c_int64,
                                         c_int64, c_void_p, c_void_p, c_void_p, c_int64,
                                         POINTER(c_int64), c_void_p, c_size_t, c_void_p,
                                         c_void_p]),
    "ps_kv_append_rope_paged": (c_int32, [POINTER(PsParams), c_void_p, c_void_p, c_int64,
                                          c_void_p, c_int32, c_int64, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    "ps_decode_attn_paged": (c_int32, [POINTER(PsParams), c_void_p, c_void_p, c_int64, c_void_p,
                                       c_int32, c_int64, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_size_t, c_void_p, c_void_p]),
    "ps_decode_step": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                 c_void_p, c_void_p]),
    "ps_decode_attn_reset_pe": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                          c_void_p, c_void_p]),
    "ps_kv_pin": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_int32, c_void_p, c_void_p,
                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "ps_decode_pinned_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64, c_int32]),
    "ps_decode_attn_pinned": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_int32,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "ps_decode_shared_prefix_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64,
                                                           c_int64]),
    "ps_decode_attn_shared_prefix": (c_int32, [POINTER(PsParams), POINTER(PsKVCache), c_int64,
                                               c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                               c_size_t, c_void_p, c_void_p]),
    "ps_prefill_bwd_workspace_bytes": (c_size_t, [POINTER(PsParams), c_int64, c_int64]),
    "ps_masked_prefill_attn_bwd": (c_int32, [POINTER(PsParams), c_void_p, c_void_p, c_void_p,
                                             c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                             c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                             c_void_p, c_void_p]),
    "ps_decode_visible_ranges": (c_int32, [POINTER(PsParams), c_void_p, c_int64, c_void_p,
                                           c_void_p]),
    "ps_check_wait_timeout": (c_int32, [c_void_p, c_void_p]),
    "ps_last_error": (c_char_p, []),
    "ps_version": (c_char_p, []),
}


def header_functions() -> list:
    """Names of the functions include/ps.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|size_t|const char\*)\s+(ps_\w+)\s*\(",
                                 text, flags=re.M)))


def load():
    """Load libps.so (raises loudly if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m prefix_sliding_window_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def last_error() -> str:
    return load().ps_last_error().decode()


def _check(rc: int, func: str):
    if rc != PS_OK:
        raise PsError(rc, func, last_error())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_params(n_q_heads, n_kv_heads, head_dim=128, l_prefix=0, window=1, rope_theta=1.0e6,
                softmax_scale=0.0) -> PsParams:
    return PsParams(int(n_q_heads), int(n_kv_heads), int(head_dim), int(l_prefix), int(window), 0,
                    float(rope_theta), float(softmax_scale), 0)


def make_cache(k_prefix, v_prefix, k_ring, v_ring, batch: int) -> PsKVCache:
    return PsKVCache(_ptr(k_prefix), _ptr(v_prefix), _ptr(k_ring), _ptr(v_ring), int(batch))


# ---------------------------------------------------------------- entry points
def ps_kv_append_rope(params: PsParams, cache: PsKVCache, k_new, v_new, q_inout, pos0, T: int,
                      dev_status=None, stream=None) -> None:
    rc = load().ps_kv_append_rope(ctypes.byref(params), ctypes.byref(cache), _ptr(k_new),
                                  _ptr(v_new), _ptr(q_inout), _ptr(pos0), int(T),
                                  _ptr(dev_status), _stream(stream))
    _check(rc, "ps_kv_append_rope")


def ps_decode_workspace_bytes(params: PsParams, batch: int) -> int:
    return int(load().ps_decode_workspace_bytes(ctypes.byref(params), int(batch)))


def ps_decode_attn(params: PsParams, cache: PsKVCache, q, pos, out, lse=None, workspace=None,
                   dev_status=None, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_attn(ctypes.byref(params), ctypes.byref(cache), _ptr(q), _ptr(pos),
                               _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _ptr(dev_status),
                               _stream(stream))
    _check(rc, "ps_decode_attn")


def ps_kv_append_rope_paged(params: PsParams, k_pool, v_pool, block_table, batch: int, k_new,
                            v_new, q_inout, pos0, T: int, dev_status=None, stream=None) -> None:
    """Append into a paged store: pools [n_blocks, Hkv, 64, D], block_table [batch, stride]."""
    rc = load().ps_kv_append_rope_paged(ctypes.byref(params), _ptr(k_pool), _ptr(v_pool),
                                        int(k_pool.shape[0]), _ptr(block_table),
                                        int(block_table.shape[1]), int(batch), _ptr(k_new),
                                        _ptr(v_new), _ptr(q_inout), _ptr(pos0), int(T),
                                        _ptr(dev_status), _stream(stream))
    _check(rc, "ps_kv_append_rope_paged")


def ps_decode_attn_paged(params: PsParams, k_pool, v_pool, block_table, batch: int, q, pos, out,
                         lse=None, workspace=None, dev_status=None, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_attn_paged(ctypes.byref(params), _ptr(k_pool), _ptr(v_pool),
                                     int(k_pool.shape[0]), _ptr(block_table),
                                     int(block_table.shape[1]), int(batch), _ptr(q), _ptr(pos),
                                     _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "ps_decode_attn_paged")


def ps_decode_step(params: PsParams, cache: PsKVCache, k_new, v_new, q_inout, pos, out,
                   lse=None, workspace=None, dev_status=None, stream=None) -> None:
    """Append one token per sequence at pos (q rotated in place), then decode at pos."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_step(ctypes.byref(params), ctypes.byref(cache), _ptr(k_new),
                               _ptr(v_new), _ptr(q_inout), _ptr(pos), _ptr(out), _ptr(lse),
                               _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check(rc, "ps_decode_step")


def ps_decode_attn_reset_pe(params: PsParams, cache: PsKVCache, q, pos, out, lse=None,
                            workspace=None, dev_status=None, stream=None) -> None:
    """Decode under Reset PE from a Continue-PE cache (prefix rows see the query at its
    Reset-PE id)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_attn_reset_pe(ctypes.byref(params), ctypes.byref(cache), _ptr(q),
                                        _ptr(pos), _ptr(out), _ptr(lse), _ptr(workspace),
                                        ws_bytes, _ptr(dev_status), _stream(stream))
    _check(rc, "ps_decode_attn_reset_pe")


def ps_kv_pin(params: PsParams, cache: PsKVCache, prefix_capacity: int, pin_count, pin_pos, t0,
              t1, pos, dev_status=None, stream=None) -> None:
    """Promote tokens [t0[b], t1[b]) (still in the window) into the pinned prefix."""
    rc = load().ps_kv_pin(ctypes.byref(params), ctypes.byref(cache), int(prefix_capacity),
                          _ptr(pin_count), _ptr(pin_pos), _ptr(t0), _ptr(t1), _ptr(pos),
                          _ptr(dev_status), _stream(stream))
    _check(rc, "ps_kv_pin")


def ps_decode_pinned_workspace_bytes(params: PsParams, batch: int, prefix_capacity: int) -> int:
    return int(load().ps_decode_pinned_workspace_bytes(ctypes.byref(params), int(batch),
                                                       int(prefix_capacity)))


def ps_decode_attn_pinned(params: PsParams, cache: PsKVCache, prefix_capacity: int, pin_count,
                          pin_pos, q, pos, out, lse=None, workspace=None, dev_status=None,
                          stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_attn_pinned(ctypes.byref(params), ctypes.byref(cache),
                                      int(prefix_capacity), _ptr(pin_count), _ptr(pin_pos),
                                      _ptr(q), _ptr(pos), _ptr(out), _ptr(lse), _ptr(workspace),
                                      ws_bytes, _ptr(dev_status), _stream(stream))
    _check(rc, "ps_decode_attn_pinned")


def ps_decode_attn_noalloc(params: PsParams, cache: PsKVCache, q, pos, out, lse=None,
                           dev_status=None, stream=None) -> None:
    """ps_decode_attn whose split-K scratch is the library's built-in device array."""
    rc = load().ps_decode_attn_noalloc(ctypes.byref(params), ctypes.byref(cache), _ptr(q),
                                       _ptr(pos), _ptr(out), _ptr(lse), _ptr(dev_status),
                                       _stream(stream))
    _check(rc, "ps_decode_attn_noalloc")


def ps_decode_shared_prefix_workspace_bytes(params: PsParams, batch: int, group_size: int) -> int:
    return int(load().ps_decode_shared_prefix_workspace_bytes(ctypes.byref(params), int(batch),
                                                              int(group_size)))


def ps_decode_attn_shared_prefix(params: PsParams, cache: PsKVCache, group_size: int, q, pos,
                                 out, lse=None, workspace=None, dev_status=None,
                                 stream=None) -> None:
    """Decode where sequences [j*group_size, (j+1)*group_size) share prefix j of
    cache.k_prefix / v_prefix ([batch / group_size, Hkv, l_prefix, D])."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_decode_attn_shared_prefix(ctypes.byref(params), ctypes.byref(cache),
                                             int(group_size), _ptr(q), _ptr(pos), _ptr(out),
                                             _ptr(lse), _ptr(workspace), ws_bytes,
                                             _ptr(dev_status), _stream(stream))
    _check(rc, "ps_decode_attn_shared_prefix")


def ps_full_attn_workspace_bytes(params: PsParams, batch: int, lmax: int) -> int:
    return int(load().ps_full_attn_workspace_bytes(ctypes.byref(params), int(batch), int(lmax)))


def ps_full_attn_ref(params: PsParams, k_full, v_full, lmax: int, q, pos, batch: int, out,
                     lse=None, workspace=None, dev_status=None, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_full_attn_ref(ctypes.byref(params), _ptr(k_full), _ptr(v_full), int(lmax),
                                 _ptr(q), _ptr(pos), int(batch), _ptr(out), _ptr(lse),
                                 _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check(rc, "ps_full_attn_ref")


def ps_prefill_tile_geometry():
    bq, bk = c_int32(0), c_int32(0)
    _check(load().ps_prefill_tile_geometry(ctypes.byref(bq), ctypes.byref(bk)),
           "ps_prefill_tile_geometry")
    return bq.value, bk.value


def ps_prefill_plan_tiles(params: PsParams, seq: int) -> int:
    n = int(load().ps_prefill_plan_tiles(ctypes.byref(params), int(seq)))
    if n < 0:
        raise PsError(n, "ps_prefill_plan_tiles", last_error())
    return n


def ps_prefill_workspace_bytes(params: PsParams, batch: int, seq: int) -> int:
    return int(load().ps_prefill_workspace_bytes(ctypes.byref(params), int(batch), int(seq)))


def ps_masked_prefill_attn(params: PsParams, q, k, v, batch: int, seq: int, out, lse=None,
                           tile_plan=None, workspace=None, dev_status=None, stream=None) -> int:
    """Returns the number of plan rows (tiles per (batch, head))."""
    n_tiles = c_int64(-1)
    cap = 0 if tile_plan is None else tile_plan.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_masked_prefill_attn(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), int(batch),
                                       int(seq), _ptr(out), _ptr(lse), _ptr(tile_plan), int(cap),
                                       ctypes.byref(n_tiles), _ptr(workspace), ws_bytes,
                                       _ptr(dev_status), _stream(stream))
    _check(rc, "ps_masked_prefill_attn")
    return n_tiles.value


def ps_prefill_bwd_workspace_bytes(params: PsParams, batch: int, seq: int) -> int:
    return int(load().ps_prefill_bwd_workspace_bytes(ctypes.byref(params), int(batch), int(seq)))


def ps_masked_prefill_attn_bwd(params: PsParams, q, k, v, out, dout, lse, batch: int, seq: int,
                               dq, dk, dv, workspace=None, dev_status=None, stream=None) -> None:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().ps_masked_prefill_attn_bwd(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(out), _ptr(dout), _ptr(lse), int(batch), int(seq),
                                           _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes,
                                           _ptr(dev_status), _stream(stream))
    _check(rc, "ps_masked_prefill_attn_bwd")


def ps_decode_visible_ranges(params: PsParams, pos, batch: int, ranges_out, stream=None) -> None:
    rc = load().ps_decode_visible_ranges(ctypes.byref(params), _ptr(pos), int(batch),
                                         _ptr(ranges_out), _stream(stream))
    _check(rc, "ps_decode_visible_ranges")


def ps_check_wait_timeout(dev_status, stream=None) -> None:
    rc = load().ps_check_wait_timeout(_ptr(dev_status), _stream(stream))
    _check(rc, "ps_check_wait_timeout")


def ps_version() -> str:
    return load().ps_version().decode()
