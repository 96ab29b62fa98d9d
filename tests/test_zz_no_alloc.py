"""ps_decode_attn_noalloc: decode for callers that cannot allocate device memory.

Some callers only get their input and output buffers from a host framework (a plugin, a
fixed-memory serving loop) and have no way to allocate the split-K scratch that
ps_decode_attn takes as its workspace argument.  ps_decode_attn_noalloc uses an array built
into the library instead.  This test calls it through the C ABI twice in a row, with
different inputs, and checks that each result is bit-identical to ps_decode_attn on the same
inputs (the same kernel runs on the same data; only where its scratch lives differs), so a
stale scratch from the first call cannot pass for the second.  One sequence of each call is
also checked against the float64 oracle.

The file name sorts last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200.cache import PrefixSlidingCache
from tests.gpu_util import assert_close, f64

pytestmark = pytest.mark.gpu

D = 128


def test_noalloc_decode_matches_workspace_decode_twice(cuda_device):
    dev = cuda_device
    Bn, hq, hkv, lp, w = 4, 16, 2, 100, 4096
    params = B.make_params(hq, hkv, D, lp, w, 1.0e6)
    # this shape splits each sequence across CTAs, so the built-in scratch is really used
    assert B.ps_decode_workspace_bytes(params, Bn) > 0
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    hist = 6000
    k = synth.normal_bf16((Bn, hist, hkv, D), 301, dev)
    v = synth.normal_bf16((Bn, hist, hkv, D), 302, dev)
    B.ps_kv_append_rope(params, cache.struct, k, v, None,
                        torch.zeros(Bn, dtype=torch.int64, device=dev), hist, st)
    ws = torch.empty(B.ps_decode_workspace_bytes(params, Bn), dtype=torch.uint8, device=dev)
    for call, (seed, positions) in enumerate([(303, [5999, 4500, 4195, 77]),
                                              (304, [5999, 5000, 300, 4196])]):
        q = synth.normal_bf16((Bn, hq, D), seed, dev)
        pos = torch.tensor(positions, dtype=torch.int64, device=dev)
        out_ws = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
        lse_ws = torch.empty((Bn, hq), dtype=torch.float32, device=dev)
        B.ps_decode_attn(params, cache.struct, q, pos, out_ws, lse_ws, ws, st)
        out_na = torch.full((Bn, hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        lse_na = torch.full((Bn, hq), float("nan"), dtype=torch.float32, device=dev)
        B.ps_decode_attn_noalloc(params, cache.struct, q, pos, out_na, lse_na, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.equal(out_na, out_ws), f"no-alloc call {call + 1}: output differs"
        assert torch.equal(lse_na, lse_ws), f"no-alloc call {call + 1}: lse differs"
        # sequence 0 (position 5999, the newest appended: its ring holds exactly its window)
        # against the oracle: keys rotated at their positions, q taken as given
        p = positions[0]
        vis = O.visible_positions(p, lp, w)
        k_rot = O.rope_rotate(f64(k[0])[vis], vis[:, None], 1.0e6)
        want, want_lse = O.attend_gqa(f64(q[0]), k_rot, f64(v[0])[vis], 1 / math.sqrt(D))
        assert_close(f64(out_na[0]), want, f"no-alloc call {call + 1} vs oracle")
        assert np.abs(f64(lse_na[0]) - want_lse).max() < 2e-2
