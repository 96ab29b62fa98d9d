"""On the device, a stalled in-kernel wait ends with a status, not a hang.

Every wait inside the library's kernels (TMA stages, MMA completion, tile hand-offs) is the
same bounded wait: after about one second it gives up, ORs PS_DEV_TIMEOUT into the call's
status word and the kernel returns.  ps_check_wait_timeout runs that wait on a barrier phase
that nothing completes; the test checks the status bit, that the wait lasted about its
limit, and that the context is still usable afterwards (a decode right after it matches the
float64 oracle).
"""
import math
import time

import pytest
import torch

import oracle as O
import synth
from prefix_sliding_window_b200 import binding as B
from prefix_sliding_window_b200.cache import PrefixSlidingCache
from tests.gpu_util import assert_close, f64
from tests.test_gpu_decode import THETA, _oracle_decode_from_history

pytestmark = pytest.mark.gpu

D = 128


def test_stalled_wait_sets_timeout_and_context_stays_usable(cuda_device):
    dev = cuda_device
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.ps_check_wait_timeout(st)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert st.item() & B.PS_DEV_TIMEOUT
    assert 0.5 < waited < 10.0, waited

    # the same context: one append and one decode, checked against the oracle
    lp, w, p = 20, 64, 150
    params = B.make_params(16, 2, D, lp, w, THETA)
    k_raw = synth.normal_bf16((1, p + 1, 2, D), 71, dev)
    v_raw = synth.normal_bf16((1, p + 1, 2, D), 72, dev)
    q_raw = synth.normal_bf16((1, 16, D), 73, dev)
    cache = PrefixSlidingCache(1, 2, lp, w, D, dev, fill=float("nan"))
    st2 = torch.zeros(1, dtype=torch.int32, device=dev)
    B.ps_kv_append_rope(params, cache.struct, k_raw[:, :p].contiguous(),
                        v_raw[:, :p].contiguous(), None,
                        torch.zeros(1, dtype=torch.int64, device=dev), p, st2)
    pos = torch.full((1,), p, dtype=torch.int64, device=dev)
    q = q_raw.clone()
    out = torch.empty((1, 16, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, 1)), dtype=torch.uint8,
                     device=dev)
    B.ps_decode_step(params, cache.struct, k_raw[:, p].contiguous(), v_raw[:, p].contiguous(),
                     q, pos, out, None, ws, st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    o, _ = _oracle_decode_from_history(O.rope_rotate(f64(q_raw)[0], p, THETA), f64(k_raw)[0],
                                       f64(v_raw)[0], p, lp, w, 1 / math.sqrt(D))
    assert_close(f64(out)[0], o, "decode after a timed-out wait")
