#!/usr/bin/env python
"""Benchmark of the Prefix Sliding attention hot path on B200.

Default workload: steady-state batched decode on one layer (batch 64, 16 query / 2 KV
heads, head_dim 128, bf16, L_prefix = 100, W = 4096, positions drawn in [8192, 131072],
KV prefilled with RoPE at every absolute position).  One step = one decode step of the
whole batch through ps_decode_step: the new token's append (Continue-PE RoPE of k and q,
ring write), then split-K decode + merge.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Under torchrun every rank decodes its own batch (weak scaling, no data-path collective);
the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

D = 128
METRIC = "decode attn tokens/s and HBM GB/s (% roofline) vs position; prefill TFLOP/s"
UNIT = "tok/s"
WORKLOAD = "decode_b64_w4096"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a background thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
            self.ok = True
        except Exception:
            self.ok = False
        self.period = period_s
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self, t0=None, t1=None):
        if not self.ok or not self.samples:
            return None
        inside = [s for s in self.samples if t0 is None or (t0 <= s[0] <= t1)]
        window = "timed"
        if len(inside) < 3:
            inside = self.samples
            window = "warmup+timed"
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [name for bit, name in self.REASONS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(inside), "window": window}


# ------------------------------------------------------------- distributed
def _recorded_traffic(entry: str = "step"):
    """DRAM bytes (read + write) per launch of `entry` from the last ncu capture, or None when
    the sources of its kernels changed since (their sha256 no longer matches the record)."""
    import hashlib
    pkg = os.path.join(ROOT, "prefix_sliding_window_b200")
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)[entry]
        h = hashlib.sha256()
        for name in rec["sources"]:
            with open(os.path.join(pkg, "csrc", name), "rb") as f:
                h.update(f.read())
    except (OSError, KeyError, ValueError):
        return None
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    return int(rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"])


def _dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Step time of the job: the slowest rank's."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Work of the whole job: every rank decodes its own batch (weak scaling)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(index: int, rank: int, k: int) -> int:
    """Seed of input stream k of workload `index` on `rank`: every rank draws its own
    sequences (the batch is sharded, not replicated)."""
    return synth.seed_for(index, 10 * rank + k)


SOAK_S = 0.3


def decode_config(wl: synth.Workload, world: int) -> dict:
    """The workload description both arms report (same keys and values)."""
    return {"workload": WORKLOAD, "batch_per_gpu": wl.batch, "global_batch": wl.batch * world,
            "n_q_heads": wl.n_q_heads, "n_kv_heads": wl.n_kv_heads, "head_dim": D,
            "l_prefix": wl.l_prefix, "window": wl.window,
            "positions": f"U[{wl.pos_lo},{wl.pos_hi}]", "layers": 1,
            "step": "one decode step of every sequence: append with Continue-PE RoPE + decode",
            "l2": "inputs larger than L2 (275 MB of K/V read per step vs 126 MB L2)",
            "parallelism": f"dp{world} (independent sequences, no collective)"}


# ------------------------------------------------------------- decode setup
class DecodeWorkload:
    """Prefix Sliding decode workload resident in HBM (one layer)."""

    def __init__(self, wl: synth.Workload, dev, rank: int, max_steps: int):
        from prefix_sliding_window_b200 import binding as B
        from prefix_sliding_window_b200.cache import PrefixSlidingCache
        self.B = B
        self.wl = wl
        self.dev = dev
        Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
        self.params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
        s = lambda k: rank_seed(wl.index, rank, k)  # noqa: E731
        self.pos_start = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, s(0), dev)
        self.cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        self.status = st
        # prefix [0, lp) and window history [p - W + 1, p - 1], RoPE at absolute positions
        k_pre = synth.normal_bf16((Bn, lp, hkv, D), s(1), dev)
        v_pre = synth.normal_bf16((Bn, lp, hkv, D), s(2), dev)
        B.ps_kv_append_rope(self.params, self.cache.struct, k_pre, v_pre, None,
                            torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
        del k_pre, v_pre
        chunk = 1024
        for c0 in range(0, w - 1, chunk):
            T = min(chunk, w - 1 - c0)
            k = synth.normal_bf16((Bn, T, hkv, D), s(3) + c0, dev)
            v = synth.normal_bf16((Bn, T, hkv, D), s(4) + c0, dev)
            B.ps_kv_append_rope(self.params, self.cache.struct, k, v, None,
                                self.pos_start - (w - 1) + c0, T, st)
        # per-step new tokens (distinct buffers per step, so no step reuses another's input)
        n = max_steps
        self.k_new = synth.normal_bf16((n, Bn, 1, hkv, D), s(5), dev)
        self.v_new = synth.normal_bf16((n, Bn, 1, hkv, D), s(6), dev)
        self.q_raw = synth.normal_bf16((n, Bn, hq, D), s(7), dev)
        self.q = self.q_raw.clone()
        self.pos = torch.stack([self.pos_start + i for i in range(n)])
        self.out = torch.empty((n, Bn, hq, D), dtype=torch.bfloat16, device=dev)
        nb = B.ps_decode_workspace_bytes(self.params, Bn)
        self.ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
        self.splits_used = nb > 0
        torch.cuda.synchronize()

    def kernels_per_step(self) -> int:
        """ps_decode_step launches the append, the decode and, when the batch is split across
        CTAs (stream-K), the merge."""
        return 2 + (1 if self.splits_used else 0)

    def append(self, i):
        B = self.B
        B.ps_kv_append_rope(self.params, self.cache.struct, self.k_new[i], self.v_new[i],
                            self.q[i], self.pos[i], 1, self.status)

    def decode(self, i):
        self.B.ps_decode_attn(self.params, self.cache.struct, self.q[i], self.pos[i], self.out[i],
                              None, self.ws, self.status)

    def step(self, i):
        """One decode step through the single-call API (append at pos, then decode)."""
        self.B.ps_decode_step(self.params, self.cache.struct, self.k_new[i], self.v_new[i],
                              self.q[i], self.pos[i], self.out[i], None, self.ws, self.status)

    def algorithmic_bytes_per_append(self) -> int:
        """One new token per sequence: k_new, v_new read and written into the cache
        (2 x Hkv x D x 2 B each way), q read and written back rotated (2 x Hq x D x 2 B),
        pos (8 B)."""
        wl = self.wl
        return wl.batch * (2 * 2 * wl.n_kv_heads * D * 2 + 2 * wl.n_q_heads * D * 2 + 8)

    def algorithmic_bytes_per_decode(self) -> int:
        """K+V of every visible key plus q and out: 1024 B per visible token per sequence
        (2 KV heads x 128 x 2 B x 2) + 2 x Hq x D x 2 B."""
        wl = self.wl
        n = self.pos_start + 1
        vis = torch.clamp(n, max=wl.l_prefix + wl.window)
        kv = int(vis.sum().item()) * 2 * wl.n_kv_heads * D * 2
        return kv + wl.batch * 2 * wl.n_q_heads * D * 2


def run_decode(args, world, rank, dev):
    wl = synth.WORKLOADS[WORKLOAD]
    K, W = args.steps, args.warmup
    work = DecodeWorkload(wl, dev, rank, K + W)
    stream = torch.cuda.current_stream()

    def step(i):
        work.step(i)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    # per-launch duration of ps_decode_attn (decode + merge), CUDA events on the stream
    work.q.copy_(work.q_raw)
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    for j in range(K):
        i = W + j
        work.append(i)
        ev_dec[j][0].record(stream)
        work.decode(i)
        ev_dec[j][1].record(stream)
    torch.cuda.synchronize()
    work.q.copy_(work.q_raw)
    graph = None
    if not args.no_graph:
        # the K timed steps as one CUDA graph (kernel launches only; programmatic
        # dependencies between append, decode and merge are kept as graph edges)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for j in range(K):
                step(W + j)
        torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    # soak: the same K steps replayed, untimed, for at least SOAK_S seconds right before the
    # timed region, so the clock sampler sees this load (the timed region itself is far
    # shorter than the sampling period)
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_a.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for j in range(K):
            step(W + j)
    e_b.record(stream)
    torch.cuda.synchronize()
    once_s = max(e_a.elapsed_time(e_b) / 1e3, 1e-6)
    reps = int(math.ceil(SOAK_S / once_s))
    t_soak0 = time.perf_counter()
    for _ in range(reps):
        if graph is not None:
            graph.replay()
        else:
            for j in range(K):
                step(W + j)
    # ps_decode_step rotates q in place, so every replay above rotated the same q again:
    # the timed steps start from the unrotated q (the work is the same either way; the last
    # output is then the one the end-to-end run below must reproduce)
    work.q.copy_(work.q_raw)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    t_host0 = time.perf_counter()
    ev0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for j in range(K):
            step(W + j)
    ev1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    _barrier(world)
    if sampler:
        sampler.stop()
    ms_local = ev0.elapsed_time(ev1)
    ms = _max_over_ranks(ms_local, world)
    dec_ms = [a.elapsed_time(b) for a, b in ev_dec]
    assert work.status.item() == 0, f"device status {work.status.item()}"
    tokens = _sum_over_ranks(float(wl.batch * K), world)
    value = tokens / (ms / 1e3)

    peaks = _peaks()
    # the dominant unit: one ps_decode_step (append + decode + merge), timed over the timed
    # region itself (graph or eager), so its duration includes everything a step launches
    alg_dec = work.algorithmic_bytes_per_decode()
    alg = alg_dec + work.algorithmic_bytes_per_append()
    step_s = ms / K / 1e3
    achieved = alg / step_s / 1e9
    dec_med_s = statistics.median(dec_ms) / 1e3
    attn = alg_dec / dec_med_s / 1e9
    roof = {"bound": "hbm",
            "kernel": "ps_decode_step (append_rope_kernel + decode_kernel + merge_kernel)",
            "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": args.traffic if args.traffic is not None else _recorded_traffic("step"),
            "peak_source": peaks["source"], "algorithmic_bytes_per_launch": alg,
            "duration_us": round(step_s * 1e6, 2), "duration_source": "timed region / steps",
            "frac_of_8tbs_spec": round(achieved / 8000.0, 4),
            "attn_call": {"what": "ps_decode_attn (decode_kernel + merge_kernel), each call "
                                  "bracketed alone by CUDA events after that step's append; "
                                  "achieved from the median call",
                          "algorithmic_bytes": alg_dec, "achieved": round(attn, 1),
                          "frac": round(attn / peaks["hbm_gbs"], 4),
                          "us_median": round(statistics.median(dec_ms) * 1e3, 2),
                          "us_p10": round(float(np.percentile(dec_ms, 10)) * 1e3, 2),
                          "us_p90": round(float(np.percentile(dec_ms, 90)) * 1e3, 2),
                          "traffic": _recorded_traffic("attn_call")}}
    e2e = run_decode_e2e(work, K, W, world, use_graph=not args.no_graph)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": decode_config(wl, world),
        "launch": "CUDA graph of the timed steps" if graph is not None else "eager",
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": work.kernels_per_step() * K,
    }
    if sampler:
        line["clocks"] = sampler.summary(t_soak0, t_host1)
        if line["clocks"]:
            line["clocks"]["window"] = (f"{reps} untimed replays of the timed steps "
                                        f"({reps * once_s:.2f} s) + the timed region")
    return line, work


class MappedHostBuffer:
    """Pinned host memory mapped into the device address space (cudaHostAlloc with
    cudaHostAllocMapped); device_ptr() is the address kernels write through, host() a uint8
    CPU tensor over the same bytes."""

    def __init__(self, nbytes: int):
        from cuda.bindings import runtime as cudart
        self._rt = cudart
        err, self.hp = cudart.cudaHostAlloc(nbytes, cudart.cudaHostAllocMapped)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc: {err}")
        err, self.dp = cudart.cudaHostGetDevicePointer(self.hp, 0)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostGetDevicePointer: {err}")
        self.nbytes = nbytes

    def device_view(self, offset: int):
        ptr = self.dp + offset

        class _P:
            def data_ptr(self):
                return ptr
        return _P()

    def host(self) -> torch.Tensor:
        import ctypes
        arr = (ctypes.c_uint8 * self.nbytes).from_address(self.hp)
        return torch.frombuffer(arr, dtype=torch.uint8)

    def __del__(self):
        try:
            self._rt.cudaFreeHost(self.hp)
        except Exception:
            pass


def run_decode_e2e(work: DecodeWorkload, K: int, W: int, world: int, use_graph: bool = True):
    """Same metric through the C ABI with host buffers: every step copies its inputs (q,
    k_new, v_new, pos: packed in one pinned host buffer, so one DMA) host->device, and
    ps_decode_step writes that step's output straight into pinned host memory mapped into the
    device's address space (the merge kernel's stores cross PCIe; no second copy).  In stream
    order: step i+1's inputs are copied after step i's output has been written, as a decode
    loop whose next inputs depend on it would.  The same steps with a device->host DMA of the
    output instead are reported beside it (dma_out)."""
    B = work.B
    dev = work.dev
    n = K + W
    parts = [("k", work.k_new[0]), ("v", work.v_new[0]), ("q", work.q[0]), ("pos", work.pos[0])]
    offs, size = {}, 0
    for name, t in parts:
        offs[name] = size
        size += (t.numel() * t.element_size() + 255) // 256 * 256
    h_in = torch.empty((n, size), dtype=torch.uint8).pin_memory()
    for i in range(n):
        for name, src in (("k", work.k_new[i]), ("v", work.v_new[i]), ("q", work.q_raw[i]),
                          ("pos", work.pos[i])):
            nb = src.numel() * src.element_size()
            h_in[i, offs[name]:offs[name] + nb].copy_(src.cpu().contiguous().view(-1).view(torch.uint8))
    d_in = torch.empty((size,), dtype=torch.uint8, device=dev)

    def view(name, like):
        nb = like.numel() * like.element_size()
        return d_in[offs[name]:offs[name] + nb].view(like.dtype).view(like.shape)
    d_k, d_v = view("k", work.k_new[0]), view("v", work.v_new[0])
    d_q, d_pos = view("q", work.q[0]), view("pos", work.pos[0])
    out_bytes = work.out[0].numel() * 2
    h_map = MappedHostBuffer(n * out_bytes)
    h_out = torch.empty((n,) + tuple(work.out.shape[1:]), dtype=torch.bfloat16).pin_memory()
    d_out = torch.empty_like(work.out[0])
    stream = torch.cuda.current_stream()

    def step_mapped(i):
        d_in.copy_(h_in[i], non_blocking=True)
        B.ps_decode_step(work.params, work.cache.struct, d_k, d_v, d_q, d_pos,
                         h_map.device_view(i * out_bytes), None, work.ws, work.status)

    def step_dma(i):
        d_in.copy_(h_in[i], non_blocking=True)
        B.ps_decode_step(work.params, work.cache.struct, d_k, d_v, d_q, d_pos, d_out, None,
                         work.ws, work.status)
        h_out[i].copy_(d_out, non_blocking=True)

    def timed(step):
        for i in range(W):
            step(i)
        torch.cuda.synchronize()
        graph = None
        if use_graph:
            # the K steps (copy in, step, output to the host, in stream order) as one graph
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for j in range(K):
                    step(W + j)
            torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _barrier(world)
        ev0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for j in range(K):
                step(W + j)
        ev1.record(stream)
        torch.cuda.synchronize()
        assert work.status.item() == 0, f"device status {work.status.item()}"
        del graph
        return _max_over_ranks(ev0.elapsed_time(ev1), world)

    ms = timed(step_mapped)
    # the timed steps really moved the data: the last output on the host equals the device
    # run's output of the same step
    last = h_map.host()[(n - 1) * out_bytes:n * out_bytes].view(torch.bfloat16)
    assert torch.equal(last.view(work.out[0].shape), work.out[n - 1].cpu())
    ms_dma = timed(step_dma)
    assert torch.equal(h_out[n - 1], work.out[n - 1].cpu())
    # where an end-to-end step's time goes: the DMA variant launched eagerly, each part
    # bracketed by CUDA events on the stream (copy in, ps_decode_step, copy out)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for j in range(K):
        i = W + j
        e = evs[j]
        e[0].record(stream)
        d_in.copy_(h_in[i], non_blocking=True)
        e[1].record(stream)
        B.ps_decode_step(work.params, work.cache.struct, d_k, d_v, d_q, d_pos, d_out, None,
                         work.ws, work.status)
        e[2].record(stream)
        h_out[i].copy_(d_out, non_blocking=True)
        e[3].record(stream)
    torch.cuda.synchronize()
    med = lambda a, b: round(statistics.median([e[a].elapsed_time(e[b]) for e in evs]) * 1e3, 2)  # noqa: E731
    split = {"h2d_us": med(0, 1), "step_us": med(1, 2), "d2h_us": med(2, 3),
             "total_us": med(0, 3), "how": "DMA variant, eager, CUDA events around each part, "
             "medians"}
    tokens = _sum_over_ranks(float(work.wl.batch * K), world)
    bi = (d_k.numel() + d_v.numel() + d_q.numel()) * 2 + d_pos.numel() * 8
    bo = d_out.numel() * 2
    del h_map
    return {"value": round(tokens / (ms / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "h2d_copies_per_step": 1,
            "d2h": "out written by ps_decode_step into mapped pinned host memory",
            "us_per_step": round(ms / K * 1e3, 2),
            "dma_out": {"value": round(tokens / (ms_dma / 1e3), 1),
                        "us_per_step": round(ms_dma / K * 1e3, 2),
                        "d2h": "one cudaMemcpyAsync of out per step"},
            "split": split,
            "launch": "CUDA graph of the timed steps" if use_graph else "eager"}


# ------------------------------------------------------------- prefill leg
def prefill_visible_pairs(S: int, lp: int, w: int) -> int:
    """Visible (row, key) pairs of one (batch, head): sum over rows of min(i + 1, Lp + W)."""
    cap = lp + w
    n1 = min(S, cap)
    return n1 * (n1 + 1) // 2 + (S - n1) * cap


def run_prefill(dev, steps: int = 10, warmup: int = 3, workload: str = "prefill_b4_s8192_w2048"):
    """Masked prefill / truncated-backprop context forward (default: batch 4, 8192 tokens,
    28/4/128, L_prefix 256, W 2048) and its backward.  TFLOP/s counts unmasked FLOPs only
    (4 * D per visible pair per query head)."""
    from prefix_sliding_window_b200 import binding as B
    wl = synth.WORKLOADS[workload]
    Bn, S, hq, hkv, lp, w = wl.batch, wl.seq, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    q = synth.normal_bf16((Bn, S, hq, D), synth.seed_for(wl.index, 1), dev)
    k = synth.normal_bf16((Bn, S, hkv, D), synth.seed_for(wl.index, 2), dev)
    v = synth.normal_bf16((Bn, S, hkv, D), synth.seed_for(wl.index, 3), dev)
    out = torch.empty_like(q)
    lse = torch.empty((Bn, hq, S), dtype=torch.float32, device=dev)
    n = B.ps_prefill_plan_tiles(params, S)
    plan = torch.empty((n, 3), dtype=torch.int32, device=dev)
    ws = torch.empty(B.ps_prefill_workspace_bytes(params, Bn, S), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        B.ps_masked_prefill_attn(params, q, k, v, Bn, S, out, lse, plan, ws, st)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        B.ps_masked_prefill_attn(params, q, k, v, Bn, S, out, lse, None, ws, st)
        b.record(stream)
    torch.cuda.synchronize()
    assert st.item() == 0, f"device status {st.item()}"
    ms = [a.elapsed_time(b) for a, b in evs]
    flags = plan[:, 2].cpu()
    n_full = int((flags == B.PS_TILE_FULL).sum())
    n_part = int((flags == B.PS_TILE_PARTIAL).sum())
    nq = -(-S // 128)
    pairs = prefill_visible_pairs(S, lp, w)
    flops = 4 * D * pairs * hq * Bn
    computed = 4 * D * 128 * 128 * n * hq * Bn
    med = statistics.median(ms) / 1e3
    tflops = flops / med / 1e12
    peaks = _peaks()
    return {"workload": wl.name, "ms": round(med * 1e3, 4),
            "ms_p10": round(float(np.percentile(ms, 10)), 4),
            "ms_p90": round(float(np.percentile(ms, 90)), 4),
            "tflops_unmasked": round(tflops, 1), "unit": "TFLOP/s",
            "peak": peaks["bf16_tflops"], "frac": round(tflops / peaks["bf16_tflops"], 4),
            "frac_of_2250_spec": round(tflops / 2250.0, 4),
            "tflops_computed_tiles": round(computed / med / 1e12, 1),
            "unmasked_gflop": round(flops / 1e9, 1), "computed_gflop": round(computed / 1e9, 1),
            "tiles_per_head": {"full": n_full, "partial": n_part, "skip": nq * nq - n},
            "launches_per_call": 2,
            "inputs": f"Q {q.numel() * 2 / 1e6:.0f} MB + K,V {2 * k.numel() * 2 / 1e6:.0f} MB per call",
            "backward": run_prefill_bwd(dev, params, wl, q, k, v, out, lse, st, pairs, n,
                                        steps, warmup, peaks)}


def run_prefill_bwd(dev, params, wl, q, k, v, out, lse, st, pairs, n_tiles, steps, warmup, peaks):
    """Backward of the same prefill (dQ, dK, dV from dO, the forward's output and lse).
    Algorithmic FLOPs = 10 * D per visible pair per query head (the score recompute, dP,
    dV, dK and dQ products: 2.5x the forward); the computed-tile figure counts the same 5
    products over every planned 128 x 128 tile (masked elements included)."""
    from prefix_sliding_window_b200 import binding as B
    Bn, S, hq, hkv = wl.batch, wl.seq, wl.n_q_heads, wl.n_kv_heads
    do = synth.normal_bf16((Bn, S, hq, D), synth.seed_for(wl.index, 4), dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(B.ps_prefill_bwd_workspace_bytes(params, Bn, S), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        B.ps_masked_prefill_attn_bwd(params, q, k, v, out, do, lse, Bn, S, dq, dk, dv, ws, st)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        B.ps_masked_prefill_attn_bwd(params, q, k, v, out, do, lse, Bn, S, dq, dk, dv, ws, st)
        b.record(stream)
    torch.cuda.synchronize()
    assert st.item() == 0, f"device status {st.item()}"
    ms = [a.elapsed_time(b) for a, b in evs]
    med = statistics.median(ms) / 1e3
    flops = 10 * D * pairs * hq * Bn
    computed = 10 * D * 128 * 128 * n_tiles * hq * Bn
    tflops = flops / med / 1e12
    return {"ms": round(med * 1e3, 4), "ms_p10": round(float(np.percentile(ms, 10)), 4),
            "ms_p90": round(float(np.percentile(ms, 90)), 4),
            "tflops_algorithmic": round(tflops, 1), "unit": "TFLOP/s",
            "frac": round(tflops / peaks["bf16_tflops"], 4),
            "tflops_computed": round(computed / med / 1e12, 1),
            "algorithmic_gflop": round(flops / 1e9, 1), "computed_gflop": round(computed / 1e9, 1),
            "launches_per_call": 4}


# -------------------------------------------------------- full attention leg
def run_full_attention(work: DecodeWorkload, steps: int = 16, warmup: int = 3):
    """Full causal attention over the same positions as the decode workload (every key in
    [0, pos] of a linear cache), one append + ps_full_attn_ref per step."""
    from prefix_sliding_window_b200 import binding as B
    from prefix_sliding_window_b200.cache import LinearCache
    wl, dev = work.wl, work.dev
    Bn, hq, hkv = wl.batch, wl.n_q_heads, wl.n_kv_heads
    n_steps = min(steps + warmup, work.k_new.shape[0])
    steps = n_steps - warmup
    lmax = int(work.pos_start.max().item()) + n_steps + 1
    lin = LinearCache(Bn, hkv, lmax, D, dev, fill=None)
    lp_params = lin.params(hq, wl.rope_theta)
    st = work.status
    chunk = 4096
    for c0 in range(0, lmax, chunk):
        T = min(chunk, lmax - c0)
        kk = synth.normal_bf16((Bn, T, hkv, D), 50_000 + c0, dev)
        vv = synth.normal_bf16((Bn, T, hkv, D), 90_000 + c0, dev)
        B.ps_kv_append_rope(lp_params, lin.struct, kk, vv, None,
                            torch.full((Bn,), c0, dtype=torch.int64, device=dev), T, st)
        del kk, vv
    params = B.make_params(hq, hkv, D, 0, 1, wl.rope_theta)
    ws = torch.empty(max(1, B.ps_full_attn_workspace_bytes(params, Bn, lmax)), dtype=torch.uint8,
                     device=dev)
    q = work.q_raw[:n_steps].clone()
    out = torch.empty_like(work.out[0])
    stream = torch.cuda.current_stream()

    def step(i):
        B.ps_kv_append_rope(lp_params, lin.struct, work.k_new[i], work.v_new[i], q[i], work.pos[i],
                            1, st)
        B.ps_full_attn_ref(params, lin.k, lin.v, lmax, q[i], work.pos[i], Bn, out, None, ws, st)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(warmup, n_steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    assert st.item() == 0
    ms = e0.elapsed_time(e1) / steps
    mean_pos = float(work.pos_start.double().mean().item()) + warmup + steps / 2
    kv_bytes = Bn * (mean_pos + 1) * 2 * hkv * D * 2
    del lin
    return {"workload": wl.name + " (full causal attention over [0, pos])",
            "ms_per_step": round(ms, 4), "tok_per_s": round(Bn / (ms / 1e3), 1),
            "kv_gb_per_step": round(kv_bytes / 1e9, 3),
            "gbs": round(kv_bytes / (ms / 1e3) / 1e9, 1)}


# ------------------------------------------------------------- latency leg
def run_latency(dev, steps: int = 256, warmup: int = 8):
    """Single-sequence decode latency: batch 1, 16/2/128, L_prefix 100, W 512, positions past
    the point where the window slides (612); one step = ps_decode_step (append + decode),
    replayed as a CUDA graph and also launched eagerly."""
    wl = synth.WORKLOADS["decode_b1_w512"]
    import dataclasses
    wl = dataclasses.replace(wl, pos_lo=2047 - steps - warmup, pos_hi=2047 - steps - warmup)
    n = steps + warmup
    work = DecodeWorkload(wl, dev, 0, n)
    stream = torch.cuda.current_stream()

    def step(i):
        work.step(i)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(warmup, n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    eager_us = e0.elapsed_time(e1) / steps * 1e3
    work.q.copy_(work.q_raw)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(warmup, n):
            step(i)
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    assert work.status.item() == 0
    graph_us = e0.elapsed_time(e1) / steps * 1e3
    return {"leg": "latency", "workload": wl.name, "positions": f"{wl.pos_lo + warmup}.."
            f"{wl.pos_lo + n - 1}", "visible_keys": wl.l_prefix + wl.window,
            "step_us_graph": round(graph_us, 2), "step_us_eager": round(eager_us, 2),
            "kernels_per_step": work.kernels_per_step()}


# ------------------------------------------------------ long-trace sweep leg
def _fill_cache(B, params, cache_struct, Bn, hkv, ranges, dev, seed, st, chunk=2048):
    """Append N(0,1) tokens at absolute positions [lo, hi) for every sequence."""
    for lo, hi in ranges:
        for c0 in range(lo, hi, chunk):
            T = min(chunk, hi - c0)
            k = synth.normal_bf16((Bn, T, hkv, D), seed + c0, dev)
            v = synth.normal_bf16((Bn, T, hkv, D), seed + 7 * c0 + 1, dev)
            B.ps_kv_append_rope(params, cache_struct, k, v, None,
                                torch.full((Bn,), c0, dtype=torch.int64, device=dev), T, st)
            del k, v


SWEEP_POINTS = (4096, 8192, 16384, 32768, 65536, 131072)


def _graph_time(fn, n: int, warmup: int):
    """Device time per call of fn(i), i = 0 .. n-1, replayed as one CUDA graph after
    `warmup` eager calls (those use the same i range: fn must be repeatable)."""
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        fn(i % n)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / n


def _eager_median(fn, n: int):
    """Median device time of n eager calls fn(i), each bracketed by CUDA events."""
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        fn(i)
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median([a.elapsed_time(b) for a, b in evs])


def run_sweep(dev, steps: int = 20, warmup: int = 3, points=SWEEP_POINTS):
    """Long-trace decode sweep: batch 256, 16/2/128, W = 8192; every sequence at position
    P + i (i = the step) for P in {4K, ..., 128K}; prefix sliding (L_prefix = 100) vs pure
    sliding window (L_prefix = 0) vs full attention over [0, P + i].  Per point and mode:
    one decode step = append of the new token (Continue-PE RoPE) + attention, `steps` steps
    replayed as a CUDA graph (step_us); the attention call alone, eager with CUDA events
    (attn_us).  GB/s on algorithmic bytes (K+V of every visible key, q and out; the step
    adds the append's bytes).  Every point's K/V is far larger than L2 (>= 1 GB)."""
    from prefix_sliding_window_b200 import binding as B
    from prefix_sliding_window_b200.cache import LinearCache, PrefixSlidingCache
    wl = synth.WORKLOADS["decode_sweep_b256_w8192"]
    Bn, hq, hkv, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.window
    peaks = _peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    n = steps
    k_new = synth.normal_bf16((n, Bn, hkv, D), synth.seed_for(wl.index, 1), dev)
    v_new = synth.normal_bf16((n, Bn, hkv, D), synth.seed_for(wl.index, 2), dev)
    q_raw = synth.normal_bf16((n, Bn, hq, D), synth.seed_for(wl.index, 3), dev)
    q = q_raw.clone()
    out = torch.empty((n, Bn, hq, D), dtype=torch.bfloat16, device=dev)
    kv_tok = 2 * hkv * D * 2
    qo = 2 * Bn * hq * D * 2
    append_bytes = Bn * (2 * 2 * hkv * D * 2 + 2 * hq * D * 2 + 8)
    res_points = []
    for P in points:
        pos = torch.stack([torch.full((Bn,), P + i, dtype=torch.int64, device=dev)
                           for i in range(n)])
        res = {"position": P}
        for mode in ("prefix_sliding", "sliding_window", "full"):
            if mode == "full":
                lmax = P + n + 1
                cache = LinearCache(Bn, hkv, lmax, D, dev, fill=None)
                aparams = cache.params(hq, wl.rope_theta)
                _fill_cache(B, aparams, cache.struct, Bn, hkv, [(0, P)], dev, 1000, st)
                dparams = B.make_params(hq, hkv, D, 0, 1, wl.rope_theta)
                ws = torch.empty(max(1, B.ps_full_attn_workspace_bytes(dparams, Bn, lmax)),
                                 dtype=torch.uint8, device=dev)

                def attn(i, cache=cache, dparams=dparams, ws=ws, lmax=lmax):
                    B.ps_full_attn_ref(dparams, cache.k, cache.v, lmax, q[i], pos[i], Bn, out[i],
                                       None, ws, st)

                def step(i, cache=cache, aparams=aparams, attn=attn):
                    B.ps_kv_append_rope(aparams, cache.struct, k_new[i].view(Bn, 1, hkv, D),
                                        v_new[i].view(Bn, 1, hkv, D), q[i].view(Bn, 1, hq, D),
                                        pos[i], 1, st)
                    attn(i)
                keys = [P + i + 1 for i in range(n)]
            else:
                lp = wl.l_prefix if mode == "prefix_sliding" else 0
                cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
                dparams = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
                _fill_cache(B, dparams, cache.struct, Bn, hkv,
                            [(0, min(lp, P)), (max(lp, P - w + 1), P)], dev, 1000, st)
                ws = torch.empty(max(1, B.ps_decode_workspace_bytes(dparams, Bn)),
                                 dtype=torch.uint8, device=dev)

                def attn(i, cache=cache, dparams=dparams, ws=ws):
                    B.ps_decode_attn(dparams, cache.struct, q[i], pos[i], out[i], None, ws, st)

                def step(i, cache=cache, dparams=dparams, ws=ws):
                    B.ps_decode_step(dparams, cache.struct, k_new[i], v_new[i], q[i], pos[i],
                                     out[i], None, ws, st)
                keys = [min(P + i + 1, lp + w) for i in range(n)]
            q.copy_(q_raw)
            step_ms = _graph_time(step, n, warmup)
            attn_ms = _eager_median(attn, n)
            torch.cuda.synchronize()
            assert st.item() == 0, st.item()
            attn_bytes = Bn * statistics.mean(keys) * kv_tok + qo
            step_bytes = attn_bytes + append_bytes
            gbs = step_bytes / (step_ms / 1e3) / 1e9
            agbs = attn_bytes / (attn_ms / 1e3) / 1e9
            res[mode] = {"step_us": round(step_ms * 1e3, 1), "attn_us": round(attn_ms * 1e3, 1),
                         "keys_per_seq": round(statistics.mean(keys), 1),
                         "step_gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "frac_of_8tbs_spec": round(gbs / 8000.0, 4),
                         "attn_gbs": round(agbs, 1),
                         "attn_frac": round(agbs / peaks["hbm_gbs"], 4),
                         "tok_per_s": round(Bn / (step_ms / 1e3), 1)}
            del cache, ws, attn, step
            torch.cuda.empty_cache()
        res["ps_over_full_speedup"] = round(res["full"]["step_us"] / res["prefix_sliding"]["step_us"],
                                            2)
        res_points.append(res)
    flat = [r["prefix_sliding"]["step_us"] for r in res_points if r["position"] >= 8192]
    fr = [r["prefix_sliding"]["frac"] for r in res_points if r["position"] >= 8192]
    return {"workload": wl.name, "batch": Bn, "l_prefix": wl.l_prefix, "window": w,
            "steps_per_point": n, "launch": "CUDA graph of the steps (step_us); eager calls "
            "with CUDA events (attn_us)", "peak_hbm_gbs": peaks["hbm_gbs"],
            "peak_source": peaks["source"], "points": res_points,
            "ps_step_us_spread_8k_128k": round((max(flat) - min(flat)) / min(flat), 4) if flat else None,
            "ps_min_frac_8k_128k": min(fr) if fr else None}


# ------------------------------------------------------- shared-prefix decode leg
def run_shared(dev, steps: int = 20, warmup: int = 3):
    """Shared-prefix decode: 256 sequences in 4 groups of 64 share their group's 2000-token
    prompt prefix; W = 4096; positions U[8192, 131072] (full windows).  The same batch runs
    through plain decode with the prefix copied into every sequence.  Attention calls only
    (the append is the same for both); HBM GB/s on each path's algorithmic bytes."""
    from prefix_sliding_window_b200 import binding as B
    wl = synth.WORKLOADS["decode_shared_b256_g64_lp2000_w4096"]
    Bn, hq, hkv, lp, w, gs = (wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window,
                              wl.group_size)
    G = Bn // gs
    peaks = _peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seed = synth.seed_for(wl.index)
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, seed, dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    # cache contents do not change the work; N(0,1) values stand in for rotated keys
    pre_k = synth.normal_bf16((G, hkv, lp, D), seed + 1, dev)
    pre_v = synth.normal_bf16((G, hkv, lp, D), seed + 2, dev)
    ring_k = synth.normal_bf16((Bn, hkv, w, D), seed + 3, dev)
    ring_v = synth.normal_bf16((Bn, hkv, w, D), seed + 4, dev)
    grp = torch.arange(Bn, device=dev) // gs
    copy_k, copy_v = pre_k[grp].contiguous(), pre_v[grp].contiguous()
    q = synth.normal_bf16((Bn, hq, D), seed + 5, dev)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    shared = B.make_cache(pre_k, pre_v, ring_k, ring_v, Bn)
    plain = B.make_cache(copy_k, copy_v, ring_k, ring_v, Bn)
    ws_s = torch.empty(B.ps_decode_shared_prefix_workspace_bytes(params, Bn, gs),
                       dtype=torch.uint8, device=dev)
    ws_p = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                       device=dev)
    stream = torch.cuda.current_stream()
    calls = {
        "shared_prefix": lambda: B.ps_decode_attn_shared_prefix(params, shared, gs, q, pos, out,
                                                                None, ws_s, st),
        "plain": lambda: B.ps_decode_attn(params, plain, q, pos, out, None, ws_p, st),
    }
    kv_tok = 2 * hkv * D * 2
    qo = 2 * Bn * hq * D * 2
    bytes_ = {"shared_prefix": G * lp * kv_tok + Bn * w * kv_tok + qo,
              "plain": Bn * (lp + w) * kv_tok + qo}
    res = {}
    for name, fn in calls.items():
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        assert st.item() == 0, st.item()
        ms = statistics.median([a.elapsed_time(b) for a, b in evs])
        gbs = bytes_[name] / (ms / 1e3) / 1e9
        res[name] = {"attn_us": round(ms * 1e3, 1), "tok_per_s": round(Bn / (ms / 1e3), 1),
                     "bytes_per_call": int(bytes_[name]), "gbs": round(gbs, 1),
                     "frac": round(gbs / peaks["hbm_gbs"], 4)}
    res["speedup"] = round(res["plain"]["attn_us"] / res["shared_prefix"]["attn_us"], 3)
    return {"leg": "shared", "workload": wl.name, "groups": G, "group_size": gs, "steps": steps,
            "peak_hbm_gbs": peaks["hbm_gbs"], **res}


# ------------------------------------------------------------- Reset PE leg
def run_reset(dev, steps: int = 16, warmup: int = 3):
    """Reset PE vs Continue PE on the batch-64 decode workload (16/2/128, L_prefix 100,
    W 4096, positions U[8192, 131072]).  Per step: Continue PE = append (T = 1) + decode;
    Reset PE here = append + Reset-PE decode (the same cache; only the query is rotated
    again for the prefix rows); Reset PE done literally = the visible tokens re-appended at
    their renumbered ids (T = L_prefix + W from un-rotated keys) + the query + decode."""
    from prefix_sliding_window_b200 import binding as B
    from prefix_sliding_window_b200.cache import PrefixSlidingCache
    wl = synth.WORKLOADS[WORKLOAD]
    Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    peaks = _peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seed = synth.seed_for(wl.index, 9)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    pos0 = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, seed, dev)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
    ring_k = synth.normal_bf16((Bn, hkv, w, D), seed + 1, dev)
    cache.k_ring.copy_(ring_k)
    cache.v_ring.copy_(ring_k)
    cache.k_prefix.normal_()
    cache.v_prefix.normal_()
    del ring_k
    T = lp + w  # visible tokens once the window is full
    raw_k = synth.normal_bf16((Bn, T, hkv, D), seed + 2, dev)  # un-rotated, in id order
    raw_v = synth.normal_bf16((Bn, T, hkv, D), seed + 3, dev)
    scratch = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
    n = warmup + steps
    k_new = synth.normal_bf16((n, Bn, 1, hkv, D), seed + 4, dev)
    v_new = synth.normal_bf16((n, Bn, 1, hkv, D), seed + 5, dev)
    q_raw = synth.normal_bf16((n, Bn, hq, D), seed + 6, dev)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    zeros = torch.zeros(Bn, dtype=torch.int64, device=dev)
    qid = torch.full((Bn,), T - 1, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def continue_pe(i, q):
        p = pos0 + i
        B.ps_kv_append_rope(params, cache.struct, k_new[i], v_new[i], q, p, 1, st)
        B.ps_decode_attn(params, cache.struct, q, p, out, None, ws, st)

    def reset_here(i, q):
        p = pos0 + i
        B.ps_kv_append_rope(params, cache.struct, k_new[i], v_new[i], q, p, 1, st)
        B.ps_decode_attn_reset_pe(params, cache.struct, q, p, out, None, ws, st)

    def reset_literal(i, q):
        B.ps_kv_append_rope(params, scratch.struct, raw_k, raw_v, None, zeros, T, st)
        B.ps_kv_append_rope(params, scratch.struct, k_new[i], v_new[i], q, qid, 1, st)
        B.ps_decode_attn(params, scratch.struct, q, qid, out, None, ws, st)

    res = {}
    kv_tok = 2 * hkv * D * 2
    for name, fn in (("continue_pe", continue_pe), ("reset_pe", reset_here),
                     ("reset_pe_literal", reset_literal)):
        qs = q_raw.clone()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n):
            evs[i][0].record(stream)
            fn(i, qs[i])
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        assert st.item() == 0, st.item()
        ms = statistics.median([a.elapsed_time(b) for a, b in evs[warmup:]])
        res[name] = {"step_us": round(ms * 1e3, 1), "tok_per_s": round(Bn / (ms / 1e3), 1)}
    # bytes per step: decode reads the visible K/V; the literal path also reads the
    # un-rotated keys/values and writes them rotated
    res["continue_pe"]["kv_bytes"] = Bn * T * kv_tok
    res["reset_pe"]["kv_bytes"] = Bn * T * kv_tok
    res["reset_pe_literal"]["kv_bytes"] = 3 * Bn * T * kv_tok
    res["literal_over_here"] = round(res["reset_pe_literal"]["step_us"] /
                                     res["reset_pe"]["step_us"], 2)
    res["here_over_continue"] = round(res["reset_pe"]["step_us"] /
                                      res["continue_pe"]["step_us"], 3)
    return {"leg": "reset", "workload": wl.name, "steps": steps,
            "peak_hbm_gbs": peaks["hbm_gbs"], **res}


# ------------------------------------------------------- appended-prefix leg
def run_pin(dev, steps: int = 20, warmup: int = 3, n_pin: int = 1024):
    """Tokens appended to the pinned prefix: the batch-64 decode workload (16/2/128,
    L_prefix 100, W 4096, positions U[8192, 131072]) where every sequence has promoted
    n_pin earlier tokens (now outside its window).  Decode reads L_prefix + n_pin + W keys
    per sequence; compared with the same batch without promotions, and the promotion of
    256 window tokens per sequence (ps_kv_pin) is timed on its own."""
    from prefix_sliding_window_b200 import binding as B
    wl = synth.WORKLOADS[WORKLOAD]
    Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    lcap = lp + n_pin + 256
    peaks = _peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seed = synth.seed_for(wl.index, 11)
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, seed, dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    k_pre = synth.normal_bf16((Bn, hkv, lcap, D), seed + 1, dev)
    v_pre = synth.normal_bf16((Bn, hkv, lcap, D), seed + 2, dev)
    k_ring = synth.normal_bf16((Bn, hkv, w, D), seed + 3, dev)
    v_ring = synth.normal_bf16((Bn, hkv, w, D), seed + 4, dev)
    cache = B.make_cache(k_pre, v_pre, k_ring, v_ring, Bn)
    # n_pin promoted tokens per sequence, all before the window start
    start = (pos - w - n_pin).clamp(min=lp).view(Bn, 1)
    pin_pos = torch.full((Bn, lcap - lp), -1, dtype=torch.int64, device=dev)
    pin_pos[:, :n_pin] = start + torch.arange(n_pin, device=dev).view(1, n_pin)
    pin_count = torch.full((Bn,), n_pin, dtype=torch.int32, device=dev)
    no_pins = torch.zeros(Bn, dtype=torch.int32, device=dev)
    q = synth.normal_bf16((Bn, hq, D), seed + 5, dev)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_pinned_workspace_bytes(params, Bn, lcap)),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n=steps):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        assert st.item() == 0, st.item()
        return statistics.median([a.elapsed_time(b) for a, b in evs])

    kv_tok = 2 * hkv * D * 2
    res = {}
    for name, cnt, keys in (("with_pins", pin_count, lp + n_pin + w), ("no_pins", no_pins,
                                                                        lp + w)):
        ms = timed(lambda cnt=cnt: B.ps_decode_attn_pinned(params, cache, lcap, cnt, pin_pos, q,
                                                           pos, out, None, ws, st))
        gbs = Bn * keys * kv_tok / (ms / 1e3) / 1e9
        res[name] = {"attn_us": round(ms * 1e3, 1), "keys_per_seq": keys,
                     "tok_per_s": round(Bn / (ms / 1e3), 1), "gbs": round(gbs, 1),
                     "frac": round(gbs / peaks["hbm_gbs"], 4)}
    # promotion of the newest 256 window tokens of every sequence (a copy of 256 KB each)
    t0 = pos - 255
    t1 = pos + 1
    base = pin_count.clone()
    pp = pin_pos.clone()

    def promote():
        pin_count.copy_(base)
        B.ps_kv_pin(params, cache, lcap, pin_count, pp, t0, t1, pos, st)
    ms = timed(promote)
    res["pin_256_tokens_us"] = round(ms * 1e3, 1)
    res["pin_bytes"] = 2 * Bn * 256 * kv_tok
    return {"leg": "pin", "workload": wl.name, "n_pin": n_pin, "peak_hbm_gbs": peaks["hbm_gbs"],
            **res}


def run_paged(dev, steps: int = 20, warmup: int = 3):
    """Paged store: the batch-64 decode workload (16/2/128, L_prefix 100, W 4096, positions
    U[8192, 131072]) held in a pool of 64-row blocks scattered in a seeded random order,
    each sequence's block table listing its prefix blocks then its W/64 ring blocks.  Paged
    decode is timed beside the contiguous store's decode of the same batch, and one step
    (append of the new token into its block + decode) on its own."""
    from prefix_sliding_window_b200 import binding as B
    from prefix_sliding_window_b200.cache import PrefixSlidingCache
    wl = synth.WORKLOADS[WORKLOAD]
    Bn, hq, hkv, lp, w = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    peaks = _peaks()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seed = synth.seed_for(wl.index, 13)
    pos = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, seed, dev)
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    pre_blocks = -(-lp // 64)
    per_seq = pre_blocks + w // 64
    n_blocks = Bn * per_seq
    g = torch.Generator(device="cpu").manual_seed(seed)
    table = torch.randperm(n_blocks, generator=g).to(torch.int32).view(Bn, per_seq).to(dev)
    k_pool = synth.normal_bf16((n_blocks, hkv, 64, D), seed + 1, dev)
    v_pool = synth.normal_bf16((n_blocks, hkv, 64, D), seed + 2, dev)
    cache = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
    for i, t in enumerate((cache.k_prefix, cache.v_prefix, cache.k_ring, cache.v_ring)):
        t.copy_(synth.normal_bf16(tuple(t.shape), seed + 10 + i, dev))
    q = synth.normal_bf16((Bn, hq, D), seed + 5, dev)
    k_new = synth.normal_bf16((Bn, 1, hkv, D), seed + 6, dev)
    v_new = synth.normal_bf16((Bn, 1, hkv, D), seed + 7, dev)
    q_new = synth.normal_bf16((Bn, 1, hq, D), seed + 8, dev)
    out = torch.empty((Bn, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n=steps):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        assert st.item() == 0, st.item()
        return statistics.median([a.elapsed_time(b) for a, b in evs])

    kv_tok = 2 * hkv * D * 2
    alg = Bn * (lp + w) * kv_tok            # rows visible at a wrapped position
    loaded = Bn * per_seq * 64 * kv_tok     # whole blocks: the last prefix block is partial
    res = {}
    for name, fn in (
            ("paged", lambda: B.ps_decode_attn_paged(params, k_pool, v_pool, table, Bn, q, pos,
                                                     out, None, ws, st)),
            ("contiguous", lambda: B.ps_decode_attn(params, cache.struct, q, pos, out, None, ws,
                                                    st))):
        ms = timed(fn)
        gbs = alg / (ms / 1e3) / 1e9
        res[name] = {"attn_us": round(ms * 1e3, 1), "tok_per_s": round(Bn / (ms / 1e3), 1),
                     "gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4)}
    res["paged"]["gbs_loaded"] = round(loaded / (res["paged"]["attn_us"] / 1e6) / 1e9, 1)

    def step():
        B.ps_kv_append_rope_paged(params, k_pool, v_pool, table, Bn, k_new, v_new, q_new, pos, 1,
                                  st)
        B.ps_decode_attn_paged(params, k_pool, v_pool, table, Bn, q_new.view(Bn, hq, D), pos,
                               out, None, ws, st)
    res["paged_step_us"] = round(timed(step) * 1e3, 1)
    return {"leg": "paged", "workload": wl.name, "n_blocks": n_blocks,
            "blocks_per_seq": per_seq, "alg_bytes": alg, "loaded_bytes": loaded,
            "peak_hbm_gbs": peaks["hbm_gbs"], **res}


# ------------------------------------------------------- full-stack decode leg
def run_stack(dev, batch: int, distinct: int, steps: int = 3, warmup: int = 1):
    """Full-stack decode step: 28 layers x ps_decode_step (append + decode), 16/2/128,
    L_prefix 2000, W 16384, positions in [32768, 262144].  The 28 logical layers are mapped
    round-robin onto `distinct` resident layer caches (all 28 caches of 1024 sequences,
    540 GB, do not fit in one GPU's 180 GB); each layer's working set is far larger than L2,
    so every layer reads its K/V from HBM."""
    from prefix_sliding_window_b200 import binding as B
    from prefix_sliding_window_b200.cache import PrefixSlidingCache
    wl = synth.WORKLOADS["decode_stack_l28_b1024_w16384"]
    Bn, hq, hkv, lp, w, L = batch, wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window, wl.n_layers
    params = B.make_params(hq, hkv, D, lp, w, wl.rope_theta)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    pos0 = synth.uniform_positions(Bn, wl.pos_lo, wl.pos_hi, synth.seed_for(5), dev)
    caches = []
    for li in range(distinct):
        c = PrefixSlidingCache(Bn, hkv, lp, w, D, dev, fill=None)
        # prefix, then the window history [p - W + 1, p - 1] of every sequence
        B.ps_kv_append_rope(params, c.struct, synth.normal_bf16((Bn, lp, hkv, D), 3 * li, dev),
                            synth.normal_bf16((Bn, lp, hkv, D), 3 * li + 1, dev), None,
                            torch.zeros(Bn, dtype=torch.int64, device=dev), lp, st)
        chunk = 1024
        for c0 in range(0, w - 1, chunk):
            T = min(chunk, w - 1 - c0)
            B.ps_kv_append_rope(params, c.struct,
                                synth.normal_bf16((Bn, T, hkv, D), 100 * li + c0, dev),
                                synth.normal_bf16((Bn, T, hkv, D), 100 * li + c0 + 1, dev), None,
                                pos0 - (w - 1) + c0, T, st)
        caches.append(c)
    torch.cuda.synchronize()
    n = warmup + steps
    k_new = synth.normal_bf16((n, L, Bn, hkv, D), 21, dev)
    v_new = synth.normal_bf16((n, L, Bn, hkv, D), 22, dev)
    q_raw = synth.normal_bf16((n, L, Bn, hq, D), 23, dev)
    q = q_raw.clone()
    out = torch.empty((L, Bn, hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, B.ps_decode_workspace_bytes(params, Bn)), dtype=torch.uint8, device=dev)
    pos = torch.stack([pos0 + i for i in range(n)])
    stream = torch.cuda.current_stream()

    def step(i):
        for layer in range(L):
            c = caches[layer % distinct]
            B.ps_decode_step(params, c.struct, k_new[i, layer], v_new[i, layer], q[i, layer],
                             pos[i], out[layer], None, ws, st)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(warmup, n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    assert st.item() == 0
    ms = e0.elapsed_time(e1) / steps
    kv_bytes = L * Bn * (lp + w) * 2 * hkv * D * 2
    step_bytes = kv_bytes + L * Bn * (2 * hq * D * 2 + 2 * 2 * hkv * D * 2 + 2 * hq * D * 2 + 8)
    gbs = step_bytes / (ms / 1e3) / 1e9
    peaks = _peaks()
    res = {"workload": wl.name, "batch": Bn, "layers": L, "distinct_layer_caches": distinct,
           "layer_map": "28 logical layers round-robin onto the distinct caches" if distinct < L
           else "28 distinct layer caches",
           "resident_kv_gb": round(distinct * caches[0].nbytes() / 1e9, 1),
           "ms_per_step": round(ms, 3), "tok_per_s": round(Bn / (ms / 1e3), 1),
           "kv_gb_per_step": round(kv_bytes / 1e9, 1), "gbs": round(gbs, 1),
           "frac": round(gbs / peaks["hbm_gbs"], 4), "frac_of_8tbs_spec": round(gbs / 8000.0, 4),
           "launch": "eager, 28 ps_decode_step calls per step"}
    del caches, k_new, v_new, q_raw, q
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------- CPU oracle leg
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_decode_sample(wl: synth.Workload, n_seq: int, seed_stream: int = 0):
    """Oracle decode of ``n_seq`` sequences of the workload (fresh CPU inputs with the
    workload's shapes).  Returns (sequences decoded, seconds)."""
    import oracle as O
    hq, hkv, lp, w = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    pos = synth.uniform_positions(n_seq, wl.pos_lo, wl.pos_hi, synth.seed_for(wl.index, 900 + seed_stream))
    scale = 1.0 / math.sqrt(D)
    data = []
    for b in range(n_seq):
        p = int(pos[b])
        vis = O.visible_positions(p, lp, w)
        k = synth.normal_bf16((len(vis), hkv, D), 7000 + b + 97 * seed_stream).double().numpy()
        v = synth.normal_bf16((len(vis), hkv, D), 8000 + b + 97 * seed_stream).double().numpy()
        q = synth.normal_bf16((hq, D), 9000 + b + 97 * seed_stream).double().numpy()
        data.append((p, vis, k, v, q))
    t0 = time.perf_counter()
    for p, vis, k, v, q in data:
        k_rot = O.rope_rotate(k, vis[:, None], wl.rope_theta)
        O.attend_gqa(O.rope_rotate(q, p, wl.rope_theta), k_rot, v, scale)
    return n_seq, time.perf_counter() - t0


def cpu_baseline(wl: synth.Workload, budget_s: float = 8.0):
    done, spent, calls = 0, 0.0, 0
    while spent < budget_s:
        n, t = oracle_decode_sample(wl, 8, calls)
        done += n
        spent += t
        calls += 1
    return {"value": round(done / spent, 2), "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{done} sequences of {wl.name} (one decode step each: all {wl.n_q_heads} "
                      f"heads over {wl.l_prefix + wl.window} visible keys), float64 numpy, "
                      f"{spent:.1f} s"}


def cpu_baseline_latency(budget_s: float = 4.0):
    """The oracle on the batch-1 workload (L_prefix 100, W 512): the prompt's 100 tokens, then
    decode steps at positions 100, 101, ... each over its visible keys, until the budget."""
    import oracle as O
    wl = synth.WORKLOADS["decode_b1_w512"]
    hq, hkv, lp, w = wl.n_q_heads, wl.n_kv_heads, wl.l_prefix, wl.window
    S = wl.pos_hi + 1
    k = synth.normal_bf16((S, hkv, D), synth.seed_for(wl.index, 1)).double().numpy()
    v = synth.normal_bf16((S, hkv, D), synth.seed_for(wl.index, 2)).double().numpy()
    q = synth.normal_bf16((S, hq, D), synth.seed_for(wl.index, 3)).double().numpy()
    scale = 1.0 / math.sqrt(D)
    t0 = time.perf_counter()
    steps = 0
    for p in range(lp, S):
        vis = O.visible_positions(p, lp, w)
        O.attend_gqa(O.rope_rotate(q[p], p, wl.rope_theta),
                     O.rope_rotate(k[vis], vis[:, None], wl.rope_theta), v[vis], scale)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    t = time.perf_counter() - t0
    return {"value": round(steps / t, 2), "unit": "tok/s", "cores": _blas_threads(),
            "kind": "oracle", "us_per_step": round(t / steps * 1e6, 1),
            "sample": f"decode steps at positions {lp}..{lp + steps - 1} of {wl.name} "
                      f"({'all' if steps == S - lp else 'first'} {steps} of {S - lp}), "
                      f"float64 numpy, {t:.1f} s"}


def cpu_baseline_prefill():
    """The oracle on one (batch, head) of the prefill workload (8192 rows, 28/4/128 heads
    reduced to one query head and its KV head), every row; the whole workload's time is
    that x heads x batch (extrapolated)."""
    import oracle as O
    wl = synth.WORKLOADS["prefill_b4_s8192_w2048"]
    S, lp, w = wl.seq, wl.l_prefix, wl.window
    Q = synth.normal_bf16((S, 1, D), synth.seed_for(wl.index, 1)).double().numpy()
    K = synth.normal_bf16((S, 1, D), synth.seed_for(wl.index, 2)).double().numpy()
    V = synth.normal_bf16((S, 1, D), synth.seed_for(wl.index, 3)).double().numpy()
    t0 = time.perf_counter()
    O.prefill_reference(Q, K, V, lp, w, 1.0 / math.sqrt(D))
    t = time.perf_counter() - t0
    flops = 4 * D * prefill_visible_pairs(S, lp, w)
    whole = t * wl.n_q_heads * wl.batch
    return {"value": round(flops / t / 1e12, 6), "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle", "s_per_head": round(t, 3),
            "whole_workload_s_extrapolated": round(whole, 1),
            "sample": f"one (batch, head) of {wl.name}: all {S} rows, float64 numpy, "
                      f"{t:.1f} s; whole workload = x {wl.n_q_heads} heads x {wl.batch} "
                      f"(extrapolated)"}


def cpu_baseline_sweep(per_point: int = 2):
    """The oracle on sampled sequences of the long-trace sweep (L_prefix 100, W 8192):
    `per_point` sequences decoded at each position."""
    import dataclasses
    wl = synth.WORKLOADS["decode_sweep_b256_w8192"]
    pts = {}
    for i, P in enumerate(SWEEP_POINTS):
        wp = dataclasses.replace(wl, pos_lo=P, pos_hi=P)
        n, t = oracle_decode_sample(wp, per_point, 300 + i)
        pts[str(P)] = {"seq_per_s": round(n / t, 2), "s_per_seq": round(t / n, 4)}
    return {"unit": "tok/s", "cores": _blas_threads(), "kind": "oracle", "points": pts,
            "sample": f"{per_point} sequences per position, one decode step each (all "
                      f"{wl.n_q_heads} heads), float64 numpy"}


def cpu_baseline_stack(pairs: int = 8):
    """The oracle on `pairs` sampled (sequence, layer) pairs of the full-stack workload
    (L_prefix 2000, W 16384, positions in [32768, 262144]); one full step (28 layers x 1024
    sequences) extrapolated from the per-pair time."""
    wl = synth.WORKLOADS["decode_stack_l28_b1024_w16384"]
    n, t = oracle_decode_sample(wl, pairs, 500)
    per = t / n
    step_s = per * wl.n_layers * wl.batch
    return {"value": round(wl.batch / step_s, 4), "unit": "tok/s", "cores": _blas_threads(),
            "kind": "oracle", "s_per_pair": round(per, 4),
            "step_s_extrapolated": round(step_s, 1),
            "sample": f"{n} (sequence, layer) pairs decoded, float64 numpy, {t:.1f} s; one step "
                      f"= {wl.n_layers} layers x {wl.batch} sequences (extrapolated)"}


def cpu_baselines():
    """Oracle timings of every workload, on this host's cores (reported, not a target)."""
    return {"decode_b1_w512": cpu_baseline_latency(),
            "prefill_b4_s8192_w2048": cpu_baseline_prefill(),
            "decode_sweep_b256_w8192": cpu_baseline_sweep(),
            "decode_stack_l28_b1024_w16384": cpu_baseline_stack()}


def run_reference(args, world, rank):
    """Reference arm: the float64 oracle on the host cores, same metric, unit and config.
    A step decodes the workload's whole batch (64 sequences) when the run is short enough
    (K + W <= 40 steps: about 0.9 s each), otherwise a sample of the batch sized to keep
    the run within about a minute."""
    if rank != 0:
        return None
    wl = synth.WORKLOADS[WORKLOAD]
    per_step = max(1, min(wl.batch, (wl.batch * 40) // (args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_decode_sample(wl, per_step, 1000 + i)
    total_t, total_n = 0.0, 0
    for i in range(args.steps):
        n, t = oracle_decode_sample(wl, per_step, 2000 + i)
        total_t += t
        total_n += n
    value = total_n / total_t
    sample = (f"{per_step} of the {wl.batch} sequences of {WORKLOAD} per step "
              f"({'the whole batch' if per_step == wl.batch else 'a sample'}), float64 numpy")
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": decode_config(wl, world),
        "launch": "host cores, float64 oracle", "sequences_per_step": per_step,
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": _blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of as a CUDA graph")
    ap.add_argument("--leg", default="main", choices=["main", "prefill", "sweep", "stack", "latency",
                                                      "shared", "reset", "pin", "paged"],
                    help="main: the default decode line; prefill/sweep/stack: one extra workload")
    ap.add_argument("--prefill-workload", default="prefill_b4_s8192_w2048",
                    choices=[k for k in synth.WORKLOADS if k.startswith("prefill")],
                    help="workload of the prefill leg")
    ap.add_argument("--stack-batch", type=int, default=1024)
    ap.add_argument("--stack-distinct", type=int, default=6)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the full-attention comparator and the prefill leg")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per decode launch, when known for this kernel")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = _dist_setup()
    dev = torch.device("cuda", local)
    if args.leg != "main":
        if args.leg == "prefill":
            res = {"leg": "prefill", **run_prefill(dev, steps=args.steps, warmup=args.warmup,
                                                   workload=args.prefill_workload)}
        elif args.leg == "sweep":
            res = {"leg": "sweep", **run_sweep(dev)}
        elif args.leg == "latency":
            res = run_latency(dev)
        elif args.leg == "shared":
            res = run_shared(dev)
        elif args.leg == "reset":
            res = run_reset(dev)
        elif args.leg == "pin":
            res = run_pin(dev)
        elif args.leg == "paged":
            res = run_paged(dev)
        else:
            res = run_stack(dev, args.stack_batch, args.stack_distinct)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    line, work = run_decode(args, world, rank, dev)
    if not args.no_extras:
        full = run_full_attention(work)
        full["ps_speedup"] = round(line["value"] / full["tok_per_s"], 2)
        line["full_attention"] = full
        del work
        torch.cuda.empty_cache()
        line["prefill"] = run_prefill(dev)
        torch.cuda.empty_cache()
        line["sweep"] = run_sweep(dev)
        # the full stack: 28 layers of 1024 sequences on 6 resident layer caches (aliased),
        # and 28 distinct layer caches at batch 192 (all that fits)
        line["stack"] = {"aliased": run_stack(dev, 1024, 6),
                         "distinct": run_stack(dev, 192, 28)}
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(synth.WORKLOADS[WORKLOAD])
            if not args.no_extras:
                line["cpu_baselines"] = cpu_baselines()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
