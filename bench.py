"""Benchmark of the LLA decode hot path on B200.

One step = one decode step of the workload: decode attention at each listed loop
t over every layer's latent cache, then encode of the finished tokens (the
per-loop K/V of the token that just completed its last loop).  Default workload:
the capacity regime, per-head LLA at 21.3x (T=4, H=16, d=128, r_k=16, r_v=32),
batch 256, 4096-token context, all 24 shared layers back to back.

Prints one JSON line (rank 0).  `value` is algorithmic HBM GB/s over the whole
step with inputs resident in HBM; `e2e` is the same metric with each step's host
inputs (queries, in-flight K/V, the finished tokens' per-loop rows and their new
positions) copied in from pinned host memory and every output copied back inside
the timed region, the latent cache resident on the device.  `sub_records` hold
the other workloads (per-head 4x, LLA-2D, the deep-loop decode and prefill
encode), each with its own roofline.  `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload (the reference arm).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "perhead_21x_T4_H16_d128_r16_32_B256_n4096_L24"
# workloads measured as sub-records of a default run (the tiny one is a parity case)
SUB_WORKLOADS = ("perhead_4x_T4_H16_d128_r96_160_B8_n4096", "lla2d_T4_H16_d128_r64_128_B512_n4096",
                 "deeploop_32x_T32_H8_d96_r64_128_B16_n32768")
METRIC = "LLA decode-attention HBM GB/s (% of peak) and ctx-tokens/s per loop step"
# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu capture of the
# current kernels (profiles/); a workload without a capture of the current code reports null.
NCU_TRAFFIC = {"perhead_4x_T4_H16_d128_r96_160_B8_n4096": 277.01e6,
               "perhead_21x_T4_H16_d128_r16_32_B256_n4096_L24": 1650.94e6,
               "lla2d_T4_H16_d128_r64_128_B512_n4096": 1008.05e6,
               # encode (the dominant kernel): a 32768-token capture scaled by 16 tokens-wise
               "deeploop_32x_T32_H8_d96_r64_128_B16_n32768": 55.24e9}
# The same for the full-memory fast path (dominant kernel: full_decode_kernel).
NCU_TRAFFIC_FULL = {"perhead_4x_T4_H16_d128_r96_160_B8_n4096": 272.19e6}
# The same for decoupled RoPE (--d-rope), keyed by (workload, d_rope).
NCU_TRAFFIC_DECOUPLED = {("perhead_4x_T4_H16_d128_r96_160_B8_n4096", 64): 276.60e6}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="lla", choices=["lla", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOAD_ORDER)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sub", action="store_true",
                   help="measure the default workload only (no sub-records of the others)")
    p.add_argument("--encode-tokens", type=int, default=0,
                   help="override the workload's tokens encoded per step (profiling aid)")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch (profiling aid: a smaller capture)")
    p.add_argument("--layers", type=int, default=0,
                   help="override the workload's layer count (profiling aid)")
    p.add_argument("--path", default="latent", choices=["latent", "full"],
                   help="latent: decode over the latent cache (rebuild on read); full: the "
                        "full-memory fast path (K/V rebuilt once per token into a full bf16 "
                        "cache per loop, ordinary attention)")
    p.add_argument("--eager", action="store_true",
                   help="launch every call of a timed step from the host; by default a step "
                        "(every layer's decode at each loop, then the encode of the finished "
                        "tokens) is captured once as CUDA graphs and the replays are timed")
    p.add_argument("--d-rope", type=int, default=0,
                   help="decoupled RoPE: rotate only the first D_ROPE dims of each head and "
                        "absorb the rest into a NoPE content path (32 or 64; 0 = whole head)")
    p.add_argument("--evict", default="",
                   help="SINK,WINDOW: decode over a sink + window retention budget of the "
                        "history (eviction composed with the latent cache)")
    return p.parse_args()


# ----------------------------------------------------------------------------- byte counts

def decode_bytes(w, n_ctx: int) -> int:
    """Algorithmic HBM bytes of one decode call (one layer, one loop)."""
    L = w.H if w.mode == synth.MODE_PER_HEAD else 1
    lat = w.B * n_ctx * (w.r_k + w.r_v) * 2 * L
    pos = w.B * n_ctx * 4
    weights = w.H * w.d * (w.r_k + w.r_v) * 4 + 2 * w.H * w.d * 4
    io = 4 * w.B * w.H * w.d * 4
    return lat + pos + weights + io


def full_decode_bytes(w, n_ctx: int) -> int:
    """Algorithmic HBM bytes of one full-memory decode call: bf16 K and V rows of the
    attended history plus the per-head inputs and output."""
    return w.B * w.H * n_ctx * 2 * w.d * 2 + 4 * w.B * w.H * w.d * 4 + 2 * w.B * 4


def full_rebuild_bytes(w, n_rows: int) -> int:
    """Bytes of rebuilding n_rows cache rows at one loop: latents and positions in,
    W_up and mu, bf16 K/V rows out."""
    L = w.H if w.mode == synth.MODE_PER_HEAD else 1
    return (n_rows * (L * (w.r_k + w.r_v) * 2 + 4 + 8) + w.H * w.d * (w.r_k + w.r_v + 2) * 4
            + n_rows * w.H * 2 * w.d * 2)


def encode_bytes(w, n_tok: int) -> int:
    L = w.H if w.mode == synth.MODE_PER_HEAD else 1
    width = w.T * w.d * (1 if L > 1 else w.H)
    x = n_tok * w.T * w.H * w.d * 2 * 2
    wd = L * (w.r_k + w.r_v) * width * 2 + L * (w.r_k + w.r_v) * 4
    out = n_tok * L * (w.r_k + w.r_v) * 2 + n_tok * 8
    return x + wd + out


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 20 ms, with host timestamps.

    Started before the last warm-up steps (nvidia-smi needs a few hundred ms to
    produce its first line); only the samples taken inside the timed region are
    kept, or, when that region is shorter than the sampling period, the samples
    nearest to it (the GPU is busy with the same steps on both sides).
    """

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-i", str(gpu_index),
                                       "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.p = None

    def lines(self) -> int:
        self.f.flush()
        try:
            return sum(1 for _ in open(self.f.name))
        except OSError:
            return 0

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        self.p.wait(timeout=10)
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        samples = []
        for r in rows:
            try:
                ts = time.mktime(time.strptime(r[0].strip().split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + r[0].strip().split(".")[1]) if "." in r[0] else 0.0
                samples.append((ts, float(r[2]), float(r[3]),
                                {n for n, v in zip(names, r[6:10]) if v.strip().lower() == "active"}))
            except (ValueError, IndexError):
                continue
        if not samples or self.t0 is None or self.t1 is None:
            return None
        inside = [x for x in samples if self.t0 <= x[0] <= self.t1]
        if not inside:   # timed region shorter than the sampling period: nearest samples
            mid = 0.5 * (self.t0 + self.t1)
            inside = sorted(samples, key=lambda x: abs(x[0] - mid))[:2]
        return {"sm_mhz": float(np.median([x[1] for x in inside])),
                "sm_max_mhz": inside[-1][2],
                "reasons": sorted(set().union(*[x[3] for x in inside])),
                "samples": len(inside)}


# ----------------------------------------------------------------------------- GPU arm

def build_state(w, device, d_rope=0):
    import torch
    import looped_transformer_decode_b200 as lla

    cfg = lla.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode, d_rope=d_rope)
    append = w.encode_tokens <= w.B               # decode-time append: one new row per sequence
    n_cap = w.n + 1 if append else w.n
    layers = []
    for layer in range(w.layers):
        cod = synth.workload_codec(w, seed_offset=layer)
        packed = lla.codec_pack(cfg, *(torch.from_numpy(cod[k]).to(device) for k in
                                       ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
        x = synth.workload_tensors(w, device, seed_offset=layer, n=n_cap)
        x["ctx_len"].fill_(w.n)
        x["q_pos"].fill_(w.n)
        layers.append({"packed": packed, **x})
    rope = lla.rope_table(cfg, n_cap + 1)
    ws = lla.decode_workspace(cfg, w.B, n_cap)
    n_tok = w.encode_tokens
    xk, xv = synth.encode_inputs(w, device, n_tok)
    if append:
        slot = torch.arange(w.B, device=device, dtype=torch.int64) * n_cap + w.n
    else:
        slot = torch.arange(n_tok, device=device, dtype=torch.int64)
    out = torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=device)
    return {"cfg": cfg, "layers": layers, "rope": rope, "ws": ws, "xk": xk, "xv": xv,
            "slot": slot, "out": out, "n_cap": n_cap}


def apply_eviction(lla, w, st, sink: int, window: int) -> int:
    """Keep a sink + window budget of each sequence's n-token history.

    Slot bookkeeping of lla_evict_slot: the kept tokens' positions are written at
    their slots and ctx_len becomes the budget; the new token of each step is
    appended at the slot lla_evict_append gives position n.  Returns the number of
    attended history tokens.
    """
    import torch

    keep = list(range(min(sink, w.n))) + list(range(max(sink, w.n - window), w.n))
    slots = [lla.evict_slot(sink, window, p) for p in keep]
    n_cap = st["n_cap"]
    for L in st["layers"]:
        pos = L["positions"]
        pos[:, torch.tensor(slots, device=pos.device)] = torch.tensor(keep, dtype=pos.dtype,
                                                                      device=pos.device)
        L["ctx_len"].fill_(len(keep))
    if w.encode_tokens <= w.B:                    # decode-time append into the ring
        pos_new = torch.full((w.B,), w.n, dtype=torch.int32, device=st["slot"].device)
        pos_tab = st["layers"][0]["positions"].clone()
        ctx_tab = st["layers"][0]["ctx_len"].clone()
        st["slot"] = lla.evict_append(w.B, n_cap, sink, window, pos_new, pos_tab, ctx_tab)
    return len(keep)


def build_full(lla, w, st, device):
    """Full-memory fast path: rebuild every history row once into a bf16 K/V cache per
    (layer, loop).  Returns the rebuild time of one (layer, loop) cache in ms."""
    import torch

    need = w.layers * len(w.loops) * 2 * lla.full_kv_bytes(st["cfg"], w.B, st["n_cap"])
    free, _ = torch.cuda.mem_get_info(device)
    if need > 0.85 * free:
        raise SystemExit(f"full-memory path needs {need / 2**30:.1f} GiB of full K/V caches for "
                         f"{w.layers} layers x {len(w.loops)} loops; {free / 2**30:.1f} GiB free")
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rebuild_ms = []
    for L in st["layers"]:
        L["full"] = {}
        for t in w.loops:
            kf, vf = lla.full_cache_alloc(st["cfg"], w.B, st["n_cap"], device)
            s.record()
            lla.full_rebuild(st["cfg"], L["packed"], st["rope"], t, L["positions"], L["c_k"],
                             L["c_v"], kf, vf)
            e.record()
            torch.cuda.synchronize()
            rebuild_ms.append(s.elapsed_time(e))
            L["full"][t] = (kf, vf)
    st["fws"] = lla.full_decode_workspace(st["cfg"], w.B, st["n_cap"], device)
    return float(np.median(rebuild_ms))


def run_step_full(lla, w, st, events=None):
    """One step of the fast path: decode every loop over its full cache, then encode
    the new tokens and rebuild their rows into every loop's cache."""
    if st.get("flush") is not None:
        st["flush"].add_(1)
    for t in ([] if st.get("skip_decode") else w.loops):
        for L in st["layers"]:
            if events is not None:
                events[0].append(_event())
            kf, vf = L["full"][t]
            lla.full_decode_attn(st["cfg"], st["rope"], L["ctx_len"], L["q"], L["k_self"],
                                 L["v_self"], L["q_pos"], kf, vf, out=st["out"], ws=st["fws"])
            if events is not None:
                events[1].append(_event())
    for L in ([] if st.get("skip_append") else st["layers"]):
        if events is not None:
            events[2].append(_event())
        lla.encode(st["cfg"], L["packed"], st["xk"], st["xv"], st["slot"], L["c_k"], L["c_v"])
        for t in w.loops:
            kf, vf = L["full"][t]
            lla.full_rebuild(st["cfg"], L["packed"], st["rope"], t, L["positions"], L["c_k"],
                             L["c_v"], kf, vf, slot=st["slot"])
        if events is not None:
            events[3].append(_event())


def capture_step_graphs(lla, w, st):
    """The step as two CUDA graphs: every layer's decode at each loop, then the
    encode (and, on the full-memory path, the row rebuild) of the finished tokens."""
    import torch

    flush = st.pop("flush", None)               # the L2 flush stays outside the graphs
    g_dec, g_enc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    dec_only = dict(st, skip_append=True)
    with torch.cuda.graph(g_dec):
        run_step(lla, w, dec_only)
    enc_only = dict(st, skip_decode=True)
    with torch.cuda.graph(g_enc):
        run_step(lla, w, enc_only)
    torch.cuda.synchronize()
    return {"dec": g_dec, "enc": g_enc, "flush": flush}


def replay_step_graphs(st, graphs, events, n_dec, n_enc):
    """One timed step from the captured graphs; the per-call times are the graph
    times divided by the calls each graph holds."""
    if graphs["flush"] is not None:
        graphs["flush"].add_(1)
    e = [_event() for _ in range(3)]
    e[0].record()
    graphs["dec"].replay()
    e[1].record()
    graphs["enc"].replay()
    e[2].record()
    events[0].append((e[0], n_dec))
    events[1].append((e[1], n_dec))
    events[2].append((e[1], n_enc))
    events[3].append((e[2], n_enc))


def run_step(lla, w, st, events=None):
    if st.get("full_path"):
        return run_step_full(lla, w, st, events)
    if st.get("flush") is not None:
        st["flush"].add_(1)                       # working set below L2: evict it first
    for t in ([] if st.get("skip_decode") else w.loops):
        for L in st["layers"]:
            if events is not None:
                events[0].append(_event())
            lla.decode_attn(st["cfg"], L["packed"], st["rope"], t, L["ctx_len"], L["q"],
                            L["k_self"], L["v_self"], L["positions"], L["q_pos"], L["c_k"],
                            L["c_v"], out=st["out"], ws=st["ws"])
            if events is not None:
                events[1].append(_event())
    for L in ([] if st.get("skip_append") else st["layers"]):
        if events is not None:
            events[2].append(_event())
        lla.encode(st["cfg"], L["packed"], st["xk"], st["xv"], st["slot"], L["c_k"], L["c_v"])
        if events is not None:
            events[3].append(_event())


def _event():
    import torch

    e = torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def barrier_sync(dist_on, cuda=True):
    import torch
    import torch.distributed as dist

    if dist_on:
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def over_ranks(values, op, device, dist_on):
    """Element-wise max ("max") or min ("min") of a list of floats over all ranks
    (every rank takes part; identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not dist_on:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.MIN)
    return [float(v) for v in t]


def _oracle_cores():
    """Host cores this process may run on (its CPU affinity set)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):  # pragma: no cover
        return os.cpu_count() or 1


def _blas_limit(n):
    """Context manager capping the BLAS threads of NumPy at n (no-op without threadpoolctl)."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=int(n))
    except Exception:  # pragma: no cover
        import contextlib
        return contextlib.nullcontext()


_ORACLE_INPUTS = {}


def _oracle_inputs(w):
    """The oracle's codec and one sequence of workload w (drawn once per process)."""
    import torch
    import oracle as O

    if w.name not in _ORACLE_INPUTS:
        cfg = O.Cfg(w.T, w.H, w.d, w.r_k, w.r_v, w.mode)
        cod = synth.workload_codec(w)
        codec = O.Codec(*(cod[k].astype(np.float64) for k in
                          ("W_down_k", "W_down_v", "W_up_k", "W_up_v", "mu_k", "mu_v")))
        x = synth.workload_tensors(w, "cpu", seed_offset=99, B=1)
        arr = {k: (v.float().numpy().astype(np.float64)
                   if v.dtype in (torch.bfloat16, torch.float32) else v.numpy())
               for k, v in x.items()}
        _ORACLE_INPUTS[w.name] = (cfg, codec, arr)
    return _ORACLE_INPUTS[w.name]


def _oracle_pairs(w, seconds, loops, d_rope, threads):
    """(b, h) pairs of workload w the float64 oracle decodes in about `seconds`,
    with its BLAS threads capped at `threads`; returns (pairs, elapsed seconds)."""
    import oracle as O

    cfg, codec, arr = _oracle_inputs(w)
    loops = loops or w.loops
    pairs = 0
    with _blas_limit(threads):
        t0 = time.perf_counter()
        while True:
            h = pairs % w.H
            t = loops[pairs % len(loops)]
            if d_rope:
                O.decode_attn_cache_decoupled(cfg, codec, t, arr["q"], arr["k_self"],
                                              arr["v_self"], arr["c_k"], arr["c_v"],
                                              arr["positions"], arr["q_pos"], arr["ctx_len"],
                                              d_rope, pairs=[(0, h)])
            else:
                O.decode_attn_cache(cfg, codec, t, arr["q"], arr["k_self"], arr["v_self"],
                                    arr["c_k"], arr["c_v"], arr["positions"], arr["q_pos"],
                                    arr["ctx_len"], pairs=[(0, h)])
            pairs += 1
            el = time.perf_counter() - t0
            if el >= seconds and pairs >= 2:
                return pairs, el


def cpu_baseline_sample(w, seconds: float, loops=None, d_rope=0, one_thread=True):
    """Time the float64 oracle on (b, h) pairs of the workload at full context.

    The oracle runs with its BLAS threads set to the host cores this process may
    use (``cores``); a second, shorter sample with one thread is reported beside
    it.  GB/s are the GPU path's algorithmic bytes per (b, h) pair over the time.
    """
    cores = _oracle_cores()
    share = 0.75 if one_thread else 1.0
    pairs, el = _oracle_pairs(w, seconds * share, loops, d_rope, cores)
    per_pair = decode_bytes(w, w.n) / (w.B * w.H)
    out = {"value": pairs * per_pair / el / 1e9, "unit": "GB/s", "cores": int(cores),
           "kind": "oracle", "seconds": round(el, 2),
           "sample": f"{pairs} (b,h) pairs x {w.n} context tokens, loops {list(loops or w.loops)}, "
                     f"float64 NumPy with BLAS threads = {cores} (the process's CPU affinity "
                     f"set); bytes scaled as the GPU path's algorithmic bytes per pair"}
    if one_thread:
        p1, e1 = _oracle_pairs(w, seconds * (1.0 - share), loops, d_rope, 1)
        out["value_1thread"] = p1 * per_pair / e1 / 1e9
        out["sample_1thread"] = f"{p1} (b,h) pairs, BLAS threads = 1"
    return out


def tflops_peak():
    """Measured dense bf16 tensor throughput (TFLOP/s): the sustained figure, for a
    kernel timed inside a long step, and the source of the number."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        if "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured sustained cuBLAS bf16"
        return float(d["bf16_tflops"]), "measured burst cuBLAS bf16"
    return 1400.0, "fallback sustained bf16"


def decode_flops(w, n_ctx: int) -> int:
    """Algorithmic FLOPs of one decode call: the loop-t K rebuild (2 r_k d per
    token-head, unavoidable under full RoPE) and the latent V sum (2 r_v)."""
    return w.B * n_ctx * w.H * 2 * (w.r_k * w.d + w.r_v)


def init_dist():
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    if dist_on:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    return world, rank, local, dist_on


def measure(lla, w, args, device, world, rank, local, dist_on, steps, warmup, path="latent",
            d_rope=0, evict_arg="", eager=False, with_e2e=False):
    """Time `steps` steps of workload w (after `warmup`), max over ranks.  Returns the
    record of the workload (the JSON line's fields apart from the run metadata)."""
    import torch

    st = build_state(w, device, d_rope)
    n_ctx = w.n
    evict = None
    if evict_arg:
        evict = tuple(int(v) for v in evict_arg.split(","))
        n_ctx = apply_eviction(lla, w, st, *evict)
    full = path == "full"
    rebuild_once_ms = None
    if full:
        if evict:
            raise SystemExit("--path full does not combine with --evict")
        rebuild_once_ms = build_full(lla, w, st, device)
        st["full_path"] = True
    dec_bytes = full_decode_bytes if full else decode_bytes
    l2_note = (f"inputs larger than L2 ({dec_bytes(w, n_ctx) * w.layers / 1e6:.0f} MB "
               f"of {'full K/V' if full else 'latents'} per loop pass)")
    if dec_bytes(w, n_ctx) * w.layers < 256e6:
        st["flush"] = torch.zeros(96 * 2**20, dtype=torch.int32, device=device)   # 384 MB
        l2_note = ("L2 flushed each step by a 384 MB write (inside the step time; the "
                   "decode call times exclude it)")
    for _ in range(max(warmup, 3)):
        run_step(lla, w, st)
    barrier_sync(dist_on)
    # the clock sampler starts before more warm-up steps, so its first samples
    # exist by the time the timed region begins (all ranks take the same steps)
    clocks = ClockSampler(local) if rank == 0 else None
    t_w = time.time()
    while True:
        run_step(lla, w, st)
        torch.cuda.synchronize()
        done = 1.0 if (clocks is None or clocks.lines() >= 2 or time.time() - t_w > 5.0) else 0.0
        done = over_ranks([done], "min", device, dist_on)[0]
        if done:
            break

    ev_pairs = ([], [], [], [])
    graphs = None if eager else capture_step_graphs(lla, w, st)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier_sync(dist_on)
    if clocks:
        clocks.mark_start()
    start.record()
    for _ in range(steps):
        if graphs:
            replay_step_graphs(st, graphs, ev_pairs, len(w.loops) * w.layers, w.layers)
        else:
            run_step(lla, w, st, ev_pairs)
    stop.record()
    barrier_sync(dist_on)
    if clocks:
        clocks.mark_stop()
    ms = start.elapsed_time(stop)
    clk = clocks.stop() if clocks else None
    if graphs:
        # graph replays: per-call times are the graph times over the calls they hold
        dec_ms = [a[0].elapsed_time(b[0]) / a[1] for a, b in zip(ev_pairs[0], ev_pairs[1])]
        enc_ms = [a[0].elapsed_time(b[0]) / a[1] for a, b in zip(ev_pairs[2], ev_pairs[3])]
    else:
        dec_ms = [a.elapsed_time(b) for a, b in zip(ev_pairs[0], ev_pairs[1])]
        enc_ms = [a.elapsed_time(b) for a, b in zip(ev_pairs[2], ev_pairs[3])]
    status = lla.decode_status(st["fws"] if full else st["ws"])
    if status:
        raise RuntimeError(f"decode reported device status bits {status}")
    # the job's time is the slowest rank's
    ms, dec_avg, enc_avg = over_ranks([ms, np.mean(dec_ms), np.mean(enc_ms)], "max", device,
                                      dist_on)

    append_bytes = encode_bytes(w, w.encode_tokens)
    if full:
        append_bytes += len(w.loops) * full_rebuild_bytes(w, st["slot"].numel())
    per_step_bytes = (len(w.loops) * w.layers * dec_bytes(w, n_ctx) + w.layers * append_bytes)
    ms_step = ms / steps
    value = world * per_step_bytes / (ms_step * 1e-3) / 1e9
    ctx_tokens = world * len(w.loops) * w.layers * w.B * n_ctx / (ms_step * 1e-3)
    peak, peak_kind = peaks()
    dec_call = dec_bytes(w, n_ctx)
    dec_gbs = dec_call / (dec_avg * 1e-3) / 1e9
    enc_gbs = append_bytes / (enc_avg * 1e-3) / 1e9
    traffic_table = NCU_TRAFFIC_FULL if full else NCU_TRAFFIC
    traffic = ((NCU_TRAFFIC_DECOUPLED.get((w.name, d_rope)) if d_rope else traffic_table.get(w.name))
               if not (args.encode_tokens or evict_arg or args.batch) else None)
    dkname = ("lla_full_decode_attn (full_decode_kernel [+ combine])" if full
              else "lla_decode_attn (prep + partial kernel [+ combine])")
    dec_roof = {"bound": "hbm", "kernel": dkname, "achieved": round(dec_gbs, 1), "peak": peak,
                "unit": "GB/s", "frac": round(dec_gbs / peak, 4),
                "traffic": traffic if len(w.loops) * w.layers * dec_avg >= w.layers * enc_avg else None,
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "call_us": round(dec_avg * 1e3, 2), "algorithmic_bytes_per_call": dec_call}
    enc_roof = {"bound": "hbm", "kernel": "lla_encode + lla_full_rebuild" if full else "lla_encode",
                "achieved": round(enc_gbs, 1), "peak": peak, "unit": "GB/s",
                "frac": round(enc_gbs / peak, 4),
                "traffic": traffic if len(w.loops) * w.layers * dec_avg < w.layers * enc_avg else None,
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "call_us": round(enc_avg * 1e3, 2), "algorithmic_bytes_per_call": append_bytes,
                "tokens_per_call": w.encode_tokens}
    # the roofline of the kernel that takes most of the step: decode (prep + partial
    # [+ combine] per call) or, for prefill-sized encodes, the encode
    if len(w.loops) * w.layers * dec_avg >= w.layers * enc_avg:
        roof = dict(dec_roof)
    else:
        roof = dict(enc_roof)
    roof["decode_call_us"] = round(dec_avg * 1e3, 2)
    roof["encode_call_us"] = round(enc_avg * 1e3, 2)
    if w.mode == synth.MODE_2D and not full:
        # LLA-2D: sixteen heads share each latent row, so the K rebuild is the tensor
        # pipe's work (about 680 FLOP per latent byte): its bound is the tensor pipe
        tp, tp_kind = tflops_peak()
        fl = decode_flops(w, n_ctx)
        tf = fl / (dec_avg * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dkname, "achieved": round(tf, 2), "peak": tp,
                "unit": "TFLOP/s", "frac": round(tf / tp, 4), "traffic": traffic,
                "peak_source": f"{tp_kind} (MEASURED_PEAKS.json)",
                "algorithmic_flops_per_call": fl, "call_us": round(dec_avg * 1e3, 2),
                "hbm": {k: dec_roof[k] for k in ("achieved", "peak", "unit", "frac",
                                                 "algorithmic_bytes_per_call")},
                "decode_call_us": round(dec_avg * 1e3, 2),
                "encode_call_us": round(enc_avg * 1e3, 2)}

    if full:
        launches_per_step = (len(w.loops) * w.layers
                             * lla.full_decode_launches(st["cfg"], w.B, st["n_cap"])
                             + w.layers * (1 + len(w.loops)))
    else:
        launches_per_step = (len(w.loops) * w.layers
                             * lla.decode_launches(st["cfg"], w.B, st["n_cap"]) + w.layers)
    rec = {
        "value": round(value, 2), "unit": "GB/s", "steps": steps, "warmup": max(warmup, 3),
        "ms_per_step": round(ms_step, 5),
        "config": workload_config(w, world, evict, n_ctx, path, d_rope, eager, l2_note),
        "ctx_tokens_per_s": round(ctx_tokens, 1),
        "decode_steps_per_s": round(world * 1e3 / ms_step, 2),
        "roofline": roof,
        "decode_roofline": dec_roof,
        "encode_roofline": enc_roof,
        "gpu_launches": launches_per_step * steps,
        "clocks": clk,
    }
    if full:
        rec["config"]["full_cache_gib"] = round(
            w.layers * len(w.loops) * 2 * lla.full_kv_bytes(st["cfg"], w.B, st["n_cap"]) / 2**30, 2)
        rec["config"]["rebuild_once_ms_per_layer_loop"] = round(rebuild_once_ms, 3)
    if with_e2e and not full:
        if graphs:
            del graphs
        rec["e2e"] = run_e2e(lla, w, st, args, dist_on, world, n_ctx)
    del st
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def workload_config(w, world, evict=None, n_ctx=None, path="latent", d_rope=0, eager=False,
                    l2_note=None):
    """The JSON line's `config`: the workload by name and sizes, and how it ran."""
    return {"workload": w.name, "T": w.T, "H": w.H, "d_head": w.d, "r_k": w.r_k,
            "r_v": w.r_v, "mode": "per_head" if w.mode == synth.MODE_PER_HEAD else "lla_2d",
            "batch": w.B, "context": w.n, "layers": w.layers, "loops": list(w.loops),
            "encode_tokens": w.encode_tokens, "parallelism": f"replicas x{world}",
            "evict": list(evict) if evict else None,
            "attended_context": w.n if n_ctx is None else n_ctx,
            "path": path, "d_rope": d_rope or None,
            "schedule": "eager launches" if eager else "cuda graphs per step",
            "l2": l2_note or (f"inputs larger than L2 ({decode_bytes(w, w.n) * w.layers / 1e6:.0f}"
                              f" MB of latents per loop pass)")}


def sub_record_steps(w):
    """Timed steps of a sub-record: about two seconds of GPU time, 5 to 200 steps
    (per-step time from the byte count at roughly half the copy bandwidth)."""
    peak, _ = peaks()
    est = (len(w.loops) * w.layers * decode_bytes(w, w.n) + w.layers * encode_bytes(
        w, w.encode_tokens)) / (0.5 * peak * 1e9)
    return int(min(200, max(5, 2.0 / max(est, 1e-6))))


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world, rank, local, dist_on = init_dist()
    device = torch.device("cuda", local)
    import looped_transformer_decode_b200 as lla

    w = synth.WORKLOADS[args.workload]
    if args.encode_tokens:
        w = dataclasses.replace(w, encode_tokens=args.encode_tokens)
    if args.batch:
        w = dataclasses.replace(w, B=args.batch, encode_tokens=min(w.encode_tokens, args.batch)
                                if w.encode_tokens <= w.B else w.encode_tokens)
    if args.layers:
        w = dataclasses.replace(w, layers=args.layers)
    rec = measure(lla, w, args, device, world, rank, local, dist_on, args.steps, args.warmup,
                  path=args.path, d_rope=args.d_rope, evict_arg=args.evict, eager=args.eager,
                  with_e2e=not args.no_e2e)
    line = {"metric": METRIC, "value": rec["value"], "unit": "GB/s", "n_gpus": world,
            "steps": rec["steps"], "warmup": rec["warmup"], "ms_per_step": rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; latents drawn in latent space as rank-R plus noise)",
            "config": rec["config"], "ctx_tokens_per_s": rec["ctx_tokens_per_s"],
            "decode_steps_per_s": rec["decode_steps_per_s"], "roofline": rec["roofline"],
            "decode_roofline": rec["decode_roofline"], "encode_roofline": rec["encode_roofline"],
            "gpu_launches": rec["gpu_launches"], "e2e": rec.get("e2e"), "clocks": rec["clocks"]}
    if args.path == "full":
        line["e2e_note"] = "no end-to-end line on the full-memory path"
    if not args.no_sub and args.workload == DEFAULT_WORKLOAD and args.path == "latent" \
            and not (args.d_rope or args.evict or args.encode_tokens or args.batch or args.layers):
        subs = []
        for name in SUB_WORKLOADS:
            sw = synth.WORKLOADS[name]
            r = measure(lla, sw, args, device, world, rank, local, dist_on, sub_record_steps(sw),
                        3, eager=args.eager)
            subs.append({"workload": name, **{k: r[k] for k in (
                "value", "unit", "steps", "ms_per_step", "ctx_tokens_per_s", "decode_steps_per_s",
                "roofline", "decode_roofline", "encode_roofline", "gpu_launches", "clocks")}})
        line["sub_records"] = subs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = (cpu_baseline_full(w, args.cpu_seconds) if args.path == "full"
                                else cpu_baseline_sample(w, args.cpu_seconds,
                                                         d_rope=args.d_rope))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_full(w, seconds: float):
    """Time the float64 oracle's full-memory attention on (b, h) pairs at full context
    (bf16-valued K/V rows drawn at random: the cost does not depend on the values)."""
    import oracle as O

    cores = _oracle_cores()
    g = synth.rng(w.seed + 7)
    K = O.bf16_round(g.standard_normal((w.n, w.d)))
    V = O.bf16_round(g.standard_normal((w.n, w.d)))
    q, ks, vs = (g.standard_normal(w.d) for _ in range(3))
    pairs = 0
    with _blas_limit(cores):
        t0 = time.perf_counter()
        while True:
            O.decode_attention_full(q, ks, vs, K, V, w.n, 10000.0)
            pairs += 1
            el = time.perf_counter() - t0
            if el >= seconds and pairs >= 2:
                break
    per_pair = full_decode_bytes(w, w.n) / (w.B * w.H)
    return {"value": pairs * per_pair / el / 1e9, "unit": "GB/s", "cores": int(cores),
            "kind": "oracle", "seconds": round(el, 2),
            "sample": f"{pairs} (b,h) pairs x {w.n} context tokens, float64 NumPy "
                      f"decode_attention_full; bytes scaled as the GPU path's per pair"}


def run_e2e(lla, w, st, args, dist_on, world, n_ctx):
    """The step end to end through the library's calls, with the latent cache
    resident on the device: every decode call's query and in-flight K/V (per layer
    and loop) and the finished tokens' per-loop rows, slots and new positions are
    copied in from pinned host memory, and every decode output is copied back,
    inside the timed region (eager launches; copies on the compute stream)."""
    import torch

    dev = st["out"].device
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 31)
    shape = (w.B, w.H, w.d)
    n_dec = len(w.loops) * w.layers
    # per (loop, layer): q, k_self, v_self drawn once, pinned
    hq = [[(torch.randn(shape, generator=g) / float(np.sqrt(w.d))).pin_memory(),
           (0.2 * torch.randn(shape, generator=g)).pin_memory(),
           (0.2 * torch.randn(shape, generator=g)).pin_memory()] for _ in range(n_dec)]
    hx = {"xk": st["xk"].cpu().pin_memory(), "xv": st["xv"].cpu().pin_memory(),
          "slot": st["slot"].cpu().pin_memory()}
    hpos = {"q_pos": st["layers"][0]["q_pos"].cpu().pin_memory(),
            "ctx_len": st["layers"][0]["ctx_len"].cpu().pin_memory()}
    outs = [torch.empty(shape, dtype=torch.float32).pin_memory() for _ in range(n_dec)]
    dq = [torch.empty(shape, dtype=torch.float32, device=dev) for _ in range(3)]
    h2d = (sum(t.numel() * t.element_size() for trip in hq for t in trip)
           + sum(v.numel() * v.element_size() for v in hx.values())
           + w.layers * sum(v.numel() * v.element_size() for v in hpos.values()))
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def step():
        for L in st["layers"]:                      # the new positions of this step
            L["q_pos"].copy_(hpos["q_pos"], non_blocking=True)
            L["ctx_len"].copy_(hpos["ctx_len"], non_blocking=True)
        i = 0
        for t in w.loops:
            for L in st["layers"]:
                for dst, src in zip(dq, hq[i]):
                    dst.copy_(src, non_blocking=True)
                lla.decode_attn(st["cfg"], L["packed"], st["rope"], t, L["ctx_len"], dq[0], dq[1],
                                dq[2], L["positions"], L["q_pos"], L["c_k"], L["c_v"],
                                out=st["out"], ws=st["ws"])
                outs[i].copy_(st["out"], non_blocking=True)
                i += 1
        st["xk"].copy_(hx["xk"], non_blocking=True)
        st["xv"].copy_(hx["xv"], non_blocking=True)
        st["slot"].copy_(hx["slot"], non_blocking=True)
        for L in st["layers"]:
            lla.encode(st["cfg"], L["packed"], st["xk"], st["xv"], st["slot"], L["c_k"], L["c_v"])
        torch.cuda.current_stream().synchronize()

    for _ in range(2):
        step()
    steps = max(3, min(args.steps, 10))
    barrier_sync(dist_on)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    barrier_sync(dist_on)
    ms = s.elapsed_time(e) / steps
    ms = over_ranks([ms], "max", dev, dist_on)[0]
    per_step_bytes = (len(w.loops) * w.layers * decode_bytes(w, n_ctx)
                      + w.layers * encode_bytes(w, w.encode_tokens))
    return {"value": round(world * per_step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "inputs": "per decode call: q, k_self, v_self; per step: the finished tokens' "
                      "per-loop K/V rows, their cache slots, q_pos and ctx_len; outputs: every "
                      "decode call's [B, H, d]; latent cache resident in HBM"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    # each step a bounded sample, so that the whole run stays near two minutes
    per_step = min(max(0.05, args.cpu_seconds / 4), 120.0 / max(1, args.steps))
    vals = []
    _oracle_inputs(w)                 # the inputs are drawn once, outside the timed steps
    for _ in range(args.warmup):
        cpu_baseline_sample(w, per_step / 4, one_thread=False)
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline_sample(w, per_step, one_thread=False)
        vals.append(last["value"])
    el = time.perf_counter() - t0
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"kind": "oracle", "cores": last["cores"], "value": round(value, 4),
                         "unit": "GB/s", "sample": last["sample"] + f"; {per_step:.1f} s per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
