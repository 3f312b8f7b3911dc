"""Benchmark: the Focus-dLLM sparse denoising step on B200.

Default workload (synthetic, LLaDA-8B-shaped attention): B=1, L=32768 (prompt 32512,
current block 32), MHA 32 x 128, 32 layers, l_dense=2 (sinks found at layer 2, reused in
layers 3..31), n(t)=4, rho=4, w=8, block size 64, C=64, S=32. A step = PCGI select +
active-row gather + 3 dense layers (+ sink column sums, sink top-S) + 29 x (block
relevance/top-C + sparse attention), replayed as one CUDA graph. The block means are
refreshed at block entry (timed separately, with the dense full refresh).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config full32k|llada8k|dream16k|sweep|all]

Prints one JSON line on rank 0 for a step workload (full32k is the default; llada8k is
the 8K LLaDA-shaped step, dream16k the 16K Dream-shaped GQA 28q/4kv step). `--config
sweep` prints one line per sweep point (B=4 at 32K, block size x C x rho; one sparse
layer each, against the dense kernel on the same active queries); `all` runs everything.
`--impl reference` times the fp64 CPU oracle on the host cores on a bounded sample of
the same step.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_long_context_b200 import configs, inputs  # noqa: E402

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the step's
# dominant kernel on the 32K workload, from the committed ncu summaries: the fused sparse
# layer (default step) and the unfused sparse attention. Each is reset to None whenever
# its kernel changes, until it is captured again; other workloads report None.
TRAFFIC_BYTES = {"fused": 78.27e6, "sparse": 69.61e6}
METRIC = "sparse dLLM attn step latency & active tok/s at 32K ctx; % of HBM/TC roofline"
WORKLOADS = {"full32k": configs.FULL_32K, "llada8k": configs.LLADA_8K, "dream16k": configs.DREAM_16K}
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- utils
def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(ms: float, ws: int, device) -> float:
    """The largest of the ranks' elapsed times: the job ends with its slowest rank."""
    if ws <= 1:
        return ms
    tt = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
    return float(tt.item())


def whole_job_rate(ws: int, n_active: int, ms_per_step: float) -> float:
    """Active tokens per second over all ranks (each rank runs its own replica)."""
    return ws * n_active / (ms_per_step * 1e-3)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """NVML sampling of SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, local_index: int, period_s: float = 0.005):
        self.ok = False
        self.samples, self.reasons = [], set()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
            if vis and local_index < len(vis):
                ident = vis[local_index]
                self.h = (pynvml.nvmlDeviceGetHandleByIndex(int(ident)) if ident.isdigit()
                          else pynvml.nvmlDeviceGetHandleByUUID(ident))
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(local_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _loop(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._loop, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def key_set_sizes(cfg, sinks, blocks_by_layer):
    """|I_p| summed over (b, kv head) for each sparse layer, from the step's index sets."""
    sinks = sinks.cpu().numpy()
    sizes = {}
    for l, blk_t in blocks_by_layer.items():
        blocks = blk_t.cpu().numpy()
        tot = 0
        for b in range(cfg.B):
            for h in range(cfg.Hkv):
                keys = set(range(cfg.g0, cfg.g1))
                for blk in blocks[b, h]:
                    if blk >= 0:
                        keys.update(range(blk * cfg.bs, min(cfg.P, (blk + 1) * cfg.bs)))
                keys.update(int(j) for j in sinks[b, h] if j >= 0)
                tot += len(keys)
        sizes[l] = tot
    return sizes


def call_work(cfg, n_act, ip_sum=None):
    """Algorithmic bytes and FLOPs of one call (the method's work, not the kernels').

    dense:  K+V of all L keys + Q + O of the active rows; 4 * n_act * Hq * L * d FLOPs
            (n_act = active queries summed over the batch).
    sparse: gathered K+V of I_p (ip_sum = |I_p| summed over (b, kv head)) + kbar + Q + O +
            the kept-block list; 4 * (n_act / B) * g * ip_sum * d FLOPs for QK^T and PV
            (exact when every sequence has the same number of active queries, as here),
            plus 2 * n_act * Hq * nb * d for the relevance scores.
    """
    c = cfg
    g = c.Hq // c.Hkv
    qo = 2 * n_act * c.Hq * c.d * 2
    if ip_sum is None:
        return (c.B * c.Hkv * c.L * c.d * 2 * 2 + qo, 4.0 * n_act * c.Hq * c.L * c.d)
    A = n_act / c.B
    kbar = c.B * c.Hkv * c.nb * c.d * 4
    blk = c.B * c.Hkv * c.C * 4
    return (ip_sum * c.d * 2 * 2 + kbar + blk + qo, 4.0 * A * g * ip_sum * c.d + 2.0 * n_act * c.Hq * c.nb * c.d)


def roof_ms(nbytes, flops, hbm_gbs, tc_tflops):
    """Roofline time of one call: the slower of its bytes at HBM peak and its FLOPs at the
    tensor peak."""
    return max(nbytes / (hbm_gbs * 1e9), flops / (tc_tflops * 1e12)) * 1e3


def make_flush(device):
    """A buffer twice the L2 size: writing it evicts every line of an earlier call."""
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    return lambda: buf.zero_()


def graph_ms(fns, reps, flush=None):
    """Mean device time of one call of `fns` (in order), each kind captured in one CUDA graph.

    Without `flush`, the graph is replayed `reps` times back to back (the callers rotate
    over distinct layers, so no layer's K/V stays in L2). With `flush`, L2 is overwritten
    before every replay and each replay is timed on its own."""
    gs = torch.cuda.Stream()
    gs.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(gs):
        for f in fns:
            f()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=gs):
            for f in fns:
                f()
        for _ in range(2):
            g.replay()
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(gs)
            for _ in range(reps):
                g.replay()
            e1.record(gs)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / (reps * len(fns))
        else:
            evs = []
            for _ in range(reps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(gs)
                g.replay()
                e1.record(gs)
                evs.append((e0, e1))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in evs) / len(fns)
    del g
    return ms


# ----------------------------------------------------------------------------- data
def build_replica(cfg, device, seed_offset=0):
    c = cfg.replace(seed=cfg.seed + seed_offset) if seed_offset else cfg
    st = inputs.step_state(c)
    Q_full = torch.empty((c.n_layers, c.B, c.Hq, c.L, c.d), dtype=torch.bfloat16, device=device)
    K, V = [], []
    for l in range(c.n_layers):
        q, k, v = inputs.make_layer(c, l, device, st.sink_pos)
        Q_full[l].copy_(q)
        K.append(k)
        V.append(v)
        del q
    torch.cuda.synchronize()
    return c, st, Q_full, K, V


# ----------------------------------------------------------------------------- oracle leg
def oracle_sample(cfg, st, layer_data, kbar_sparse):
    """Time the oracle on select + the sink layer (dense + colsum + top-S) + one sparse layer.

    layer_data = {"dense": (Q, K, V) of layer l_dense, "sparse": (Q, K, V) of layer l_dense+1}
    as float64 arrays; kbar_sparse = oracle block means of that sparse layer (block entry).
    Returns (seconds per extrapolated full step, n_active, details).
    """
    from oracle import focus_oracle as orc
    rho = float(np.float32(cfg.rho))
    scale = float(np.float32(1 / math.sqrt(cfg.d)))
    t0 = time.perf_counter()
    _, active = orc.select_queries(st.conf_prev, st.mask, cfg.g0, cfg.g1, cfg.n_t, rho, cfg.w)
    t_sel = time.perf_counter() - t0
    nA = [a.size for a in active]
    Qd, Kd, Vd = layer_data["dense"]
    t0 = time.perf_counter()
    Qa = orc.gather_rows(Qd, active, cfg.acap)
    _, colsum, _ = orc.dense_attention(Qa, nA, Kd, Vd, scale, want_colsum=True)
    sinks = orc.sink_identify(colsum, cfg.S)
    t_dense = time.perf_counter() - t0
    Qs, Ks, Vs = layer_data["sparse"]
    t0 = time.perf_counter()
    Qa = orc.gather_rows(Qs, active, cfg.acap)
    blocks, _ = orc.block_select(Qa, nA, kbar_sparse, cfg.C)
    orc.sparse_attention(Qa, nA, Ks, Vs, sinks, blocks, cfg.bs, cfg.P, cfg.g0, cfg.g1, scale)
    t_sparse = time.perf_counter() - t0
    n_dense = len(cfg.dense_layers)
    n_sparse = cfg.n_layers - n_dense
    t_step = t_sel + n_dense * t_dense + n_sparse * t_sparse
    return t_step, sum(nA), {"select_s": t_sel, "dense_layer_s": t_dense, "sparse_layer_s": t_sparse}


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_inputs(cfg, st, device):
    """float64 host copies of layers l_dense and l_dense+1 (generated on `device`)."""
    ld = cfg.l_dense
    dense = tuple(inputs.to_f64(t) for t in inputs.make_layer(cfg, ld, device, st.sink_pos))
    sparse = tuple(inputs.to_f64(t) for t in inputs.make_layer(cfg, ld + 1, device, st.sink_pos))
    from oracle import focus_oracle as orc
    kbar = orc.block_means(sparse[1], cfg.P, cfg.bs)
    return {"dense": dense, "sparse": sparse}, kbar


def _config_dict(c, n_act=None, **extra):
    d = {"workload": c.name, "B": c.B, "L": c.L, "P": c.P, "G": c.G, "Hq": c.Hq, "Hkv": c.Hkv, "d": c.d,
         "layers": c.n_layers, "l_dense": c.l_dense, "n_t": c.n_t, "rho": c.rho, "w": c.w, "bs": c.bs, "C": c.C,
         "S": c.S}
    if n_act is not None:
        d["n_active"] = n_act
    d.update(extra)
    return d


def run_reference(args):
    ws, rank, local = _dist()
    if rank != 0:
        return 0
    cfg = WORKLOADS.get(args.config, configs.FULL_32K)
    st = inputs.step_state(cfg)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    data, kbar = oracle_inputs(cfg, st, dev)
    per_step = []
    n_act = 0
    for i in range(args.warmup + args.steps):
        t_step, n_act, det = oracle_sample(cfg, st, data, kbar)
        if i >= args.warmup:
            per_step.append(t_step)
    t = float(np.mean(per_step))
    value = n_act / t
    cores = _oracle_threads()
    n_dense = len(cfg.dense_layers)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "active tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config_dict(cfg),
        "cpu_baseline": {"value": value, "unit": "active tok/s", "cores": cores, "kind": "oracle",
                         "sample": "oracle (numpy fp64) on select + sink layer (dense+colsum+top-S) + one sparse "
                                   f"layer per step, extrapolated to {n_dense} dense + "
                                   f"{cfg.n_layers - n_dense} sparse layers"},
        "e2e": {"value": value, "unit": "active tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our leg
def run_step_workload(cfg0, args, ws, rank, local, dev, F):
    """One JSON line for a full denoising step of `cfg0` (one replica per rank)."""
    from diffusion_long_context_b200.step import SparseStep

    cfg, st, Q_full, K, V = build_replica(cfg0, dev, seed_offset=rank)
    step = SparseStep(cfg, Q_full, K, V, device=dev, fused=not args.unfused)
    step.set_state(torch.from_numpy(st.conf_prev), torch.from_numpy(st.mask), non_blocking=False)
    c = cfg
    # K/V bytes one step reads: dense layers whole, sparse layers their kept share (below)
    kv_layer = c.B * c.Hkv * c.L * c.d * 2 * 2

    # ---- block entry: block means of the sparse layers (timed once, after a warm run)
    step.block_entry()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    step.block_entry()
    e1.record()
    torch.cuda.synchronize()
    block_means_ms = e0.elapsed_time(e1)

    # ---- graph capture of the sparse step
    step.capture()
    for _ in range(max(3, args.warmup)):
        step.replay()
    torch.cuda.synchronize()
    n_act = int(step.n_active.sum().item())
    ip_sizes = key_set_sizes(c, step.sinks, step.blocks)
    mean_ip = float(np.mean(list(ip_sizes.values()))) if ip_sizes else 0.0
    n_dense = len(step.dense_layers)
    n_sparse = len(step.sparse_layers)
    step_read = n_dense * kv_layer + n_sparse * mean_ip * c.d * 4
    # the step's inputs exceed L2 by far at 8K and 32K; at smaller footprints L2 is
    # overwritten before every timed step
    flush = make_flush(dev) if step_read < 4 * L2_BYTES else None

    def barrier():
        if ws > 1:
            torch.distributed.barrier(device_ids=[local])
        torch.cuda.synchronize()

    sampler = ClockSampler(local)
    with sampler:
        t_pre = time.perf_counter()
        while time.perf_counter() - t_pre < 0.3:
            step.replay()
        barrier()
        if flush is None:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(args.steps):
                step.replay()
            t1.record()
            barrier()
            ms_total = t0.elapsed_time(t1)
        else:
            evs = []
            for _ in range(args.steps):
                flush()
                t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                t0.record()
                step.replay()
                t1.record()
                evs.append((t0, t1))
            barrier()
            ms_total = sum(a.elapsed_time(b) for a, b in evs)
    ms_total = max_over_ranks(ms_total, ws, dev)
    ms_step = ms_total / args.steps
    value = whole_job_rate(ws, n_act, ms_step)
    gpu_launches = step.launches_per_step * args.steps

    # ---- per-call durations: each call kind of the step captured in its own CUDA graph
    # (one replay = that call for every layer of the step, so layers rotate and no layer's
    # K/V stays in L2), timed with CUDA events on the replay stream
    reps = max(3, min(args.steps, 20))
    dense_plain = [l for l in step.dense_layers if l != c.l_dense]
    call_ms = {
        "select_and_gather": graph_ms([step.select], reps, flush),
        "dense_attention": (graph_ms([lambda l=l: step.dense_layer(l) for l in dense_plain], reps, flush)
                            if dense_plain else None),
        "dense_attention_colsum_sinks": graph_ms([lambda: step.dense_layer(c.l_dense)], reps, flush),
        "sparse_layer_fused": graph_ms([lambda l=l: step.sparse_layer_fused(l) for l in step.sparse_layers], reps,
                                       flush),
        "block_select": graph_ms([lambda l=l: step.block_select_layer(l) for l in step.sparse_layers], reps, flush),
        "sparse_attention": graph_ms([lambda l=l: step.sparse_attention_layer(l) for l in step.sparse_layers], reps,
                                     flush),
    }

    # ---- roofline of the dominant call: the sparse layer
    hbm, tc, tc_sus, peak_kind = _peaks()
    A = n_act / c.B
    g = c.Hq // c.Hkv
    sp_bytes, sp_flops = call_work(c, n_act, mean_ip)
    dn_bytes, dn_flops = call_work(c, n_act)
    att_bytes = mean_ip * c.d * 2 * 2 + 2 * n_act * c.Hq * c.d * 2
    att_flops = 4.0 * A * g * mean_ip * c.d
    if step.fused:
        dom_kind, dom_bytes, dom_flops, dom_call = "fused", sp_bytes, sp_flops, "sparse_layer_fused"
        dom_name = ("focus_sparse_attention_fused (block relevance + top-C + sparse attention in one launch), one "
                    "layer; CUDA-graph replay of all sparse layers")
    else:
        dom_kind, dom_bytes, dom_flops, dom_call = "sparse", att_bytes, att_flops, "sparse_attention"
        dom_name = "focus_sparse_attention, one layer; CUDA-graph replay of all sparse layers"
    t_dom = call_ms[dom_call] * 1e-3
    dom_bound = "hbm" if dom_bytes / (hbm * 1e9) >= dom_flops / (tc * 1e12) else "tensor"
    achieved_gbs = dom_bytes / t_dom / 1e9
    achieved_tf = dom_flops / t_dom / 1e12
    if dom_bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s", "frac": achieved_gbs / hbm}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": tc, "unit": "TFLOP/s", "frac": achieved_tf / tc}
    roof.update({"traffic": TRAFFIC_BYTES[dom_kind] if c.name == configs.FULL_32K.name else None,
                 "kernel": dom_name, "bytes_per_launch": dom_bytes, "flops_per_launch": dom_flops,
                 "achieved_gbs": achieved_gbs, "achieved_tflops": achieved_tf, "launch_ms": call_ms[dom_call],
                 "peak_source": f"{peak_kind} hbm_gbs / bf16_tflops (burst)"})

    # ---- step roofline: per call the slower of bytes at HBM peak and FLOPs at the
    # sustained tensor peak, summed over the calls of the method (no re-read of the sink
    # layer's K for the column sums: the method's bytes only)
    colsum_io = 2 * c.B * c.Hkv * c.L * 4                 # colsum written by the sink layer, read by top-S
    step_calls = [(dn_bytes, dn_flops)] * n_dense + [(colsum_io, 0.0)] + [(sp_bytes, sp_flops)] * n_sparse
    step_bytes = sum(b for b, _ in step_calls)
    step_flops = sum(f for _, f in step_calls)
    step_roof = sum(roof_ms(b, f, hbm, tc_sus) for b, f in step_calls)

    # ---- dense comparator: the same kernel on the same active queries of every sparse
    # layer, over all L keys (graph replay, as above)
    Od = torch.empty_like(step.O_active[step.sparse_layers[0]])
    dense_cmp_ms = graph_ms([lambda l=l: F.focus_dense_attention(step.Q_active[l], step.n_active, step.K[l],
                                                                 step.V[l], Od, ws=step.ws)
                             for l in step.sparse_layers], reps, flush)
    kept_ratio = mean_ip / (c.B * c.Hkv * c.L)

    # ---- block entry: the full refresh of a sparse layer (all L queries over all L keys), with
    # the layer's block means summed from the same K stream (focus_full_refresh)
    refresh = None
    if not args.skip_refresh:
        O_full = torch.empty((c.B, c.Hq, c.L, c.d), dtype=torch.bfloat16, device=dev)
        step.full_refresh_layer(step.sparse_layers[0], O_full)
        torch.cuda.synchronize()
        times = []
        for r in range(3):
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record()
            step.full_refresh_layer(step.sparse_layers[1 + r % (len(step.sparse_layers) - 1)], O_full)
            r1.record()
            torch.cuda.synchronize()
            times.append(r0.elapsed_time(r1))
        del O_full
        refresh_ms = statistics.median(times)
        refresh_flops = 4.0 * c.B * c.Hq * c.L * c.L * c.d
        refresh = {"ms_per_layer": refresh_ms, "tflops": refresh_flops / (refresh_ms * 1e-3) / 1e12,
                   "frac_of_bf16_burst": refresh_flops / (refresh_ms * 1e-3) / 1e12 / tc,
                   "step_ms_est": refresh_ms * c.n_layers, "with_block_means": True,
                   "timed": "median of 3 single launches (sparse layers: attention + block means)"}

    # ---- end to end through the public API: pinned host state in, last layer's output out
    conf_h = torch.from_numpy(st.conf_prev).pin_memory()
    mask_h = torch.from_numpy(st.mask).pin_memory()
    out_h = torch.empty(step.O_active[-1].shape, dtype=torch.bfloat16).pin_memory()
    act_h = torch.empty(step.i_active.shape, dtype=torch.int32).pin_memory()
    nact_h = torch.empty(step.n_active.shape, dtype=torch.int32).pin_memory()
    # one graph per step holds the copies in, the step and the copies out; the host waits
    # for every step's result before it launches the next
    step.capture_io(conf_h, mask_h, [(out_h, step.O_active[-1]), (act_h, step.i_active), (nact_h, step.n_active)])
    for _ in range(3):
        step.replay_io()
        torch.cuda.current_stream().synchronize()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record()
    for _ in range(args.steps):
        step.replay_io()
        torch.cuda.current_stream().synchronize()
    x1.record()
    barrier()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), ws, dev)
    e2e_value = whole_job_rate(ws, n_act, e2e_ms / args.steps)
    h2d = conf_h.numel() * 4 + mask_h.numel()
    d2h = out_h.numel() * 2 + act_h.numel() * 4 + nact_h.numel() * 4

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu_baseline = None
    if ws == 1 and not args.skip_cpu:
        data, kbar = oracle_inputs(c, st, dev)
        t_step, n_o, det = oracle_sample(c, st, data, kbar)
        cpu_baseline = {"value": n_o / t_step, "unit": "active tok/s", "cores": _oracle_threads(),
                        "kind": "oracle",
                        "sample": "numpy fp64 oracle on select + the sink layer (dense + colsum + top-S) + one "
                                  f"sparse layer, extrapolated to {n_dense} dense + {n_sparse} sparse layers; "
                                  f"dense {det['dense_layer_s']:.2f} s, sparse {det['sparse_layer_s']:.3f} s"}
        del data, kbar
    err = F.device_error()

    line = {
        "metric": METRIC, "value": value, "unit": "active tok/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config_dict(
            c, n_act,
            l2=("inputs larger than L2: every layer distinct, %.2f GB of K/V read per step" % (step_read / 1e9)
                if flush is None else "L2 overwritten (252 MB write) before every timed step"),
            replay="one CUDA graph per step",
            sparse_layer="fused relevance/top-C + attention" if step.fused else "two calls",
            parallelism=f"replicas x{ws}"),
        "roofline": roof,
        "step_roofline": {"bytes": step_bytes, "flops": step_flops, "roofline_ms": step_roof,
                          "frac": step_roof / ms_step, "effective_tflops": step_flops / (ms_step * 1e-3) / 1e12,
                          "achieved_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
                          "basis": "per call max(method bytes / hbm_gbs, FLOPs / bf16_tflops_sustained), "
                                   "summed; sink column sums counted as written + read once, not as a "
                                   "second K pass"},
        "calls_ms": call_ms,
        "calls_timing": ("per call kind: a CUDA graph of that call over every layer of the step, replayed "
                         + ("back to back" if flush is None else "after an L2 overwrite each time")),
        "dense_comparator": {"ms": dense_cmp_ms, "kept_kv_ratio": kept_ratio,
                             "sparse_over_dense": call_ms["sparse_attention"] / dense_cmp_ms,
                             "fused_over_dense": call_ms["sparse_layer_fused"] / dense_cmp_ms},
        "block_entry": {"full_refresh": refresh,
                        "block_means_standalone_ms_all_sparse_layers": block_means_ms,
                        "block_means_note": "standalone pass, for reference: at block entry the means come "
                                            "out of the full refresh's K stream"},
        "e2e": {"value": e2e_value, "unit": "active tok/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
        "cpu_baseline": cpu_baseline,
        "clocks": sampler.summary(),
        "gpu_launches": gpu_launches,
        "device_error": err,
    }
    step.release()
    del step, Q_full, K, V
    torch.cuda.empty_cache()
    return line


def run_sweep_point(cfg0, args, dev, F, flush):
    """One sweep point: B=4 at 32K, layer 0 dense (yields the sinks), layer 1 sparse.

    The sparse layer (fused relevance/top-C + attention, as in the step) is timed against
    the dense kernel on the same active queries over all L keys, each after an L2
    overwrite."""
    from diffusion_long_context_b200.step import SparseStep

    cfg = cfg0.replace(n_layers=2, l_dense=0)
    cfg, st, Q_full, K, V = build_replica(cfg, dev)
    step = SparseStep(cfg, Q_full, K, V, device=dev, fused=True)
    step.set_state(torch.from_numpy(st.conf_prev), torch.from_numpy(st.mask), non_blocking=False)
    step.block_entry()
    step.run()
    torch.cuda.synchronize()
    c = cfg
    n_act = int(step.n_active.sum().item())
    reps = max(5, min(args.steps, 20))
    ms_fused = graph_ms([lambda: step.sparse_layer_fused(1)], reps, flush)
    ms_select = graph_ms([step.select], reps, flush)
    ms_two = graph_ms([lambda: step.block_select_layer(1), lambda: step.sparse_attention_layer(1)], reps, flush) * 2
    Od = torch.empty_like(step.O_active[1])
    ms_dense = graph_ms([lambda: F.focus_dense_attention(step.Q_active[1], step.n_active, step.K[1], step.V[1], Od,
                                                         ws=step.ws)], reps, flush)
    ip = key_set_sizes(c, step.sinks, {1: step.blocks[1]})[1]
    hbm, tc, _, peak_kind = _peaks()
    sp_bytes, sp_flops = call_work(c, n_act, ip)
    dn_bytes, dn_flops = call_work(c, n_act)
    sp_roof = roof_ms(sp_bytes, sp_flops, hbm, tc)
    dn_roof = roof_ms(dn_bytes, dn_flops, hbm, tc)
    err = F.device_error()
    pt = {
        "metric": "sparse layer latency per sweep point vs dense; % of HBM/TC roofline",
        "value": n_act / (ms_fused * 1e-3), "unit": "active tok/s (one sparse layer)",
        "ms_sparse_layer": ms_fused, "dtype": "bf16", "data": "synthetic",
        "config": _config_dict(c, n_act, l2="L2 overwritten (252 MB write) before every timed launch"),
        "sparse_layer": {"ms": ms_fused, "bytes": sp_bytes, "flops": sp_flops, "roofline_ms": sp_roof,
                         "frac": sp_roof / ms_fused, "achieved_gbs": sp_bytes / (ms_fused * 1e-3) / 1e9,
                         "effective_tflops": sp_flops / (ms_fused * 1e-3) / 1e12,
                         "two_call_ms": ms_two},
        "select_and_gather_ms": ms_select,
        "dense_comparator": {"ms": ms_dense, "bytes": dn_bytes, "roofline_ms": dn_roof, "frac": dn_roof / ms_dense,
                             "kept_kv_ratio": ip / (c.B * c.Hkv * c.L), "sparse_over_dense": ms_fused / ms_dense},
        "peak_source": f"{peak_kind} hbm_gbs / bf16_tflops (burst)",
        "device_error": err,
    }
    step.release()
    del step, Q_full, K, V
    torch.cuda.empty_cache()
    return pt


def run_ours(args):
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    from diffusion_long_context_b200 import focus as F

    names = list(WORKLOADS) + ["sweep"] if args.config == "all" else [args.config]
    for name in names:
        if name == "sweep":
            if ws > 1:
                continue                      # the sweep is a single-GPU table
            flush = make_flush(dev)
            for p in configs.sweep_points():
                line = run_sweep_point(p, args, dev, F, flush)
                print(json.dumps(line), flush=True)
            continue
        line = run_step_workload(WORKLOADS[name], args, ws, rank, local, dev, F)
        if rank == 0:
            print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier(device_ids=[local])
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=list(WORKLOADS) + ["sweep", "all"], default="full32k")
    ap.add_argument("--skip-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--skip-refresh", action="store_true", help="skip the full-refresh comparator")
    ap.add_argument("--unfused", action="store_true",
                    help="run block select and sparse attention as two launches per sparse layer")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
