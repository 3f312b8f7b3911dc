"""Benchmark: one Focus-dLLM sparse denoising step at 32K context on B200.

Workload (synthetic, LLaDA-8B-shaped attention): B=1, L=32768 (prompt 32512, current
block 32), MHA 32 x 128, 32 layers, l_dense=2 (sinks found at layer 2, reused in
layers 3..31), n(t)=4, rho=4, w=8, block size 64, C=64, S=32. A step = PCGI select +
active-row gather + 3 dense layers (+ sink column sums, sink top-S) + 29 x (block
relevance/top-C + sparse attention), replayed as one CUDA graph. The block means are
refreshed at block entry (timed separately, with the dense full refresh).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0. `--impl reference` times the fp64 CPU oracle on the
host cores on a bounded sample of the same step.
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
# dominant kernel on this workload, from the committed ncu summaries: the fused sparse
# layer (default step) and the unfused sparse attention. Each is reset to None whenever
# its kernel changes, until it is captured again.
TRAFFIC_BYTES = {"fused": 78.79e6, "sparse": 69.77e6}
METRIC = "sparse dLLM attn step latency & active tok/s at 32K ctx; % of HBM/TC roofline"
CFG = configs.FULL_32K


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


def _ev_ms(pairs):
    return [s.elapsed_time(e) for s, e in pairs]


def _key_set_sizes(step):
    """|I_p| per (b, h) for every sparse layer, from the index sets of the last step."""
    c = step.cfg
    sinks = step.sinks.cpu().numpy()
    sizes = {}
    for l in step.sparse_layers:
        blocks = step.blocks[l].cpu().numpy()
        tot = 0
        for b in range(c.B):
            for h in range(c.Hkv):
                keys = set(range(c.g0, c.g1))
                for blk in blocks[b, h]:
                    if blk >= 0:
                        keys.update(range(blk * c.bs, min(c.P, (blk + 1) * c.bs)))
                keys.update(int(j) for j in sinks[b, h] if j >= 0)
                tot += len(keys)
        sizes[l] = tot
    return sizes


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
    n_dense = cfg.l_dense + 1
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


def run_reference(args):
    ws, rank, local = _dist()
    if rank != 0:
        return 0
    cfg = CFG
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
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "active tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "L": cfg.L, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                   "layers": cfg.n_layers, "l_dense": cfg.l_dense, "bs": cfg.bs, "C": cfg.C, "S": cfg.S},
        "cpu_baseline": {"value": value, "unit": "active tok/s", "cores": cores, "kind": "oracle",
                         "sample": "oracle (numpy fp64) on select + sink layer (dense+colsum+top-S) + one sparse "
                                   "layer per step, extrapolated to 3 dense + 29 sparse layers"},
        "e2e": {"value": value, "unit": "active tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our leg
def run_ours(args):
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    from diffusion_long_context_b200 import focus as F
    from diffusion_long_context_b200.step import SparseStep

    cfg, st, Q_full, K, V = build_replica(CFG, dev, seed_offset=rank)
    step = SparseStep(cfg, Q_full, K, V, device=dev, fused=not args.unfused)
    step.set_state(torch.from_numpy(st.conf_prev), torch.from_numpy(st.mask), non_blocking=False)

    # ---- block entry: block means of the 29 sparse layers (timed once, after a warm run)
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

    # sustained pre-load so the clock sampler sees the GPU under this load
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
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(args.steps):
            step.replay()
        t1.record()
        barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1), ws, dev)
    ms_step = ms_total / args.steps
    n_act = int(step.n_active.sum().item())
    value = whole_job_rate(ws, n_act, ms_step)
    gpu_launches = step.launches_per_step * args.steps

    # ---- per-call durations: each call kind of the step captured in its own CUDA graph
    # (one replay = that call for every layer of the step, so layers rotate and no layer's
    # K/V stays in L2), timed with CUDA events on the replay stream
    def graph_ms(fns, reps):
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
            e0_, e1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0_.record(gs)
            for _ in range(reps):
                g.replay()
            e1_.record(gs)
        torch.cuda.synchronize()
        ms = e0_.elapsed_time(e1_) / (reps * len(fns))
        del g
        return ms

    reps = max(3, min(args.steps, 20))
    c = cfg
    call_ms = {
        "select_and_gather": graph_ms([step.select], reps),
        "dense_attention": graph_ms([lambda l=l: step.dense_layer(l) for l in range(c.l_dense)], reps),
        "dense_attention_colsum_sinks": graph_ms([lambda: step.dense_layer(c.l_dense)], reps),
        "sparse_layer_fused": graph_ms([lambda l=l: step.sparse_layer_fused(l) for l in step.sparse_layers], reps),
        "block_select": graph_ms([lambda l=l: step.block_select_layer(l) for l in step.sparse_layers], reps),
        "sparse_attention": graph_ms([lambda l=l: step.sparse_attention_layer(l) for l in step.sparse_layers], reps),
    }

    # ---- roofline of the dominant call: the sparse attention of one layer
    hbm, tc, tc_sus, peak_kind = _peaks()
    ip_sizes = _key_set_sizes(step)
    mean_ip = float(np.mean(list(ip_sizes.values())))            # summed over (b, kv head)
    A = n_act / c.B
    g = c.Hq // c.Hkv
    sparse_bytes = mean_ip * c.d * 2 * 2 + 2 * c.B * c.Hq * A * c.d * 2
    sparse_flops = 4.0 * A * g * mean_ip * c.d
    dense_bytes = c.B * c.Hkv * c.L * c.d * 2 * 2 + 2 * c.B * c.Hq * A * c.d * 2
    kbar_bytes = c.B * c.Hkv * c.nb * c.d * 4
    # the step runs one fused launch per sparse layer (kbar + gathered K/V + Q + O + the
    # kept-block list), or focus_block_select then focus_sparse_attention (the attention
    # launch is reported: gathered K/V + Q + O)
    blocks_bytes = c.B * c.Hkv * c.C * 4
    if step.fused:
        dom_kind, dom_bytes, dom_call = "fused", sparse_bytes + kbar_bytes + blocks_bytes, "sparse_layer_fused"
        dom_name = ("focus_sparse_attention_fused (decode kernel with the relevance/top-C prologue, cluster "
                    "split), one layer; CUDA-graph replay of all sparse layers")
    else:
        dom_kind, dom_bytes, dom_call = "sparse", sparse_bytes, "sparse_attention"
        dom_name = ("focus_sparse_attention (decode kernel, cluster split), one layer; CUDA-graph replay of all "
                    "sparse layers")
    t_sp = call_ms[dom_call] * 1e-3
    achieved = dom_bytes / t_sp / 1e9
    # step roofline: slower of bytes at HBM peak and flops at the tensor peak, summed over calls
    n_dense, n_sparse = c.l_dense + 1, c.n_layers - c.l_dense - 1
    colsum_bytes = c.B * c.Hkv * c.L * c.d * 2
    step_bytes = n_dense * dense_bytes + colsum_bytes + n_sparse * (sparse_bytes + kbar_bytes)
    step_roof_ms = step_bytes / (hbm * 1e9) * 1e3

    # ---- dense comparator: the same kernel on the same active queries of every sparse
    # layer, over all L keys (graph replay, as above)
    Od = torch.empty_like(step.O_active[step.sparse_layers[0]])
    dense_cmp_ms = graph_ms([lambda l=l: F.focus_dense_attention(step.Q_active[l], step.n_active, step.K[l],
                                                                 step.V[l], Od, ws=step.ws)
                             for l in step.sparse_layers], reps)
    kept_ratio = mean_ip / (c.B * c.Hkv * c.L)

    # ---- full refresh (block entry comparator): one layer, all L queries
    refresh_ms = None
    if not args.skip_refresh:
        O_full = torch.empty((c.B, c.Hq, c.L, c.d), dtype=torch.bfloat16, device=dev)
        step.full_refresh_layer(0, O_full)
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record()
        step.full_refresh_layer(1, O_full)
        r1.record()
        torch.cuda.synchronize()
        refresh_ms = r0.elapsed_time(r1)
        del O_full
    refresh_flops = 4.0 * c.B * c.Hq * c.L * c.L * c.d

    # ---- end to end through the public API: pinned host state in, last layer's output out
    conf_h = torch.from_numpy(st.conf_prev).pin_memory()
    mask_h = torch.from_numpy(st.mask).pin_memory()
    out_h = torch.empty(step.O_active[-1].shape, dtype=torch.bfloat16).pin_memory()
    act_h = torch.empty(step.i_active.shape, dtype=torch.int32).pin_memory()
    nact_h = torch.empty(step.n_active.shape, dtype=torch.int32).pin_memory()
    barrier()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record()
    for _ in range(args.steps):
        step.set_state(conf_h, mask_h, non_blocking=True)
        step.replay()
        out_h.copy_(step.O_active[-1], non_blocking=True)
        act_h.copy_(step.i_active, non_blocking=True)
        nact_h.copy_(step.n_active, non_blocking=True)
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
                                  "sparse layer, extrapolated to 3 dense + 29 sparse layers; "
                                  f"dense {det['dense_layer_s']:.2f} s, sparse {det['sparse_layer_s']:.3f} s"}
    err = F.device_error()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "active tok/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": c.name, "B": c.B, "L": c.L, "P": c.P, "G": c.G, "Hq": c.Hq, "Hkv": c.Hkv,
                       "d": c.d, "layers": c.n_layers, "l_dense": c.l_dense, "n_t": c.n_t, "rho": c.rho,
                       "w": c.w, "bs": c.bs, "C": c.C, "S": c.S, "n_active": n_act,
                       "l2": "inputs larger than L2: 17.2 GB of K/V per step, every layer distinct",
                       "replay": "one CUDA graph per step",
                       "sparse_layer": "fused relevance/top-C + attention" if step.fused else "two calls",
                       "parallelism": f"replicas x{ws}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": TRAFFIC_BYTES[dom_kind],
                         "kernel": dom_name, "bytes_per_launch": dom_bytes, "flops_per_launch": sparse_flops,
                         "launch_ms": call_ms[dom_call], "peak_source": f"{peak_kind} hbm_gbs"},
            "step_roofline": {"bytes": step_bytes, "roofline_ms": step_roof_ms, "frac": step_roof_ms / ms_step},
            "calls_ms": call_ms,
            "dense_comparator": {"ms": dense_cmp_ms, "kept_kv_ratio": kept_ratio,
                                 "sparse_over_dense": call_ms["sparse_attention"] / dense_cmp_ms},
            "block_entry": {"block_means_ms_all_sparse_layers": block_means_ms,
                            "full_refresh_ms_per_layer": refresh_ms,
                            "full_refresh_tflops": (refresh_flops / (refresh_ms * 1e-3) / 1e12) if refresh_ms else None,
                            "full_refresh_step_ms_est": refresh_ms * c.n_layers if refresh_ms else None},
            "e2e": {"value": e2e_value, "unit": "active tok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps},
            "cpu_baseline": cpu_baseline,
            "clocks": sampler.summary(),
            "gpu_launches": gpu_launches,
            "device_error": err,
        }
        print(json.dumps(line), flush=True)
    step.release()
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
