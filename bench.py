"""Benchmark: one pre-fill attention layer of the 1M-token LLaMA-3-8B-shaped
workload (32 query / 8 KV heads, d=128, N=1048576; 24 Vertical-Slash heads
with vertical 2000 / slash 12000, 6 Block-Sparse heads with top-100 blocks,
2 A-shape heads with 128 sink + 4096 local) through libminf.

A step is the whole hot path for every head: index estimation, index build
and sparse attention.  ``value`` is the effective throughput: the attention
work the masks keep (4 d per kept score entry: Q K^T and P V) divided by the
device time of the step, with inputs already in HBM.  ``e2e`` is the same
quantity with pinned-host inputs copied in and the output copied out inside
the timed region.  The roofline object reports the dominant kernel (the
Vertical-Slash attention launch) against the measured bf16 tensor peak, on
the tiles it actually executes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) the layer is split across the ranks by KV-head group
(``--shard kv``, the default): rank r computes the query heads of KV heads
[r Hkv/N, (r+1) Hkv/N) with their rows of the pattern table, O stays
head-sharded and no collective touches the data path (strong scaling).
``--shard replicas`` runs one independent layer per rank instead (weak
scaling).  Time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

WORKLOAD_ID = 4
METRIC = "prefill sparse-attention ms and effective TFLOP/s at N=128K–1M, % bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, index: int, path: str | None = None):
        import tempfile
        self.index = index
        self.proc = None
        if path is None:
            fd, path = tempfile.mkstemp(prefix=f"minf_clocks_{index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def __enter__(self):
        if os.path.dirname(self.path):
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        try:
            lines = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.strip()]
        except OSError:
            return None
        if not lines:
            return None
        mhz = [float(l[1]) for l in lines if l[1].strip().replace(".", "").isdigit()]
        mx = max(float(l[2]) for l in lines)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for l in lines for i in range(4)
                          if len(l) > 5 + i and l[5 + i].strip() == "Active"})
        loaded = [m for m in mhz if m > 0.5 * mx] or mhz
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(lines)}


_KERNEL_SOURCES = ("csrc/attn.cu", "csrc/minf_device.cuh", "csrc/minf_internal.h")
_TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "attn_vs_n256k_dram.md")


def _code_only(src: str) -> str:
    """C++ source with comments removed and whitespace collapsed, so that a
    documentation edit does not count as a kernel change."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in _KERNEL_SOURCES:
        with open(os.path.join(ROOT, "dynamic_sparse_attention_minf_b200", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()


def _recorded_traffic():
    """DRAM bytes (read + write) per executed 128 x 128 tile of the attention
    kernel, from the committed ncu summary of one Vertical-Slash launch at
    256K tokens (8 query / 2 KV heads), or None when the attention sources no
    longer hash to the ones that summary was captured from.  The bench scales
    it by the executed tiles of the launch it reports."""
    try:
        text = open(_TRAFFIC_PROFILE).read()
        vals = dict(line.split(": ", 1) for line in text.splitlines()
                    if line.startswith(("traffic_bytes_per_tile: ", "kernel_sources_sha256: ")))
        if vals.get("kernel_sources_sha256", "").strip() != kernel_sources_digest():
            return None
        return float(vals["traffic_bytes_per_tile"])
    except (OSError, KeyError, ValueError):
        return None


def _patterns_text(w) -> str:
    """Head -> pattern table of a workload, as text for the JSON line."""
    from dynamic_sparse_attention_minf_b200 import workloads as wl
    parts = []
    nvs, nbs, na = (len(w.heads_of(p)) for p in (wl.PAT_VS, wl.PAT_BS, wl.PAT_A))
    if nvs:
        parts.append(f"{nvs} vertical-slash ({w.k_v}/{w.k_s})")
    if nbs:
        parts.append(f"{nbs} block-sparse (top-{w.k_b})")
    if na:
        parts.append(f"{na} a-shape ({w.n_sink}+{w.n_local})")
    return ", ".join(parts)


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, rank, ws, local
    return None, 0, 1, 0


def _max_over_ranks(dist, x: float) -> float:
    """The slowest rank's time: every rank contributes, every rank gets the max."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _throughput(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job TFLOP/s when every rank processes its own layer (weak scaling)."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def _sum_over_ranks(dist, x: float) -> float:
    """Sum of a per-rank quantity (every rank gets it)."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def _counters(ws):
    from dynamic_sparse_attention_minf_b200 import minf
    return minf.attn_counters(ws)


# ----------------------------------------------------------- CPU oracle leg
def oracle_sample(w, q, k, v, plan, rows_per_pattern=16, seed=0):
    """The oracle on a bounded sample of the workload: one head of each
    pattern gets its full index estimation and `rows_per_pattern` sampled
    query rows of attention.  Returns (useful FLOPs, seconds, seconds per row
    and per head estimate) so that callers can scale to the whole layer."""
    import numpy as np
    from oracle import minf_oracle as orc
    from dynamic_sparse_attention_minf_b200 import workloads as wl

    sc = orc.default_scale(w.d)
    rows = wl.sample_rows(w.N, rows_per_pattern, seed).numpy()
    out = {}
    for pat in (wl.PAT_VS, wl.PAT_BS, wl.PAT_A):
        heads = w.heads_of(pat)
        if not heads:
            continue
        h = heads[0]
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        kn = orc.to_f64(k[0, kv])
        vn = orc.to_f64(v[0, kv])
        qr = orc.to_f64(q[0, h])
        t0 = time.perf_counter()
        if pat == wl.PAT_VS:
            vv, ss = orc.vs_estimate(qr[w.N - w.last_q:], kn, sc)
            V, S = orc.vs_select(vv, ss, w.k_v, w.k_s)
            fn = lambda r: orc.mask_vs(r, w.N, V, S)
        elif pat == wl.PAT_BS:
            # pooling for the whole head, selection for the sampled rows' query
            # blocks only (its time is scaled to all blocks below)
            blks = np.unique(rows // w.block)
            orc.bs_pool(qr, w.block), orc.bs_pool(kn, w.block)
            t_pool = time.perf_counter() - t0
            bi_s, bc_s = orc.bs_select(qr, kn, sc, w.k_b, blocks=blks)
            nb = w.N // w.block
            bi = np.full((nb, w.k_b), -1, np.int64)
            bc = np.zeros(nb, np.int64)
            bi[blks], bc[blks] = bi_s, bc_s
            fn = lambda r, bi=bi, bc=bc: orc.mask_bs(r, w.N, bi, bc)
        else:
            fn = lambda r: orc.mask_ashape(r, w.N, w.n_sink, w.n_local)
        t1 = time.perf_counter()
        if pat == wl.PAT_BS:
            sel = (t1 - t0) - 2 * t_pool
            t0 = t1 - (t_pool + max(sel, 0.0) * (w.N // w.block) / len(np.unique(rows // w.block)))
        nnz = int(fn(rows).sum())
        orc.attention_head(qr, kn, vn, rows, fn, sc)
        t2 = time.perf_counter()
        out[pat] = dict(est_s=t1 - t0, row_s=(t2 - t1) / len(rows), nnz_per_row=nnz / len(rows),
                        heads=len(heads))
    # scale to the whole layer: estimation per head + attention per row
    total_s = sum(o["heads"] * (o["est_s"] + o["row_s"] * w.N) for o in out.values())
    flops = sum(o["heads"] * 4.0 * w.d * o["nnz_per_row"] * w.N for o in out.values())
    sample_s = sum(o["est_s"] + o["row_s"] * len(rows) for o in out.values())
    return flops, total_s, sample_s, out


def _cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=1)
        return int(n)
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def run_reference(args, dist, rank, world):
    """The oracle (test infrastructure, as it stands) timed on host cores."""
    if rank != 0:
        return
    from dynamic_sparse_attention_minf_b200 import workloads as wl
    w = wl.config(args.config)
    q, k, v = wl.make_qkv(w, "cuda" if torch.cuda.is_available() else "cpu")
    times, flops_l, samples = [], [], []
    for step in range(args.warmup + args.steps):
        flops, total_s, sample_s, _ = oracle_sample(w, q, k, v, None, rows_per_pattern=8, seed=step)
        if step >= args.warmup:
            times.append(total_s)
            flops_l.append(flops)
            samples.append(sample_s)
    val = sum(flops_l) / sum(times) / 1e12
    ms = 1000.0 * statistics.mean(times)
    cores = _cores()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": "per step: one head of each pattern with full index estimation "
                                       "and 8 sampled query rows, scaled to all heads and rows "
                                       f"(measured {statistics.mean(samples):.1f} s of CPU per step)"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- our arm
def run_ours(args, dist, rank, world, local):
    from dynamic_sparse_attention_minf_b200 import layer, minf
    from dynamic_sparse_attention_minf_b200 import workloads as wl

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w_full = wl.config(args.config)
    shard = world > 1 and args.shard == "kv"
    if shard:
        # one layer split by KV-head group: every rank draws the same inputs
        # and keeps its own heads
        hq0, hq1, hk0, hk1 = layer.kv_group_slice(w_full, rank, world)
        qf, kf, vf = wl.make_qkv(w_full, dev)
        q, k, v = (x[:, a:b].contiguous() for x, a, b in ((qf, hq0, hq1), (kf, hk0, hk1), (vf, hk0, hk1)))
        del qf, kf, vf
        torch.cuda.empty_cache()
        w = layer.local_workload(w_full, rank, world)
    else:
        w = w_full
        w.seed += 100 * rank                  # independent prompts per rank
        q, k, v = wl.make_qkv(w, dev)
    plan = layer.make_plan(w, dev)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    # one counted run per pattern (one attention launch each): executed
    # tiles and kept entries of every pattern; then the same layer with one
    # attention launch for all heads, whose counters must add up to them
    attn_ws = [n for n in ("ws_vs_attn", "ws_bs_attn", "ws_a") if n in plan.bufs]
    for name in attn_ws + ["ws_attn"]:
        plan.bufs[name].zero_()
    layer.run_layer(plan, q, k, v, o, fused=False)
    layer.run_layer(plan, q, k, v, o, fused=True)
    torch.cuda.synchronize()
    status = layer.device_status(plan)
    if status:
        raise RuntimeError(f"device status {status}")
    cnt = {n: _counters(plan.bufs[n]) for n in attn_ws}
    fused_cnt = _counters(plan.bufs["ws_attn"])
    tile_flops = 4.0 * 128 * 128 * w.d
    useful = sum(4.0 * w.d * c[1] for c in cnt.values())
    executed = sum(tile_flops * c[0] for c in cnt.values())
    exec_tiles = sum(c[0] for c in cnt.values())
    if fused_cnt != (exec_tiles, sum(c[1] for c in cnt.values())):
        raise RuntimeError(f"one-launch counters {fused_cnt} differ from the per-pattern launches {cnt}")

    # warm-up
    for _ in range(args.warmup):
        layer.run_layer(plan, q, k, v, o)
    torch.cuda.synchronize()

    # timed device steps, with events around every call of the layer
    marks = []

    class Marks:
        def __init__(self):
            self.events = []

        def mark(self, name):
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            self.events.append((name, e))

    def phase_means(events):
        phases = {}
        for a_, b_ in zip(events[0::2], events[1::2]):
            name = a_[0].split(":")[0]
            assert a_[0] == name + ":pre" and b_[0] == name + ":post"
            phases.setdefault(name, []).append(a_[1].elapsed_time(b_[1]))
        return {n: round(statistics.mean(t), 3) for n, t in phases.items()}

    mk = Marks()
    clock_log = args.clock_log.replace("{rank}", str(rank)) if args.clock_log else None
    with ClockSampler(local, clock_log) as clk:
        time.sleep(1.0)                      # let the sampler start before timing
        _barrier(dist)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(stream)
        for s_ in range(args.steps):
            layer.run_layer(plan, q, k, v, o, marks=mk)
            ev[s_ + 1].record(stream)
        torch.cuda.synchronize()
        _barrier(dist)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    step_ms = ev[0].elapsed_time(ev[-1]) / args.steps
    step_ms = _max_over_ranks(dist, step_ms)
    phase_ms = phase_means(mk.events)
    attn_ms = phase_ms.get("attn")

    # the same layer with one attention launch per pattern, for comparison
    # (outside the timed steps)
    mk_sep = Marks()
    for _ in range(2):
        layer.run_layer(plan, q, k, v, o, marks=mk_sep, fused=False)
    torch.cuda.synchronize()
    sep_ms = phase_means(mk_sep.events)
    attn_sep = {n: sep_ms[n] for n in ("vs_attn", "bs_attn", "a_attn") if n in sep_ms}

    # end to end through the public API: pinned host in, host out
    hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hq.copy_(q)
    hk.copy_(k)
    hv.copy_(v)
    e2e_steps = max(3, min(args.steps + 3, 8))
    pbufs = layer.PipelineBuffers(hq, hk, hv, ho, dev)
    layer.run_pipelined(plan, hq, hk, hv, ho, 2, pbufs, compute=stream)   # warm the copy streams
    _barrier(dist)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e1 = layer.run_pipelined(plan, hq, hk, hv, ho, e2e_steps, pbufs, compute=stream, start_event=e0)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(dist, e0.elapsed_time(e1) / e2e_steps)
    del pbufs
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = o.numel() * 2

    # dense baseline from the same library: one head, scaled to all heads
    dense_ms = None
    if rank == 0 and not args.no_dense:
        od = torch.empty_like(q)
        wsd = minf.workspace(minf.OP_DENSE_ATTN, plan.shape, 1, device=dev)
        h0 = torch.tensor([0], dtype=torch.int32, device=dev)
        minf.minf_dense_attn(q, k, v, h0, o=od, want_lse=False, ws=wsd)
        torch.cuda.synchronize()
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        minf.minf_dense_attn(q, k, v, h0, o=od, want_lse=False, ws=wsd)
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = d0.elapsed_time(d1) * w.Hq
        del od

    # element-exact Vertical-Slash variant on the layer's VS heads and sets
    # (outside the timed step: index build and attention, CUDA events)
    vs_exact = None
    if rank == 0 and not args.no_exact and plan.vs_heads is not None:
        b = plan.bufs
        ws_x = minf.workspace(minf.OP_SPARSE_ATTN_VS_EXACT, plan.shape, plan.vs_heads.numel(), device=dev)
        ws_xi = minf.workspace(minf.OP_BUILD_INDEX_EXACT, plan.shape, plan.vs_heads.numel(), device=dev)
        xi = minf.minf_build_index_exact(plan.shape, b["v_idx"], b["s_idx"], ws=ws_xi)
        ox = o  # the timed steps are done; reuse the output buffer
        ws_x.zero_()
        minf.minf_sparse_attn_vs_exact(q, k, v, plan.vs_heads, xi, o=ox, want_lse=False, ws=ws_x)
        torch.cuda.synchronize()
        if minf.minf_get_device_status(ws_xi) or minf.minf_get_device_status(ws_x):
            raise RuntimeError("exact variant reported a device error")
        x_tiles, x_nnz = _counters(ws_x)
        xe = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        xe[0].record(stream)
        minf.minf_build_index_exact(plan.shape, b["v_idx"], b["s_idx"], index=xi, ws=ws_xi)
        xe[1].record(stream)
        for _ in range(2):
            minf.minf_sparse_attn_vs_exact(q, k, v, plan.vs_heads, xi, o=ox, want_lse=False, ws=ws_x)
        xe[2].record(stream)
        torch.cuda.synchronize()
        x_ms = xe[1].elapsed_time(xe[2]) / 2
        vs_exact = {
            "attn_ms": round(x_ms, 3), "index_ms": round(xe[0].elapsed_time(xe[1]), 3),
            "executed_tflop": tile_flops * x_tiles / 1e12, "useful_tflop": 4.0 * w.d * x_nnz / 1e12,
            "executed_tflops": tile_flops * x_tiles / (x_ms * 1e-3) / 1e12,
            "useful_tflops": 4.0 * w.d * x_nnz / (x_ms * 1e-3) / 1e12,
            "band_useful_tflop": 4.0 * w.d * cnt["ws_vs_attn"][1] / 1e12,
            "band_tiles": cnt["ws_vs_attn"][0], "band_ms": attn_sep.get("vs_attn"),
        }
        del xi

    # whole-job work: the ranks' shares of one layer add up (KV-head split),
    # or every rank runs a layer of its own (replicas)
    useful_job = _sum_over_ranks(dist, useful) if shard else world * useful
    if rank != 0:
        return
    peaks, src = _peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = executed / (attn_ms * 1e-3) / 1e12 if attn_ms else None
    cpu = None
    if world == 1 and not args.no_cpu:
        flops_c, total_s, sample_s, _ = oracle_sample(w, q, k, v, plan, rows_per_pattern=96)
        cpu = {"value": flops_c / total_s / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
               "sample": "one head of each pattern with full index estimation and 96 sampled query rows, "
                         f"scaled to all heads and rows ({sample_s:.1f} s of CPU)"}
    clocks = clk.summary()
    val = useful_job / (step_ms * 1e-3) / 1e12
    dense_flops = 4.0 * w.d * (w.N * (w.N + 1) / 2) * w.Hq
    traffic = _recorded_traffic()
    # tensor-pipe utilisation at the run's own clock: the bf16 MMA of this
    # kernel (M = N = 128, K = 16) retires 8192 FLOP per clock per SM
    sm_mhz = (clocks or {}).get("sm_mhz")
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    tensor_at_clock = (achieved / (8192.0 * nsm * sm_mhz * 1e6 / 1e12)) if (achieved and sm_mhz) else None
    line = {
        "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "strong" if shard else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w_full.name, "N": w.N, "Hq": w_full.Hq, "Hkv": w_full.Hkv, "d": w.d,
                   "patterns": _patterns_text(w_full),
                   "parallelism": (f"kv-head groups x{world}" if shard else f"replicas{world}") if world > 1
                   else "single",
                   "l2": f"inputs {(q.numel() + k.numel() + v.numel()) * 2 / 2**30:.1f} GiB per step and rank, "
                         "larger than the 126 MB L2 (no flush needed)"},
        "step_ms_each": [round(x, 2) for x in per_step],
        "phase_ms": phase_ms,
        "attn_ms_one_launch_per_pattern": attn_sep,
        "useful_tflop_per_step": useful_job / 1e12, "executed_tflop_per_step": executed / 1e12,
        "density_vs_dense": useful / dense_flops,
        "dense_attn_ms_est": dense_ms,
        "speedup_vs_dense": (dense_ms / step_ms) if dense_ms else None,
        "roofline": {"kernel": f"attn_kernel<{w.d}> (one launch, every head of the layer)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": (achieved / peak) if achieved else None,
                     "traffic": (traffic * exec_tiles) if traffic else None,
                     "traffic_unit": "bytes per launch: ncu dram__bytes_read.sum + dram__bytes_write.sum per "
                                     "executed tile of the 256K Vertical-Slash capture, times this launch's tiles",
                     "peak_source": f"{src} bf16_tflops_sustained (of measured)" if src == "measured"
                                    else f"{src} (of fallback)",
                     "ms_per_launch": attn_ms, "executed_tflop_per_launch": executed / 1e12,
                     "tensor_active_at_run_clock": tensor_at_clock,
                     "vs_launch": {"tiles": cnt["ws_vs_attn"][0] if "ws_vs_attn" in cnt else None,
                                   "ms_one_launch_per_pattern": attn_sep.get("vs_attn")}},
        "e2e": {"value": useful_job / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "mode": "layer.run_pipelined: every step uploads its Q/K/V from pinned host memory and "
                        "downloads its O, on copy streams overlapping the neighbouring steps' compute"},
        "gpu_launches": layer.launches_per_step(plan) * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "vs_exact": ({**vs_exact, "frac": vs_exact["executed_tflops"] / peak} if vs_exact else None),
    }
    print(json.dumps(line), flush=True)


def run_kernel_case(args):
    """One kernel on a small case, for profilers: ``--kernel dense|vs`` at
    ``--N`` tokens (8 query / 2 KV heads, d = 128; the VS case uses the 1M
    workload's budgets, vertical 2000 / slash 12000).  The index is built
    once; then the kernel runs ``--warmup`` + ``--steps`` times.
    ``--kernel vs_est|bs_est`` runs the index estimation of those 8 heads
    instead (vertical 2000 / slash 12000; top-100 blocks), and ``--kernel grid``
    the Grid-pattern attention of the 8 heads over ``--N`` / 256 frames of 256
    tokens (top-100 frame blocks), timed with CUDA events.  ``--kernel
    vs_est_layer`` times the Vertical-Slash estimation of all VS heads of the
    ``--config`` layer at full size."""
    from dynamic_sparse_attention_minf_b200 import layer, minf
    from dynamic_sparse_attention_minf_b200 import workloads as wl
    if args.kernel == "vs_est_layer":
        # Vertical-Slash estimation of every VS head of the --config layer at
        # its full size, 3 rounds of one untimed and 5 timed calls (CUDA events)
        w = wl.config(args.config)
        q, k, v = wl.make_qkv(w, "cuda")
        heads = w.heads_of(wl.PAT_VS)
        ws = minf.workspace(minf.OP_ESTIMATE_VS, minf.shape_of(q, k), len(heads))
        out, res = None, []
        for _ in range(3):
            minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, ws=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(5):
                out = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            res.append(round(e0.elapsed_time(e1) / 5, 3))
        print(json.dumps({"kernel": args.kernel, "workload": w.name, "N": w.N, "heads": len(heads),
                          "vs_est_ms": res, "status": minf.minf_get_device_status(ws),
                          "v_sum": int(out[0].sum().item()), "s_sum": int(out[1].sum().item())}))
        return
    w = wl.config(WORKLOAD_ID, N=args.N)
    w.Hq, w.Hkv = 8, 2
    w.patterns = [wl.PAT_VS] * 8
    q, k, v = wl.make_qkv(w, "cuda")
    o = torch.empty_like(q)
    if args.kernel == "grid":
        shp = minf.shape_of(q, k)
        heads = list(range(8))
        P, k_b = 256, 100
        ws = minf.workspace(minf.OP_ATTN_GRID, shp, 8, k_b=k_b)
        fn = lambda: minf.minf_attn_grid(q, k, v, heads, P, k_b, o=o, want_lse=False, ws=ws)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ws.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        tiles, nnz = _counters(ws)
        # permutation traffic: Q and O of the 8 heads and K and V of the 2 KV heads, read and written
        perm_bytes = 2 * (2 * 8 + 2 * 2) * w.N * w.d * 2
        print(json.dumps({"kernel": "grid", "N": args.N, "frame_tokens": P, "frames": args.N // P, "k_b": k_b,
                          "ms": ms, "tiles_per_call": tiles // args.steps, "useful_tflop": 4.0 * w.d * nnz / args.steps / 1e12,
                          "permuted_bytes": perm_bytes, "status": minf.minf_get_device_status(ws)}))
        return
    if args.kernel in ("vs_est", "bs_est"):
        shp = minf.shape_of(q, k)
        heads = list(range(8))
        if args.kernel == "vs_est":
            ws = minf.workspace(minf.OP_ESTIMATE_VS, shp, 8)
            fn = lambda: minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, ws=ws)
        else:
            ws = minf.workspace(minf.OP_ESTIMATE_BS, shp, 8, k_b=100)
            fn = lambda: minf.minf_estimate_bs(q, k, heads, 100, ws=ws)
        for _ in range(args.warmup + args.steps):
            fn()
        torch.cuda.synchronize()
        print(json.dumps({"kernel": args.kernel, "N": args.N, "launches": args.warmup + args.steps,
                          "status": minf.minf_get_device_status(ws)}))
        return
    if args.kernel == "vs":
        plan = layer.make_plan(w, "cuda")
        layer.run_layer(plan, q, k, v, o)
        b = plan.bufs
        fn = lambda: minf.minf_sparse_attn_vs(q, k, v, plan.vs_heads, b["vs_index"], o=o, want_lse=False,
                                              ws=b["ws_vs_attn"])
    else:
        ws = minf.workspace(minf.OP_DENSE_ATTN, minf.shape_of(q, k), 1)
        fn = lambda: minf.minf_dense_attn(q, k, v, [0], o=o, want_lse=False, ws=ws)
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    # executed tiles of one launch (the device counter of a fresh workspace)
    ws_k = b["ws_vs_attn"] if args.kernel == "vs" else ws
    ws_k.zero_()
    fn()
    torch.cuda.synchronize()
    tiles = _counters(ws_k)[0]
    print(json.dumps({"kernel": args.kernel, "N": args.N, "launches": args.warmup + args.steps + 1,
                      "tiles_per_launch": tiles, "kernel_sources_sha256": kernel_sources_digest()}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle leg")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense baseline")
    ap.add_argument("--no-exact", action="store_true", help="skip the element-exact VS variant")
    ap.add_argument("--config", type=int, default=WORKLOAD_ID, choices=[2, 3, 4],
                    help="workload: 4 (default) the 1M-token mixed layer, 2 the 128K mixed layer, "
                         "3 the 512K all-Vertical-Slash layer")
    ap.add_argument("--kernel", choices=["dense", "vs", "vs_est", "bs_est", "grid", "vs_est_layer"], default=None,
                    help="run only this kernel on a small case (for profiling); vs_est_layer times the "
                         "Vertical-Slash estimation of the --config layer's VS heads at full size")
    ap.add_argument("--N", type=int, default=262144, help="tokens of the --kernel case")
    ap.add_argument("--shard", choices=["kv", "replicas"], default="kv",
                    help="with several GPUs: split one layer by KV-head group (default) or run a layer per rank")
    ap.add_argument("--clock-log", default=None,
                    help="keep the nvidia-smi clock samples in this CSV file ({rank} is replaced by the "
                         "rank); default: a temporary file")
    args = ap.parse_args()
    if args.kernel:
        run_kernel_case(args)
        return
    dist, rank, world, local = _dist()
    try:
        if args.impl == "reference":
            run_reference(args, dist, rank, world)
        else:
            run_ours(args, dist, rank, world, local)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
