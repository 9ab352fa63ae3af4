"""One attention layer's pre-fill through libminf: a head -> pattern table
routes every query head to Vertical-Slash, Block-Sparse or A-shape ("MInference
1.0" summary, "Summary": a pattern per head chosen offline, indices built
online, attention over the indices only).

This module only sequences C-ABI calls and owns their buffers (allocated once,
up front, so that a timed step launches kernels and nothing else).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import minf
from .workloads import PAT_A, PAT_BS, PAT_VS, Workload


@dataclass
class LayerPlan:
    w: Workload
    device: torch.device
    vs_heads: torch.Tensor | None = None
    bs_heads: torch.Tensor | None = None
    a_heads: torch.Tensor | None = None
    bufs: dict = field(default_factory=dict)

    @property
    def shape(self):
        w = self.w
        return minf.Shape(w.B, w.Hq, w.Hkv, w.N, w.d, 0.0)


def kv_group_slice(w: Workload, rank: int, world: int):
    """The share of rank ``rank`` when one layer is split across ``world``
    GPUs by KV-head group: KV heads [hk0, hk1) and their query heads
    [hq0, hq1) (contiguous, since query head h reads KV head h // g).  Heads
    are independent, so the shares need no exchange; O stays head-sharded."""
    if world < 1 or w.Hkv % world:
        raise ValueError(f"{w.Hkv} KV heads do not split over {world} ranks")
    per = w.Hkv // world
    hk0, hk1 = rank * per, (rank + 1) * per
    return hk0 * w.group, hk1 * w.group, hk0, hk1


def local_workload(w: Workload, rank: int, world: int) -> Workload:
    """The workload one rank runs under :func:`kv_group_slice`: its query and
    KV heads only, with their rows of the head -> pattern table."""
    import dataclasses
    hq0, hq1, hk0, hk1 = kv_group_slice(w, rank, world)
    return dataclasses.replace(w, name=f"{w.name}_kv{hk0}-{hk1 - 1}", Hq=hq1 - hq0, Hkv=hk1 - hk0,
                               patterns=list(w.patterns[hq0:hq1]))


def make_plan(w: Workload, device="cuda") -> LayerPlan:
    dev = torch.device(device)
    plan = LayerPlan(w, dev)
    shp = plan.shape
    i32 = dict(dtype=torch.int32, device=dev)
    vs = w.heads_of(PAT_VS)
    bs = w.heads_of(PAT_BS)
    ah = w.heads_of(PAT_A)
    B, N = w.B, w.N
    if vs:
        plan.vs_heads = torch.tensor(vs, **i32)
        nv = len(vs)
        plan.bufs["v_idx"] = torch.empty(B, nv, w.k_v, **i32)
        plan.bufs["s_idx"] = torch.empty(B, nv, w.k_s, **i32)
        plan.bufs["ws_vs_est"] = minf.workspace(minf.OP_ESTIMATE_VS, shp, nv, device=dev)
        plan.bufs["ws_vs_idx"] = minf.workspace(minf.OP_BUILD_INDEX, shp, nv, device=dev)
        plan.bufs["ws_vs_attn"] = minf.workspace(minf.OP_SPARSE_ATTN_VS, shp, nv, device=dev)
        plan.bufs["vs_index"] = minf.VSIndex.empty(B, nv, N, w.k_v, w.k_s, device=dev)
    if bs:
        plan.bs_heads = torch.tensor(bs, **i32)
        nbh = len(bs)
        plan.bufs["blk_idx"] = torch.empty(B, nbh, N // 64, w.k_b, **i32)
        plan.bufs["blk_cnt"] = torch.empty(B, nbh, N // 64, **i32)
        plan.bufs["ws_bs_est"] = minf.workspace(minf.OP_ESTIMATE_BS, shp, nbh, k_b=w.k_b, device=dev)
        plan.bufs["ws_bs_attn"] = minf.workspace(minf.OP_SPARSE_ATTN_BS, shp, nbh, device=dev)
    if ah:
        plan.a_heads = torch.tensor(ah, **i32)
        plan.bufs["ws_a"] = minf.workspace(minf.OP_ATTN_ASHAPE, shp, len(ah), device=dev)
    plan.bufs["ws_attn"] = minf.workspace(minf.OP_SPARSE_ATTN_LAYER, shp, len(vs) + len(bs) + len(ah), device=dev)
    return plan


# rows longer than this take the many-CTA top-k (nine launches instead of one)
TOPK_LONG_ROW = 32768


def launches_per_step(plan: LayerPlan, fused: bool = True) -> int:
    """Kernels one run_layer call launches: VS estimation (two score passes,
    row combine, slash combine, two top-k), VS index build 3, BS estimation
    3 (pool, pooled scores, top-k), and the attention: one launch for every
    head (fused) or one per pattern."""
    n = 0
    if plan.vs_heads is not None:
        topk = 9 if plan.w.N > TOPK_LONG_ROW else 1
        n += 4 + 2 * topk + 3
    if plan.bs_heads is not None:
        n += 3
    if fused:
        n += 1
    else:
        n += sum(1 for h in (plan.vs_heads, plan.bs_heads, plan.a_heads) if h is not None)
    return n


def run_layer(plan: LayerPlan, q, k, v, o, lse=None, stream=None, marks=None, fused: bool = True):
    """Estimation, index build and sparse attention for every head of the
    layer, in stream order; O (and LSE) are filled head by head.  With
    ``fused`` the attention of all heads runs as one launch
    (minf_sparse_attn_layer), otherwise as one launch per pattern.  ``marks``
    (optional) gets ``mark(name)`` calls, ``<phase>:pre`` and ``<phase>:post``,
    around every call of the layer."""
    mark = marks.mark if marks is not None else (lambda name: None)
    w, b = plan.w, plan.bufs
    shp = plan.shape
    L = minf.lib()
    st = minf._stream(stream)
    P = minf._p
    nv = plan.vs_heads.numel() if plan.vs_heads is not None else 0
    nbh = plan.bs_heads.numel() if plan.bs_heads is not None else 0
    na = plan.a_heads.numel() if plan.a_heads is not None else 0
    ic = b["vs_index"].c() if nv else None
    if nv:
        mark("vs_est:pre")
        minf._check("minf_estimate_vs", L.minf_estimate_vs(
            minf.ctypes.byref(shp), P(q), P(k), P(plan.vs_heads), nv, w.last_q, w.k_v, w.k_s,
            P(b["v_idx"]), P(b["s_idx"]), None, None, P(b["ws_vs_est"]), b["ws_vs_est"].numel(), st))
        mark("vs_est:post")
        mark("vs_index:pre")
        minf._check("minf_build_index", L.minf_build_index(
            minf.ctypes.byref(shp), nv, P(b["v_idx"]), w.k_v, P(b["s_idx"]), w.k_s, minf.ctypes.byref(ic),
            P(b["ws_vs_idx"]), b["ws_vs_idx"].numel(), st))
        mark("vs_index:post")
    if nbh:
        mark("bs_est:pre")
        minf._check("minf_estimate_bs", L.minf_estimate_bs(
            minf.ctypes.byref(shp), P(q), P(k), P(plan.bs_heads), nbh, w.block, w.k_b,
            P(b["blk_idx"]), P(b["blk_cnt"]), None, P(b["ws_bs_est"]), b["ws_bs_est"].numel(), st))
        mark("bs_est:post")
    if fused:
        mark("attn:pre")
        minf._check("minf_sparse_attn_layer", L.minf_sparse_attn_layer(
            minf.ctypes.byref(shp), P(q), P(k), P(v), P(plan.vs_heads) if nv else None, nv,
            minf.ctypes.byref(ic) if nv else None, w.k_v, w.k_s,
            P(plan.bs_heads) if nbh else None, nbh, P(b["blk_idx"]) if nbh else None,
            P(b["blk_cnt"]) if nbh else None, w.k_b, P(plan.a_heads) if na else None, na,
            w.n_sink, w.n_local, P(o), P(lse), P(b["ws_attn"]), b["ws_attn"].numel(), st))
        mark("attn:post")
        return o, lse
    if nv:
        mark("vs_attn:pre")
        minf._check("minf_sparse_attn_vs", L.minf_sparse_attn_vs(
            minf.ctypes.byref(shp), P(q), P(k), P(v), P(plan.vs_heads), nv, minf.ctypes.byref(ic),
            w.k_v, w.k_s, P(o), P(lse), P(b["ws_vs_attn"]), b["ws_vs_attn"].numel(), st))
        mark("vs_attn:post")
    if nbh:
        mark("bs_attn:pre")
        minf._check("minf_sparse_attn_bs", L.minf_sparse_attn_bs(
            minf.ctypes.byref(shp), P(q), P(k), P(v), P(plan.bs_heads), nbh, P(b["blk_idx"]),
            P(b["blk_cnt"]), w.k_b, P(o), P(lse), P(b["ws_bs_attn"]), b["ws_bs_attn"].numel(), st))
        mark("bs_attn:post")
    if na:
        mark("a_attn:pre")
        minf._check("minf_attn_ashape", L.minf_attn_ashape(
            minf.ctypes.byref(shp), P(q), P(k), P(v), P(plan.a_heads), na, w.n_sink, w.n_local,
            P(o), P(lse), P(b["ws_a"]), b["ws_a"].numel(), st))
        mark("a_attn:post")
    return o, lse


class PipelineBuffers:
    """Two device copies of a layer's Q, K, V and O for :func:`run_pipelined`."""

    def __init__(self, hq, hk, hv, ho, device):
        self.sets = [tuple(torch.empty(x.shape, dtype=x.dtype, device=device) for x in (hq, hk, hv, ho))
                     for _ in range(2)]


def run_pipelined(plan: LayerPlan, hq, hk, hv, ho, steps: int, bufs: PipelineBuffers,
                  compute=None, start_event=None):
    """Runs the layer ``steps`` times on host-resident (pinned) inputs, end to
    end: every step copies its Q, K and V to the device and its O back to the
    host.  The copies run on their own streams (one per direction) into two
    alternating device buffer sets, so that step s+1's inputs upload and step
    s-1's output downloads while step s computes.  Work is queued behind
    ``start_event`` (if given) on the ``compute`` stream; returns the event
    recorded there once the last output has reached the host."""
    compute = compute or torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    if start_event is not None:
        up.wait_event(start_event)
        compute.wait_event(start_event)
    ev_in = [torch.cuda.Event() for _ in range(steps)]
    ev_done = [torch.cuda.Event() for _ in range(steps)]
    ev_out = [torch.cuda.Event() for _ in range(steps)]
    for s_ in range(steps):
        q, k, v, o = bufs.sets[s_ % 2]
        with torch.cuda.stream(up):
            if s_ >= 2:
                up.wait_event(ev_done[s_ - 2])      # step s-2 has read these inputs
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            ev_in[s_].record(up)
        compute.wait_event(ev_in[s_])
        if s_ >= 2:
            compute.wait_event(ev_out[s_ - 2])      # step s-2's output is on the host
        run_layer(plan, q, k, v, o, stream=compute)
        ev_done[s_].record(compute)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[s_])
            ho.copy_(o, non_blocking=True)
            ev_out[s_].record(down)
    compute.wait_event(ev_out[steps - 1])
    end = torch.cuda.Event(enable_timing=True)
    end.record(compute)
    return end


def device_status(plan: LayerPlan):
    """First device-side error code across the plan's workspaces (0 = none)."""
    for name, t in plan.bufs.items():
        if name.startswith("ws_"):
            code = minf.minf_get_device_status(t)
            if code:
                return code
    return 0
