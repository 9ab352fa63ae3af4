"""Full-size parity: the whole mixed-pattern layer at N = 128K, 512K and 1M
tokens, in the launch configuration bench.py times, and the element-exact
Vertical-Slash variant on the same heads and sets.  Index sets are checked
in full (bit-exact up to the score-gap rule, the index build bit-exact);
attention outputs on 512 seeded sampled query rows per head.  The oracle runs
in a spawn-started process pool, one query head per task."""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import layer, minf
from dynamic_sparse_attention_minf_b200 import workloads as wl
from tests import oracle_pool as op

pytestmark = [pytest.mark.gpu, pytest.mark.large]


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("cid", [2, 3, 4])
def test_full_size_layer(cid):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    minf.lib()
    w = wl.config(cid)
    q, k, v = wl.make_qkv(w, "cuda")
    plan = layer.make_plan(w, "cuda")
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    layer.run_layer(plan, q, k, v, o, lse)
    torch.cuda.synchronize()
    assert layer.device_status(plan) == 0
    rows = wl.sample_rows(w.N, 512, w.seed)
    rows_d = rows.to("cuda")
    o_rows = o[0][:, rows_d].float().cpu().numpy()
    lse_rows = lse[0][:, rows_d].cpu().numpy()
    # the element-exact variant on the same VS heads and sets (into the same
    # output buffers, whose sampled rows are already copied)
    xi = None
    if plan.vs_heads is not None:
        b = plan.bufs
        ws_xi = minf.workspace(minf.OP_BUILD_INDEX_EXACT, plan.shape, plan.vs_heads.numel())
        xi = minf.minf_build_index_exact(plan.shape, b["v_idx"], b["s_idx"], ws=ws_xi)
        ws_x = minf.workspace(minf.OP_SPARSE_ATTN_VS_EXACT, plan.shape, plan.vs_heads.numel())
        minf.minf_sparse_attn_vs_exact(q, k, v, plan.vs_heads, xi, o=o, lse=lse, ws=ws_x)
        assert minf.minf_get_device_status(ws_xi) == 0 and minf.minf_get_device_status(ws_x) == 0
        ox_rows = o[0][:, rows_d].float().cpu().numpy()
        lsex_rows = lse[0][:, rows_d].cpu().numpy()

    keep = []
    try:
        Q = op.share(_bits(q[0]), keep)
        K = op.share(_bits(k[0]), keep)
        V = op.share(_bits(v[0]), keep)
        b = plan.bufs
        vs_pos = {h: i for i, h in enumerate(w.heads_of(wl.PAT_VS))}
        bs_pos = {h: i for i, h in enumerate(w.heads_of(wl.PAT_BS))}
        if vs_pos:
            idx = b["vs_index"]
            VI = op.share(idx.vidx[0].cpu().numpy(), keep)
            TV = op.share(idx.tvidx[0].cpu().numpy(), keep)
            tvcnt = idx.tvcnt[0].cpu().numpy()
            v_idx, s_idx = b["v_idx"][0].cpu().numpy(), b["s_idx"][0].cpu().numpy()
            grp, grp_cnt = idx.grp[0].cpu().numpy(), idx.grp_cnt[0].cpu().numpy()
            tgrp, tgrp_cnt = idx.tgrp[0].cpu().numpy(), idx.tgrp_cnt[0].cpu().numpy()
            vcnt = idx.vcnt[0].cpu().numpy()
            XI = op.share(xi.vidx[0].cpu().numpy(), keep)
            xcnt = xi.vcnt[0].cpu().numpy()
        if bs_pos:
            blk_idx, blk_cnt = b["blk_idx"][0].cpu().numpy(), b["blk_cnt"][0].cpu().numpy()
        tasks = []
        for h in range(w.Hq):
            t = dict(head=h, kv=h // w.group, N=w.N, d=w.d, Q=Q, K=K, V=V, rows=rows.numpy(),
                     o_rows=o_rows[h], lse_rows=lse_rows[h], last_q=w.last_q)
            if h in vs_pos:
                a = vs_pos[h]
                t.update(pattern="vs", k_v=w.k_v, k_s=w.k_s, v_idx=v_idx[a], s_idx=s_idx[a],
                         grp=grp[a, :grp_cnt[a]], tgrp=tgrp[a, :tgrp_cnt[a]], vcnt=vcnt[a], vidx=VI, slot=a,
                         tvcnt=tvcnt[a], tvidx=TV,
                         ox_rows=ox_rows[h], lsex_rows=lsex_rows[h], xcnt=xcnt[a], xidx=XI)
            elif h in bs_pos:
                a = bs_pos[h]
                t.update(pattern="bs", k_b=w.k_b, blk_idx=blk_idx[a], blk_cnt=blk_cnt[a])
            else:
                t.update(pattern="a", n_sink=w.n_sink, n_local=w.n_local)
            tasks.append(t)
        old = os.environ.get("OPENBLAS_NUM_THREADS")
        os.environ["OPENBLAS_NUM_THREADS"] = "1"
        try:
            with mp.get_context("spawn").Pool(processes=min(16, os.cpu_count() or 1)) as pool:
                results = pool.map(op.check_head, tasks, chunksize=1)
        finally:
            if old is None:
                os.environ.pop("OPENBLAS_NUM_THREADS", None)
            else:
                os.environ["OPENBLAS_NUM_THREADS"] = old
    finally:
        for s in keep:
            s.close()
            s.unlink()
    bad = [r for r in results if r["errors"]]
    flips = sum(r["flips"] for r in results)
    worst = max(r["max_abs"] for r in results if "max_abs" in r)
    print(f"\nconfig {cid} ({w.name}): {len(results)} heads, index flips within the gap rule: {flips}, "
          f"worst max-abs {worst:.3g}")
    assert not bad, bad[:3]
