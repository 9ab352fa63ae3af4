"""The offline pattern search on the GPU against the oracle: every trial's
kept share of the dense attention equals the oracle's on the masks of the
same indices, and each head's choice is the oracle's best within the budget
(or ties it within the tolerance)."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import minf, search
from dynamic_sparse_attention_minf_b200 import workloads as wl
from oracle import minf_oracle as orc

pytestmark = pytest.mark.gpu
TOL = 2e-2  # kept shares come from LSEs within 1e-2 of the oracle's


def _oracle_kept(q, k, h, kv, rows, pattern, setting, N, qg, kg):
    sc = orc.default_scale(q.shape[1])
    if pattern == "a_shape":
        mask = orc.mask_ashape(rows, N, *setting)
    elif pattern == "vertical_slash":
        v_idx, s_idx = minf.minf_estimate_vs(qg, kg, [h], *setting)
        mask = orc.mask_vs(rows, N, v_idx[0, 0].cpu().numpy(), s_idx[0, 0].cpu().numpy())
    else:
        bi, bc = minf.minf_estimate_bs(qg, kg, [h], setting)
        mask = orc.mask_bs(rows, N, bi[0, 0].cpu().numpy(), bc[0, 0].cpu().numpy())
    return float(orc.kept_mass(q[rows], k, rows, mask, sc).mean())


def test_search_matches_oracle_kept_mass():
    N = 4096
    w = wl.small(Hq=4, Hkv=2, N=N, d=128, seed=41, bias="sink+band")
    qg, kg, vg = wl.make_qkv(w, "cuda")
    rows = wl.sample_rows(N, 96, w.seed).numpy()
    cands = {"a_shape": [(64, 256), (64, 1024)], "vertical_slash": [(32, 64), (64, 256)],
             "block_sparse": [2, 6]}
    res = search.search_patterns(qg, kg, vg, candidates=cands, reference=("vertical_slash", (64, 128)),
                                 rows=rows)
    qn, kn = orc.to_f64(qg[0]), orc.to_f64(kg[0])
    for r in res:
        h = r.head
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        assert r.budget_tiles > 0 and len(r.trials) == 6
        ref = {}
        for t in r.trials:
            assert t.tiles > 0
            ok = _oracle_kept(qn[h], kn[kv], h, kv, rows, t.pattern, t.setting, N, qg, kg)
            assert abs(t.kept - ok) <= TOL, (h, t, ok)
            ref[(t.pattern, t.setting)] = ok
        fit = search.choose([search.Trial(t.pattern, t.setting, t.tiles, ref[(t.pattern, t.setting)])
                             for t in r.trials], r.budget_tiles)
        assert r.choice is not None and fit is not None
        assert ref[(r.choice.pattern, r.choice.setting)] >= ref[(fit.pattern, fit.setting)] - 2 * TOL


def test_full_masks_keep_everything():
    """An A-shape window over the whole prompt keeps all of the attention."""
    N = 2048
    w = wl.small(Hq=2, Hkv=1, N=N, d=64, seed=43)
    qg, kg, vg = wl.make_qkv(w, "cuda")
    ev = search.Evaluator(qg, kg, vg)
    for h in range(2):
        tiles, kept = ev.run(h, "a_shape", (0, N))
        assert tiles == (N // 128) * (N // 128 + 1) // 2
        assert kept == pytest.approx(1.0, abs=1e-3)
