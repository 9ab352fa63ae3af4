"""GPU parity of the one-launch mixed-pattern layer (minf_sparse_attn_layer):
every head against the oracle, and bit-identical to one launch per pattern
(the work items of a head are computed the same way in both)."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import layer, minf
from dynamic_sparse_attention_minf_b200 import workloads as wl
from oracle import minf_oracle as orc
from tests.parity import check_close, check_lse

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    minf.lib()


@pytest.mark.parametrize("N,d", [(1152, 128), (2048, 64)])
def test_fused_layer_matches_oracle_and_per_pattern_launches(N, d):
    pats = [wl.PAT_VS, wl.PAT_BS, wl.PAT_A, wl.PAT_VS, wl.PAT_BS, wl.PAT_VS, wl.PAT_A, wl.PAT_VS]
    w = wl.small(Hq=8, Hkv=2, N=N, d=d, seed=71, patterns=pats, k_v=48, k_s=80, k_b=5,
                 n_sink=32, n_local=200)
    q, k, v = wl.make_qkv(w, DEV)
    plan = layer.make_plan(w, DEV)
    o_f = torch.zeros_like(q)
    l_f = torch.zeros(q.shape[:3], dtype=torch.float32, device=DEV)
    layer.run_layer(plan, q, k, v, o_f, l_f, fused=True)
    o_s = torch.zeros_like(q)
    l_s = torch.zeros(q.shape[:3], dtype=torch.float32, device=DEV)
    layer.run_layer(plan, q, k, v, o_s, l_s, fused=False)
    torch.cuda.synchronize()
    assert layer.device_status(plan) == 0
    assert torch.equal(o_f, o_s) and torch.equal(l_f, l_s)
    qn, kn, vn = orc.to_f64(q[0]), orc.to_f64(k[0]), orc.to_f64(v[0])
    sc = orc.default_scale(d)
    V, S = plan.bufs["v_idx"][0].cpu().numpy(), plan.bufs["s_idx"][0].cpu().numpy()
    BI, BC = plan.bufs["blk_idx"][0].cpu().numpy(), plan.bufs["blk_cnt"][0].cpu().numpy()
    vs_pos = {h: i for i, h in enumerate(w.heads_of(wl.PAT_VS))}
    bs_pos = {h: i for i, h in enumerate(w.heads_of(wl.PAT_BS))}
    rows = np.arange(N)
    on, ln = o_f[0].float().cpu().numpy(), l_f[0].cpu().numpy()
    for h in range(w.Hq):
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        if h in vs_pos:
            a = vs_pos[h]
            fn = lambda r, a=a: orc.mask_vs(r, N, V[a], S[a])
        elif h in bs_pos:
            a = bs_pos[h]
            fn = lambda r, a=a: orc.mask_bs(r, N, BI[a], BC[a])
        else:
            fn = lambda r: orc.mask_ashape(r, N, w.n_sink, w.n_local)
        O, L = orc.attention_head(qn[h], kn[kv], vn[kv], rows, fn, sc)
        check_close(on[h], O, f"head {h}")
        check_lse(ln[h], L, f"head {h}")


def test_fused_layer_argument_checks():
    w = wl.small(Hq=4, Hkv=2, N=256, d=128, seed=72)
    q, k, v = wl.make_qkv(w, DEV)
    with pytest.raises(minf.MinfError):           # no head at all
        minf.minf_sparse_attn_layer(q, k, v)
    with pytest.raises(minf.MinfError):           # more heads than Hq
        minf.minf_sparse_attn_layer(q, k, v, a_heads=[0, 1, 2, 3, 0], n_sink=4, n_local=16)


def test_kv_group_halves_equal_the_full_layer():
    """The multi-GPU split of a layer by KV-head group, run here one rank
    after the other: each rank's heads (sliced inputs, its rows of the pattern
    table) reproduce those heads of the full layer bit for bit."""
    pats = [wl.PAT_VS, wl.PAT_BS, wl.PAT_A, wl.PAT_VS, wl.PAT_VS, wl.PAT_A, wl.PAT_BS, wl.PAT_VS]
    w = wl.small(Hq=8, Hkv=4, N=1024, d=128, seed=73, patterns=pats, k_v=40, k_s=72, k_b=4,
                 n_sink=16, n_local=160)
    q, k, v = wl.make_qkv(w, DEV)
    plan = layer.make_plan(w, DEV)
    o = torch.zeros_like(q)
    lse = torch.zeros(q.shape[:3], dtype=torch.float32, device=DEV)
    layer.run_layer(plan, q, k, v, o, lse)
    world = 2
    for rank in range(world):
        hq0, hq1, hk0, hk1 = layer.kv_group_slice(w, rank, world)
        lw = layer.local_workload(w, rank, world)
        lq, lk, lv = q[:, hq0:hq1].contiguous(), k[:, hk0:hk1].contiguous(), v[:, hk0:hk1].contiguous()
        lplan = layer.make_plan(lw, DEV)
        lo = torch.zeros_like(lq)
        llse = torch.zeros(lq.shape[:3], dtype=torch.float32, device=DEV)
        layer.run_layer(lplan, lq, lk, lv, lo, llse)
        torch.cuda.synchronize()
        assert layer.device_status(lplan) == 0
        assert torch.equal(lo, o[:, hq0:hq1]) and torch.equal(llse, lse[:, hq0:hq1]), f"rank {rank}"
