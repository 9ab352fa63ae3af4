"""Grid-pattern attention (NEXT-4) through the C ABI against the oracle: the
per-position Block-Sparse selections under the index rule, the outputs on
the Grid mask, and the case of one token per frame, which is plain
Block-Sparse attention."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import minf
from dynamic_sparse_attention_minf_b200 import workloads as wl
from oracle import minf_oracle as orc
from tests.parity import check_close, check_index_set, check_lse

pytestmark = pytest.mark.gpu


def _grid_case(w, heads, P, k_b):
    q, k, v = wl.make_qkv(w, "cuda")
    o, lse, bi, bc = minf.minf_attn_grid(q, k, v, heads, P, k_b, return_selection=True)
    torch.cuda.synchronize()
    sc = orc.default_scale(w.d)
    F = w.N // P
    for bb in range(w.B):
        qn, kn, vn = orc.to_f64(q[bb]), orc.to_f64(k[bb]), orc.to_f64(v[bb])
        gi, gc = bi[bb].cpu().numpy(), bc[bb].cpu().numpy()
        for hi, h in enumerate(heads):
            kv = orc.kv_head(h, w.Hq, w.Hkv)
            ri, rc = orc.grid_select(qn[h], kn[kv], P, sc, k_b)
            for p in range(P):
                t = orc.bs_scores(orc.bs_pool(qn[h][p::P]), orc.bs_pool(kn[kv][p::P]), sc)
                assert np.array_equal(gc[p, hi], rc[p])
                for b in range(F // 64):
                    check_index_set(gi[p, hi, b, :gc[p, hi, b]], ri[p][b, :rc[p][b]], t[b, :b + 1], forced=b,
                                    what=f"batch {bb} head {h} position {p} block {b}")
            sel_i = gi[:, hi]
            sel_c = gc[:, hi]
            rows = np.arange(w.N)
            oref, lref = orc.attention_head(qn[h], kn[kv], vn[kv], rows,
                                            lambda r: orc.mask_grid(r, w.N, P, sel_i, sel_c), sc)
            check_close(o[bb, h].float().cpu().numpy(), oref, what=f"O batch {bb} head {h}")
            check_lse(lse[bb, h].cpu().numpy(), lref, what=f"LSE batch {bb} head {h}")
    return q, k, v, o, lse


@pytest.mark.parametrize("P,d", [(4, 128), (2, 64)])
def test_grid_attention_matches_oracle(P, d):
    w = wl.small(Hq=4, Hkv=2, N=256 * P, d=d, seed=51 + P)
    _grid_case(w, [0, 3], P, 3)


def test_grid_attention_batch_of_two():
    w = wl.small(Hq=2, Hkv=1, N=768, d=128, seed=57, B=2)
    _grid_case(w, [1], 3, 2)


def test_grid_with_one_token_per_frame_is_block_sparse():
    """frame_tokens = 1: the permutation is the identity and the result is the
    Block-Sparse path's, bit for bit."""
    w = wl.small(Hq=4, Hkv=2, N=1024, d=128, seed=59)
    q, k, v = wl.make_qkv(w, "cuda")
    heads = [1, 2]
    og, lg, bi, bc = minf.minf_attn_grid(q, k, v, heads, 1, 5, return_selection=True)
    ws = minf.workspace(minf.OP_ESTIMATE_BS, minf.shape_of(q, k), 2, k_b=5)
    ri, rc = minf.minf_estimate_bs(q, k, heads, 5, ws=ws)
    ob, lb = minf.minf_sparse_attn_bs(q, k, v, heads, ri, rc)
    assert torch.equal(bi[:, 0], ri) and torch.equal(bc[:, 0], rc)
    for h in heads:
        assert torch.equal(og[:, h], ob[:, h]) and torch.equal(lg[:, h], lb[:, h])


def test_grid_rejects_frames_not_a_multiple_of_128():
    w = wl.small(Hq=2, Hkv=1, N=1024, d=128, seed=61)
    q, k, v = wl.make_qkv(w, "cuda")
    with pytest.raises(minf.MinfError):
        minf.minf_attn_grid(q, k, v, [0], 3, 2)      # 1024 is not a multiple of 3
    with pytest.raises(minf.MinfError):
        minf.minf_attn_grid(q, k, v, [0], 16, 2)     # 64 frames
