"""GPU parity: every C-ABI entry point against the CPU oracle on the same
seeded bf16 inputs (indices bit-exact up to the score-gap rule, attention
within max-abs 2e-2 / mean-abs 2e-3)."""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_minf_b200 import minf
from dynamic_sparse_attention_minf_b200 import workloads as wl
from oracle import minf_oracle as orc
from tests.parity import check_close, check_index_set, check_lse, tile_list_errors

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    minf.lib()


def _inputs(w):
    q, k, v = wl.make_qkv(w, DEV)
    return q, k, v, orc.to_f64(q[0]), orc.to_f64(k[0]), orc.to_f64(v[0])


def _check_attn(o, lse, qn, kn, vn, heads, w, mask_for_head, rows=None):
    N = w.N
    rows = np.arange(N) if rows is None else np.asarray(rows)
    sc = orc.default_scale(w.d)
    on = o[0].float().cpu().numpy()
    ln = lse[0].cpu().numpy()
    for hi, h in enumerate(heads):
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        O, L = orc.attention_head(qn[h], kn[kv], vn[kv], rows, mask_for_head(hi, h), sc)
        check_close(on[h][rows], O, f"head {h}")
        check_lse(ln[h][rows], L, f"head {h}")


# ------------------------------------------------------------------ dense
@pytest.mark.parametrize("Hq,Hkv,N,d", [(2, 1, 512, 64), (2, 2, 1024, 128), (4, 2, 640, 128)])
def test_dense_attention(Hq, Hkv, N, d):
    w = wl.small(Hq=Hq, Hkv=Hkv, N=N, d=d, seed=N + d)
    q, k, v, qn, kn, vn = _inputs(w)
    ws = minf.workspace(minf.OP_DENSE_ATTN, minf.shape_of(q, k), Hq)
    o, lse = minf.minf_dense_attn(q, k, v, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    _check_attn(o, lse, qn, kn, vn, range(Hq), w, lambda hi, h: (lambda r: orc.mask_dense(r, N)))


# ---------------------------------------------------------------- A-shape
@pytest.mark.parametrize("n_sink,n_local,N,d", [(64, 300, 1024, 128), (100, 129, 768, 64), (0, 64, 512, 128),
                                                (128, 4096, 1024, 128)])
def test_ashape_attention(n_sink, n_local, N, d):
    w = wl.small(Hq=4, Hkv=2, N=N, d=d, seed=3 + n_local)
    q, k, v, qn, kn, vn = _inputs(w)
    heads = [1, 2]
    ws = minf.workspace(minf.OP_ATTN_ASHAPE, minf.shape_of(q, k), 2)
    o, lse = minf.minf_attn_ashape(q, k, v, heads, n_sink, n_local, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    _check_attn(o, lse, qn, kn, vn, heads, w,
                lambda hi, h: (lambda r: orc.mask_ashape(r, N, n_sink, n_local)))


# --------------------------------------------------------- Vertical-Slash
def _vs_pipeline(w, heads, rows=None):
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(w.d)
    ws = minf.workspace(minf.OP_ESTIMATE_VS, minf.shape_of(q, k), len(heads))
    v_idx, s_idx, vs, ss = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, return_scores=True, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    gv, gs = v_idx[0].cpu().numpy(), s_idx[0].cpu().numpy()
    for hi, h in enumerate(heads):
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        rv, rs = orc.vs_estimate(qn[h][w.N - 64:], kn[kv], sc)
        np.testing.assert_allclose(vs[0, hi].cpu().numpy(), rv, rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(ss[0, hi].cpu().numpy(), rs, rtol=1e-4, atol=1e-7)
        ov, os_ = orc.vs_select(rv, rs, w.k_v, w.k_s)
        check_index_set(gv[hi], ov, rv, what=f"vertical h{h}")
        check_index_set(gs[hi], os_, rs, forced=0, what=f"slash h{h}")
    ws_i = minf.workspace(minf.OP_BUILD_INDEX, minf.shape_of(q, k), len(heads))
    index = minf.minf_build_index(minf.shape_of(q, k), v_idx, s_idx, ws=ws_i)
    ws_a = minf.workspace(minf.OP_SPARSE_ATTN_VS, minf.shape_of(q, k), len(heads))
    o, lse = minf.minf_sparse_attn_vs(q, k, v, heads, index, ws=ws_a)
    assert minf.minf_get_device_status(ws_i) == 0
    assert minf.minf_get_device_status(ws_a) == 0
    # index build is integer work: bit-exact against the oracle on the GPU's own V and S
    for hi in range(len(heads)):
        groups, vcnt, vidx = orc.vs_build_index(gv[hi], gs[hi], w.N)
        G = int(index.grp_cnt[0, hi])
        assert G == groups.shape[0]
        assert np.array_equal(index.grp[0, hi, :G].cpu().numpy(), groups)
        tg = orc.vs_groups(gs[hi], block=128)
        T = int(index.tgrp_cnt[0, hi])
        assert T == tg.shape[0] and np.array_equal(index.tgrp[0, hi, :T].cpu().numpy(), tg)
        assert np.array_equal(index.vcnt[0, hi].cpu().numpy(), vcnt)
        gvi = index.vidx[0, hi].cpu().numpy()
        for b in range(w.N // 64):
            assert np.array_equal(gvi[b, :vcnt[b]], vidx[b, :vcnt[b]]), f"block {b}"
        bad = tile_list_errors(index.tvcnt[0, hi].cpu().numpy(), index.tvidx[0, hi].cpu().numpy(), vcnt, vidx)
        assert not bad, f"tile gather lists differ in tiles {bad[:4]}"
    _check_attn(o, lse, qn, kn, vn, heads, w,
                lambda hi, h: (lambda r: orc.mask_vs(r, w.N, gv[hi], gs[hi])), rows)
    return gv, gs


@pytest.mark.parametrize("N", [2048, 1152])
def test_vs_pipeline_small(N):
    """N = 1152 is nine 128-row tiles: the last pair of query tiles has one tile."""
    w = wl.small(Hq=4, Hkv=2, N=N, d=128, seed=21, k_v=64, k_s=128)
    _vs_pipeline(w, [0, 3])


def test_vs_config0():
    """Vertical-Slash, H=1, N=4096, d=64, vertical 128 / slash 256, sink bias."""
    w = wl.config(0)
    _vs_pipeline(w, [0])


def test_vs_all_selected_equals_dense():
    """Closed form: with every column and every offset kept, VS is dense causal."""
    w = wl.small(Hq=2, Hkv=1, N=512, d=64, seed=5, k_v=512, k_s=512)
    q, k, v, *_ = _inputs(w)
    v_idx, s_idx = minf.minf_estimate_vs(q, k, [0, 1], 512, 512)
    assert torch.equal(v_idx[0, 0].cpu(), torch.arange(512, dtype=torch.int32))
    index = minf.minf_build_index(minf.shape_of(q, k), v_idx, s_idx)
    o, lse = minf.minf_sparse_attn_vs(q, k, v, [0, 1], index)
    od, ld = minf.minf_dense_attn(q, k, v)
    assert (o.float() - od.float()).abs().max().item() <= 1e-2
    assert (lse - ld).abs().max().item() <= 1e-3


def test_vs_index_from_oracle_sets():
    """build_index + attention on oracle-chosen sets with wide gaps and long groups."""
    w = wl.small(Hq=2, Hkv=1, N=4096, d=128, seed=8, k_v=300, k_s=700)
    q, k, v, qn, kn, vn = _inputs(w)
    rng = np.random.default_rng(0)
    S = np.unique(np.concatenate([[0], np.arange(1, 400), rng.choice(4096, 400, replace=False)]))[:700]
    V = np.unique(rng.choice(4096, 300, replace=False))
    assert S.size == 700 and V.size == 300
    v_idx = torch.tensor(np.stack([V, V])[None], dtype=torch.int32, device=DEV)
    s_idx = torch.tensor(np.stack([S, S])[None], dtype=torch.int32, device=DEV)
    index = minf.minf_build_index(minf.shape_of(q, k), v_idx, s_idx)
    ws_a = minf.workspace(minf.OP_SPARSE_ATTN_VS, minf.shape_of(q, k), 2)
    o, lse = minf.minf_sparse_attn_vs(q, k, v, [0, 1], index, ws=ws_a)
    assert minf.minf_get_device_status(ws_a) == 0
    _check_attn(o, lse, qn, kn, vn, [0, 1], w, lambda hi, h: (lambda r: orc.mask_vs(r, w.N, V, S)))


# ----------------------------------------------------------- Block-Sparse
def _bs_pipeline(w, heads, rows=None):
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(w.d)
    ws = minf.workspace(minf.OP_ESTIMATE_BS, minf.shape_of(q, k), len(heads))
    blk_idx, blk_cnt, t = minf.minf_estimate_bs(q, k, heads, w.k_b, return_scores=True, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    gi, gc = blk_idx[0].cpu().numpy(), blk_cnt[0].cpu().numpy()
    # with a workspace sized for the budget (d = 128): scores on the tensor
    # cores from the split means, one warp per row selecting; held to the
    # same rules against the oracle
    ws_f = minf.workspace(minf.OP_ESTIMATE_BS, minf.shape_of(q, k), len(heads), k_b=w.k_b)
    fi, fc, tf = minf.minf_estimate_bs(q, k, heads, w.k_b, return_scores=True, ws=ws_f)
    assert minf.minf_get_device_status(ws_f) == 0
    fi, fc = fi[0].cpu().numpy(), fc[0].cpu().numpy()
    nb = w.N // 64
    flips = 0
    for hi, h in enumerate(heads):
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        ri, rc = orc.bs_select(qn[h], kn[kv], sc, w.k_b)
        tref = orc.bs_scores(orc.bs_pool(qn[h]), orc.bs_pool(kn[kv]), sc)
        tg = t[0, hi].cpu().numpy()
        low = np.tril(np.ones((nb, nb), bool))
        np.testing.assert_allclose(tg[low], tref[low], rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(tf[0, hi].cpu().numpy()[low], tref[low], rtol=1e-4, atol=1e-5)
        for xi, xc, how in ((gi, gc, "fp32 FMA"), (fi, fc, "tensor cores")):
            assert np.array_equal(xc[hi], rc), how
            for b in range(nb):
                flips += check_index_set(xi[hi, b, :xc[hi, b]], ri[b, :rc[b]], tref[b, :b + 1], forced=b,
                                         what=f"{how} h{h} block {b}")
                assert (xi[hi, b, xc[hi, b]:] == -1).all(), how
    ws_a = minf.workspace(minf.OP_SPARSE_ATTN_BS, minf.shape_of(q, k), len(heads))
    o, lse = minf.minf_sparse_attn_bs(q, k, v, heads, blk_idx, blk_cnt, ws=ws_a)
    assert minf.minf_get_device_status(ws_a) == 0
    _check_attn(o, lse, qn, kn, vn, heads, w,
                lambda hi, h: (lambda r: orc.mask_bs(r, w.N, gi[hi], gc[hi])), rows)
    return flips


@pytest.mark.parametrize("N,d", [(2048, 128), (640, 128), (1152, 64), (8448, 128)])
def test_bs_pipeline_small(N, d):
    w = wl.small(Hq=4, Hkv=2, N=N, d=d, seed=4, bias="block", patterns=[wl.PAT_BS] * 4, k_b=7)
    _bs_pipeline(w, [1, 2])


def test_bs_config1_sampled_rows():
    """Block-Sparse, 8 heads (MHA), N=32768, d=128, top-64 blocks."""
    w = wl.config(1)
    rows = wl.sample_rows(w.N, 512, w.seed).numpy()
    _bs_pipeline(w, list(range(8)), rows)


@pytest.mark.parametrize("k_b", [1, 128])
def test_bs_fused_selection_long_rows(k_b):
    """The tensor-core path over several 128-block row tiles, at the largest
    budget it takes (a row's candidate list compacts several times) and at
    k_b = 1 (only the forced diagonal), against the oracle's selection."""
    w = wl.small(Hq=2, Hkv=1, N=32768, d=128, seed=17, bias="block", patterns=[wl.PAT_BS] * 2, k_b=k_b)
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(w.d)
    gi, gc = minf.minf_estimate_bs(q, k, [0, 1], k_b)
    gi, gc = gi[0].cpu().numpy(), gc[0].cpu().numpy()
    for h in range(2):
        ri, rc = orc.bs_select(qn[h], kn[0], sc, k_b)
        tref = orc.bs_scores(orc.bs_pool(qn[h]), orc.bs_pool(kn[0]), sc)
        assert np.array_equal(gc[h], rc)
        for b in range(w.N // 64):
            check_index_set(gi[h, b, :gc[h, b]], ri[b, :rc[b]], tref[b, :b + 1], forced=b, what=f"h{h} block {b}")
            assert (gi[h, b, gc[h, b]:] == -1).all()


def test_bs_fused_selection_all_ties():
    """Zero queries and keys: every pooled score ties, so each row keeps its
    diagonal block and the lowest other blocks."""
    N, k_b = 16384, 128
    q = torch.zeros(1, 2, N, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 1, N, 128, dtype=torch.bfloat16, device=DEV)
    gi, gc = minf.minf_estimate_bs(q, k, [0, 1], k_b)
    gi, gc = gi[0].cpu().numpy(), gc[0].cpu().numpy()
    z = np.zeros((N, 128))
    ri, rc = orc.bs_select(z, z, orc.default_scale(128), k_b)
    for h in range(2):
        assert np.array_equal(gc[h], rc)
        for b in range(N // 64):
            assert np.array_equal(gi[h, b, :gc[h, b]], ri[b, :rc[b]]), f"block {b}"


def test_bs_all_blocks_equals_dense():
    w = wl.small(Hq=2, Hkv=1, N=1024, d=128, seed=9, bias="block", patterns=[wl.PAT_BS] * 2, k_b=64)
    q, k, v, *_ = _inputs(w)
    blk_idx, blk_cnt = minf.minf_estimate_bs(q, k, [0, 1], 64)
    o, lse = minf.minf_sparse_attn_bs(q, k, v, [0, 1], blk_idx, blk_cnt)
    od, ld = minf.minf_dense_attn(q, k, v)
    assert (o.float() - od.float()).abs().max().item() <= 1e-2
    assert (lse - ld).abs().max().item() <= 1e-3


# -------------------------------------------------------------- edge cases
def test_vs_offset_zero_and_one_vertical():
    """k_s = 1 keeps only the forced offset 0 (block-diagonal bands) and k_v = 1 one column."""
    w = wl.small(Hq=2, Hkv=1, N=1024, d=64, seed=31, k_v=1, k_s=1)
    gv, gs = _vs_pipeline(w, [0, 1])
    assert (gs == 0).all()


def test_bs_diagonal_block_only():
    """k_b = 1: every query block attends to its own (forced) diagonal block only."""
    w = wl.small(Hq=2, Hkv=1, N=1024, d=128, seed=32, bias="block", patterns=[wl.PAT_BS] * 2, k_b=1)
    _bs_pipeline(w, [0, 1])


@pytest.mark.parametrize("d", [64, 128])
def test_minimum_size_one_tile(d):
    """N = 128: one query tile, one key tile, for every pattern."""
    w = wl.small(Hq=2, Hkv=1, N=128, d=d, seed=33, k_v=16, k_s=8)
    _vs_pipeline(w, [0, 1])
    wb = wl.small(Hq=2, Hkv=1, N=128, d=d, seed=34, bias="block", patterns=[wl.PAT_BS] * 2, k_b=2)
    _bs_pipeline(wb, [0, 1])
    q, k, v, qn, kn, vn = _inputs(w)
    o, lse = minf.minf_attn_ashape(q, k, v, [0, 1], 16, 32)
    _check_attn(o, lse, qn, kn, vn, [0, 1], w, lambda hi, h: (lambda r: orc.mask_ashape(r, w.N, 16, 32)))
    o, lse = minf.minf_dense_attn(q, k, v)
    _check_attn(o, lse, qn, kn, vn, [0, 1], w, lambda hi, h: (lambda r: orc.mask_dense(r, w.N)))


@pytest.mark.parametrize("last_q,d", [(1, 64), (17, 128), (32, 64), (64, 128)])
def test_vs_estimation_last_rows(last_q, d):
    """Fewer than 64 scoring rows: the rows before the last `last_q` are masked
    in both passes, scores and sets match the oracle fed only those rows."""
    N = 1280
    w = wl.small(Hq=4, Hkv=2, N=N, d=d, seed=36, k_v=100, k_s=200)
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(d)
    heads = [3, 0]
    ws = minf.workspace(minf.OP_ESTIMATE_VS, minf.shape_of(q, k), 2)
    v_idx, s_idx, vs, ss = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, last_q=last_q,
                                                 return_scores=True, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    gv, gs = v_idx[0].cpu().numpy(), s_idx[0].cpu().numpy()
    for hi, h in enumerate(heads):
        kv = orc.kv_head(h, w.Hq, w.Hkv)
        rv, rs = orc.vs_estimate(qn[h][N - last_q:], kn[kv], sc)
        np.testing.assert_allclose(vs[0, hi].cpu().numpy(), rv, rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(ss[0, hi].cpu().numpy(), rs, rtol=1e-4, atol=1e-7)
        ov, os_ = orc.vs_select(rv, rs, w.k_v, w.k_s)
        check_index_set(gv[hi], ov, rv, what=f"vertical h{h}")
        check_index_set(gs[hi], os_, rs, forced=0, what=f"slash h{h}")


def test_vs_estimation_bit_reproducible():
    """Fixed-order sums: two runs give identical scores, bit for bit."""
    w = wl.small(Hq=2, Hkv=1, N=4096, d=128, seed=37)
    q, k, v = wl.make_qkv(w, DEV)
    runs = [minf.minf_estimate_vs(q, k, [0, 1], 300, 600, return_scores=True) for _ in range(2)]
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("N,k_v,k_s", [(65536, 1000, 3000), (131072, 2000, 6000)])
def test_vs_estimation_long_rows(N, k_v, k_s):
    """Rows longer than 32K take the many-CTA top-k (several segments per row)."""
    w = wl.small(Hq=2, Hkv=1, N=N, d=64, seed=35, k_v=k_v, k_s=k_s)
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(w.d)
    ws = minf.workspace(minf.OP_ESTIMATE_VS, minf.shape_of(q, k), 2)
    v_idx, s_idx, vs, ss = minf.minf_estimate_vs(q, k, [0, 1], k_v, k_s, return_scores=True, ws=ws)
    assert minf.minf_get_device_status(ws) == 0
    gv, gs = v_idx[0].cpu().numpy(), s_idx[0].cpu().numpy()
    for h in range(2):
        rv, rs = orc.vs_estimate(qn[h][N - 64:], kn[0], sc)
        np.testing.assert_allclose(vs[0, h].cpu().numpy(), rv, rtol=1e-4, atol=1e-7)
        ov, os_ = orc.vs_select(rv, rs, k_v, k_s)
        assert np.all(np.diff(gv[h]) > 0) and np.all(np.diff(gs[h]) > 0)
        check_index_set(gv[h], ov, rv, what=f"vertical h{h}")
        check_index_set(gs[h], os_, rs, forced=0, what=f"slash h{h}")


# ------------------------------------------- element-exact Vertical-Slash
def _vs_exact_check(w, heads, V_sets, S_sets, q, k, v, qn, kn, vn):
    """Build the exact index from per-head (V, S), check it bit-exactly against
    the oracle's, run the exact attention and compare with mask_vs_exact."""
    k_v = max(len(x) for x in V_sets)
    k_s = max(len(x) for x in S_sets)
    assert all(len(x) == k_v for x in V_sets) and all(len(x) == k_s for x in S_sets)
    v_idx = torch.tensor(np.stack(V_sets)[None], dtype=torch.int32, device=DEV)
    s_idx = torch.tensor(np.stack(S_sets)[None], dtype=torch.int32, device=DEV)
    shp = minf.shape_of(q, k)
    ws_i = minf.workspace(minf.OP_BUILD_INDEX_EXACT, shp, len(heads))
    index = minf.minf_build_index_exact(shp, v_idx, s_idx, ws=ws_i)
    assert minf.minf_get_device_status(ws_i) == 0
    nt = w.N // 128
    for hi in range(len(heads)):
        V, S = np.asarray(V_sets[hi]), np.asarray(S_sets[hi])
        groups, vcnt, vidx = orc.vs_exact_index(V, S, w.N)
        T = int(index.tgrp_cnt[0, hi])
        assert T == groups.shape[0] and np.array_equal(index.tgrp[0, hi, :T].cpu().numpy(), groups)
        assert np.array_equal(index.vcnt[0, hi].cpu().numpy(), vcnt)
        gvi = index.vidx[0, hi].cpu().numpy()
        for t in range(nt):
            assert np.array_equal(gvi[t, :vcnt[t]], vidx[t, :vcnt[t]]), f"tile {t}"
        sb = index.sbits[0, hi].cpu().numpy().view(np.uint32)
        vb = index.vbits[0, hi].cpu().numpy().view(np.uint32)
        bits = lambda words, n: np.unpackbits(words.view(np.uint8), bitorder="little")[:n].astype(bool)
        ref_s = np.zeros(w.N, bool); ref_s[S] = True
        ref_v = np.zeros(w.N, bool); ref_v[V] = True
        assert np.array_equal(bits(sb, w.N), ref_s) and not bits(sb, 32 * sb.size)[w.N:].any()
        assert np.array_equal(bits(vb, w.N), ref_v) and not bits(vb, 32 * vb.size)[w.N:].any()
    ws_a = minf.workspace(minf.OP_SPARSE_ATTN_VS_EXACT, shp, len(heads))
    o, lse = minf.minf_sparse_attn_vs_exact(q, k, v, heads, index, ws=ws_a)
    assert minf.minf_get_device_status(ws_a) == 0
    _check_attn(o, lse, qn, kn, vn, heads, w,
                lambda hi, h: (lambda r: orc.mask_vs_exact(r, w.N, V_sets[hi], S_sets[hi])))
    return o, lse


@pytest.mark.parametrize("N", [2048, 896])
def test_vs_exact_pipeline_small(N):
    """Estimated V and S (GPU top-k, checked against the oracle), then the exact variant."""
    w = wl.small(Hq=4, Hkv=2, N=N, d=128, seed=41, k_v=64, k_s=128)
    q, k, v, qn, kn, vn = _inputs(w)
    sc = orc.default_scale(w.d)
    heads = [1, 2]
    v_idx, s_idx = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s)
    gv, gs = v_idx[0].cpu().numpy(), s_idx[0].cpu().numpy()
    for hi, h in enumerate(heads):
        rv, rs = orc.vs_estimate(qn[h][w.N - 64:], kn[orc.kv_head(h, w.Hq, w.Hkv)], sc)
        ov, os_ = orc.vs_select(rv, rs, w.k_v, w.k_s)
        check_index_set(gv[hi], ov, rv, what=f"vertical h{h}")
        check_index_set(gs[hi], os_, rs, forced=0, what=f"slash h{h}")
    _vs_exact_check(w, heads, list(gv), list(gs), q, k, v, qn, kn, vn)


@pytest.mark.parametrize("d", [64, 128])
def test_vs_exact_oracle_sets(d):
    """Oracle-chosen sets: a long run of small offsets, scattered offsets with
    wide gaps, and verticals inside and outside the offset ranges."""
    w = wl.small(Hq=2, Hkv=1, N=4096, d=d, seed=42 + d)
    q, k, v, qn, kn, vn = _inputs(w)
    rng = np.random.default_rng(d)
    S = np.unique(np.concatenate([[0], np.arange(1, 300), rng.choice(4096, 300, replace=False)]))[:500]
    V = np.unique(rng.choice(4096, 200, replace=False))[:180]
    S2 = np.unique(np.concatenate([[0], rng.choice(4096, 600, replace=False)]))[:500]
    V2 = np.unique(np.concatenate([np.arange(0, 64), rng.choice(4096, 200, replace=False)]))[:180]
    _vs_exact_check(w, [0, 1], [V, V2], [S, S2], q, k, v, qn, kn, vn)


def test_vs_exact_all_offsets_equals_dense():
    w = wl.small(Hq=2, Hkv=1, N=512, d=64, seed=43)
    q, k, v, qn, kn, vn = _inputs(w)
    V = np.arange(8)
    S = np.arange(512)
    o, lse = _vs_exact_check(w, [0, 1], [V, V], [S, S], q, k, v, qn, kn, vn)
    od, ld = minf.minf_dense_attn(q, k, v)
    assert (o.float() - od.float()).abs().max().item() <= 1e-2
    assert (lse - ld).abs().max().item() <= 1e-3


def test_vs_exact_minimum_size():
    w = wl.small(Hq=2, Hkv=1, N=128, d=128, seed=44)
    q, k, v, qn, kn, vn = _inputs(w)
    _vs_exact_check(w, [0, 1], [np.array([3, 77]), np.array([0, 127])],
                    [np.array([0, 5, 64]), np.array([0, 1, 2])], q, k, v, qn, kn, vn)


def test_pipelined_layer_matches_direct_run():
    """layer.run_pipelined (host inputs, two device buffer sets, copy streams)
    produces the same output as run_layer on device inputs."""
    from dynamic_sparse_attention_minf_b200 import layer
    w = wl.small(Hq=4, Hkv=2, N=1024, d=128, seed=51, k_v=64, k_s=96, k_b=4, n_sink=16, n_local=128,
                 patterns=[wl.PAT_VS, wl.PAT_BS, wl.PAT_A, wl.PAT_VS])
    q, k, v = wl.make_qkv(w, DEV)
    plan = layer.make_plan(w, DEV)
    o_ref = torch.empty_like(q)
    layer.run_layer(plan, q, k, v, o_ref)
    torch.cuda.synchronize()
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    bufs = layer.PipelineBuffers(hq, hk, hv, ho, DEV)
    layer.run_pipelined(plan, hq, hk, hv, ho, 3, bufs)
    torch.cuda.synchronize()
    assert layer.device_status(plan) == 0
    assert torch.equal(ho, o_ref.cpu())


# ------------------------------------------------------------- batch > 1
def test_batch_of_two_every_entry_point():
    """B = 2: every entry point, each batch element against the oracle on its
    own inputs (the kernels index the batch by grid z)."""
    w = wl.small(Hq=4, Hkv=2, N=1024, d=128, seed=61, k_v=48, k_s=96, k_b=4, B=2)
    q, k, v = wl.make_qkv(w, DEV)
    assert q.shape[0] == 2
    sc = orc.default_scale(w.d)
    shp = minf.shape_of(q, k)
    heads = [1, 2]
    # Vertical-Slash: estimation, index, attention (band and exact)
    v_idx, s_idx, vsc, ssc = minf.minf_estimate_vs(q, k, heads, w.k_v, w.k_s, return_scores=True)
    index = minf.minf_build_index(shp, v_idx, s_idx)
    o_vs, l_vs = minf.minf_sparse_attn_vs(q, k, v, heads, index)
    xi = minf.minf_build_index_exact(shp, v_idx, s_idx)
    o_x, l_x = minf.minf_sparse_attn_vs_exact(q, k, v, heads, xi)
    # Block-Sparse, A-shape, dense
    blk_idx, blk_cnt = minf.minf_estimate_bs(q, k, heads, w.k_b)
    o_bs, l_bs = minf.minf_sparse_attn_bs(q, k, v, heads, blk_idx, blk_cnt)
    o_a, l_a = minf.minf_attn_ashape(q, k, v, heads, 16, 100)
    o_d, l_d = minf.minf_dense_attn(q, k, v)
    torch.cuda.synchronize()
    rows = np.arange(w.N)
    for bb in range(2):
        qn, kn, vn = orc.to_f64(q[bb]), orc.to_f64(k[bb]), orc.to_f64(v[bb])
        gv, gs = v_idx[bb].cpu().numpy(), s_idx[bb].cpu().numpy()
        gi, gc = blk_idx[bb].cpu().numpy(), blk_cnt[bb].cpu().numpy()
        for hi, h in enumerate(heads):
            kv = orc.kv_head(h, w.Hq, w.Hkv)
            rv, rs = orc.vs_estimate(qn[h][w.N - 64:], kn[kv], sc)
            np.testing.assert_allclose(vsc[bb, hi].cpu().numpy(), rv, rtol=1e-4, atol=1e-7)
            ov, os_ = orc.vs_select(rv, rs, w.k_v, w.k_s)
            check_index_set(gv[hi], ov, rv, what=f"b{bb} vertical h{h}")
            check_index_set(gs[hi], os_, rs, forced=0, what=f"b{bb} slash h{h}")
            cases = [
                (o_vs, l_vs, lambda r: orc.mask_vs(r, w.N, gv[hi], gs[hi]), "vs"),
                (o_x, l_x, lambda r: orc.mask_vs_exact(r, w.N, gv[hi], gs[hi]), "vs exact"),
                (o_bs, l_bs, lambda r: orc.mask_bs(r, w.N, gi[hi], gc[hi]), "bs"),
                (o_a, l_a, lambda r: orc.mask_ashape(r, w.N, 16, 100), "a-shape"),
                (o_d, l_d, lambda r: orc.mask_dense(r, w.N), "dense"),
            ]
            for o, l, mfn, name in cases:
                O, L = orc.attention_head(qn[h], kn[kv], vn[kv], rows, mfn, sc)
                check_close(o[bb, h].float().cpu().numpy(), O, f"b{bb} {name} h{h}")
                check_lse(l[bb, h].cpu().numpy(), L, f"b{bb} {name} h{h}")
