"""Pins for the CPU oracle: each check comes from something other than the
oracle itself (a hand-derived fixture, a library routine, a closed form, an
invariant, planted structure, or brute force written as plain loops)."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import minf_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "masks_small.txt")


def _golden_cases():
    cases = {}
    name = None
    for line in open(GOLDEN):
        line = line.rstrip("\n")
        if not line or line.startswith("#"):
            continue
        if line.startswith("case "):
            parts = line.split()
            name = parts[1]
            params = dict(p.split("=") for p in parts[2:])
            cases[name] = (params, [])
        else:
            cases[name][1].append([int(t) for t in line.split()])
    return cases


def _to_mask(rows_lists, N):
    m = np.zeros((len(rows_lists), N), bool)
    for i, js in enumerate(rows_lists):
        m[i, js] = True
    return m


# ----------------------------------------------------------------- masks

def test_golden_ashape_mask():
    p, rows = _golden_cases()["ashape"]
    N = int(p["N"])
    got = orc.mask_ashape(np.arange(N), N, int(p["n_sink"]), int(p["n_local"]))
    assert np.array_equal(got, _to_mask(rows, N))


def test_golden_vs_mask():
    p, rows = _golden_cases()["vs"]
    N, blk = int(p["N"]), int(p["block"])
    V = [int(x) for x in p["V"].split(",")]
    S = [int(x) for x in p["S"].split(",")]
    got = orc.mask_vs(np.arange(N), N, V, S, block=blk)
    assert np.array_equal(got, _to_mask(rows, N))


def test_golden_vs_exact_mask():
    p, rows = _golden_cases()["vs_exact"]
    N = int(p["N"])
    V = [int(x) for x in p["V"].split(",")]
    S = [int(x) for x in p["S"].split(",")]
    got = orc.mask_vs_exact(np.arange(N), N, V, S)
    assert np.array_equal(got, _to_mask(rows, N))


def test_golden_bs_mask():
    p, rows = _golden_cases()["bs"]
    N, blk = int(p["N"]), int(p["block"])
    sels = [[int(x) for x in p[f"sel{b}"].split(",")] for b in range(N // blk)]
    k = max(len(s) for s in sels)
    idx = np.full((len(sels), k), -1)
    for b, s in enumerate(sels):
        idx[b, :len(s)] = s
    cnt = np.array([len(s) for s in sels])
    got = orc.mask_bs(np.arange(N), N, idx, cnt, block=blk)
    assert np.array_equal(got, _to_mask(rows, N))


@pytest.mark.parametrize("N", [64, 192, 320])
def test_masks_reduce_to_causal(N):
    """All-selected closed forms: every pattern with everything kept is causal."""
    rows = np.arange(N)
    dense = np.tril(np.ones((N, N), bool))
    assert np.array_equal(orc.mask_dense(rows, N), dense)
    assert np.array_equal(orc.mask_ashape(rows, N, 0, N), dense)
    assert np.array_equal(orc.mask_ashape(rows, N, N, 1), dense)
    assert np.array_equal(orc.mask_vs(rows, N, np.arange(N), [0]), dense)
    assert np.array_equal(orc.mask_vs(rows, N, [], np.arange(N)), dense)
    nb = N // 64
    idx = np.tile(np.arange(nb), (nb, 1))
    cnt = np.arange(1, nb + 1)
    idx = np.where(np.arange(nb)[None, :] < cnt[:, None], idx, -1)
    assert np.array_equal(orc.mask_bs(rows, N, idx, cnt), dense)


def test_vs_mask_offset0_is_block_diagonal_causal():
    N = 256
    m = orc.mask_vs(np.arange(N), N, [], [0])
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    assert np.array_equal(m, (j <= i) & (i // 64 == j // 64))


def test_vs_mask_covers_exact_diagonals():
    """Every element on a selected diagonal (i - j = o) lies in the mask."""
    rng = np.random.default_rng(3)
    N = 512
    S = np.unique(np.concatenate([[0], rng.choice(N, 20, replace=False)]))
    V = np.unique(rng.choice(N, 12, replace=False))
    m = orc.mask_vs(np.arange(N), N, V, S)
    for o in S:
        i = np.arange(o, N)
        assert m[i, i - o].all()
    for j in V:
        assert m[np.arange(j, N), j].all()
    assert not m[np.triu_indices(N, 1)].any()


# ------------------------------------------------------------- attention

def _sdpa_ref(q, k, v):
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)[0, 0].numpy()


@pytest.mark.parametrize("N,d", [(37, 8), (200, 16), (257, 32)])
def test_dense_attention_matches_library(N, d):
    rng = np.random.default_rng(N)
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    O, L = orc.attention_head(q, k, v, np.arange(N), lambda r: orc.mask_dense(r, N),
                              orc.default_scale(d))
    assert np.allclose(O, _sdpa_ref(q, k, v), atol=1e-12, rtol=1e-10)
    s = (q @ k.T) / math.sqrt(d)
    from scipy.special import logsumexp
    ref_lse = np.array([logsumexp(s[i, :i + 1]) for i in range(N)])
    assert np.allclose(L, ref_lse, atol=1e-12)


def test_masked_attention_bruteforce_loops():
    """Arbitrary mask vs plain Python loops (math.exp), including an empty row."""
    rng = np.random.default_rng(11)
    N, d = 12, 3
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    mask = rng.random((N, N)) < 0.5
    mask[4] = False
    scale = 0.7
    O, L = orc.attention_rows(q, k, v, mask, scale)
    for i in range(N):
        js = [j for j in range(N) if mask[i, j]]
        if not js:
            assert np.all(O[i] == 0) and L[i] == -np.inf
            continue
        s = [scale * sum(q[i, t] * k[j, t] for t in range(d)) for j in js]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        for t in range(d):
            ref = sum(w[a] * v[js[a], t] for a in range(len(js))) / tot
            assert abs(O[i, t] - ref) < 1e-12
        assert abs(L[i] - (mx + math.log(tot))) < 1e-12


def test_sparse_with_all_indices_equals_dense():
    """Closed form: VS with every column (and BS with every block) is dense causal."""
    rng = np.random.default_rng(5)
    N, d = 256, 16
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    sc = orc.default_scale(d)
    rows = np.arange(N)
    Od, Ld = orc.attention_head(q, k, v, rows, lambda r: orc.mask_dense(r, N), sc)
    V, S = orc.vs_select(*orc.vs_estimate(q[-64:], k, sc), N, N)
    Ov, Lv = orc.attention_head(q, k, v, rows, lambda r: orc.mask_vs(r, N, V, S), sc)
    assert np.allclose(Ov, Od, atol=1e-12) and np.allclose(Lv, Ld, atol=1e-12)
    idx, cnt = orc.bs_select(q, k, sc, N // 64)
    Ob, Lb = orc.attention_head(q, k, v, rows, lambda r: orc.mask_bs(r, N, idx, cnt), sc)
    assert np.allclose(Ob, Od, atol=1e-12) and np.allclose(Lb, Ld, atol=1e-12)


# ------------------------------------------------------- VS estimation

def test_vs_estimate_bruteforce_loops():
    rng = np.random.default_rng(2)
    N, L, d = 40, 8, 4
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    scale = 0.5
    v, sg = orc.vs_estimate(q[N - L:], k, scale, row_chunk=3)
    vr = [0.0] * N
    sr = [0.0] * N
    for i in range(N - L, N):
        s = [scale * sum(q[i, t] * k[j, t] for t in range(d)) for j in range(i + 1)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        for j in range(i + 1):
            vr[j] += e[j] / tot
            sr[i - j] += e[j] / tot
    assert np.allclose(v, vr, atol=1e-13) and np.allclose(sg, sr, atol=1e-13)


def test_vs_estimate_mass_closed_form():
    """Each of the L rows is a probability distribution: both score vectors sum to L."""
    rng = np.random.default_rng(4)
    N, d = 1000, 32
    q, k = rng.standard_normal((64, d)), rng.standard_normal((N, d))
    v, sg = orc.vs_estimate(q, k, 1 / math.sqrt(d))
    assert abs(v.sum() - 64) < 1e-9 and abs(sg.sum() - 64) < 1e-9
    assert (v >= 0).all() and (sg >= 0).all()
    # the last row sees every key: column N-1 only gets that row's mass
    assert v[N - 1] < 1.0


def test_vs_estimate_single_last_row():
    """One scoring row (the last, i = N - 1): v is that row's softmax and the
    slash score of offset o is the entry of key N - 1 - o, so sigma is v
    reversed; the softmax itself is scipy's."""
    from scipy.special import softmax
    rng = np.random.default_rng(5)
    N, d = 300, 16
    q, k = rng.standard_normal((1, d)), rng.standard_normal((N, d))
    sc = 1 / math.sqrt(d)
    v, sg = orc.vs_estimate(q, k, sc)
    assert np.allclose(v, softmax(sc * (k @ q[0])), atol=1e-14)
    assert np.allclose(sg, v[::-1], atol=1e-14)


def test_vs_planted_column_and_diagonal():
    rng = np.random.default_rng(9)
    N, d = 1024, 32
    q = rng.standard_normal((N, d))
    k = 0.05 * rng.standard_normal((N, d))
    u = q[N - 64:].mean(axis=0)
    j_star = 137
    k[j_star] = 6.0 * u / np.linalg.norm(u) * math.sqrt(d)
    V, _ = orc.vs_select(*orc.vs_estimate(q[N - 64:], k, 1 / math.sqrt(d)), 1, 1)
    assert V.tolist() == [j_star]

    o_star = 300
    k2 = 0.05 * rng.standard_normal((N, d))
    k2[: N - o_star] = 1.5 * q[o_star:]          # k_j aligned with q_{j + o*}
    v2, s2 = orc.vs_estimate(q[N - 64:], k2, 1 / math.sqrt(d))
    _, S = orc.vs_select(v2, s2, 1, 2)
    assert S.tolist() == [0, o_star]


# ------------------------------------------------------------ selection

@pytest.mark.parametrize("seed", range(6))
def test_select_topk_equals_full_sort(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    scores = rng.integers(0, 12, n).astype(np.float64)       # many ties
    k = int(rng.integers(1, n + 3))
    forced = int(rng.integers(0, n)) if seed % 2 else None
    got = orc.select_topk(scores, k, forced=forced)
    key = [(-(math.inf if j == forced else scores[j]), j) for j in range(n)]
    ref = sorted(j for _, j in sorted(key)[:min(k, n)])
    assert got.tolist() == ref


def test_select_topk_rows_matches_rowwise():
    rng = np.random.default_rng(1)
    R, C, k = 40, 40, 7
    scores = rng.integers(-5, 5, (R, C)).astype(np.float64)
    valid = np.arange(C)[None, :] <= np.arange(R)[:, None]
    idx, cnt = orc.select_topk_rows(scores, valid, k, forced_col=np.arange(R))
    for r in range(R):
        ref = orc.select_topk(scores[r, : r + 1], k, forced=r)
        assert cnt[r] == min(k, r + 1)
        assert idx[r, : cnt[r]].tolist() == ref.tolist()
        assert (idx[r, cnt[r]:] == -1).all()


# ------------------------------------------------------- BS estimation

def test_bs_pool_loops():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((256, 5))
    p = orc.bs_pool(x)
    for b in range(4):
        for t in range(5):
            assert abs(p[b, t] - sum(x[64 * b + r, t] for r in range(64)) / 64) < 1e-14


def test_bs_select_planted_and_forced_diagonal():
    rng = np.random.default_rng(8)
    N, d = 64 * 16, 16
    q = rng.standard_normal((N, d))
    k = rng.standard_normal((N, d))
    dirn = rng.standard_normal(d)
    q[64 * 12: 64 * 13] += 4 * dirn                 # query block 12
    k[64 * 3: 64 * 4] += 4 * dirn                   # key block 3
    idx, cnt = orc.bs_select(q, k, 1 / math.sqrt(d), 2)
    assert idx[12].tolist() == [3, 12]
    nb = N // 64
    for b in range(nb):
        assert cnt[b] == min(b + 1, 2)
        assert b in idx[b, : cnt[b]].tolist()
        assert (idx[b, : cnt[b]] <= b).all()


def test_bs_select_all_blocks_closed_form():
    rng = np.random.default_rng(6)
    N, d = 64 * 9, 8
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    idx, cnt = orc.bs_select(q, k, 0.3, 100)
    for b in range(9):
        assert cnt[b] == b + 1 and idx[b, : b + 1].tolist() == list(range(b + 1))


def test_bs_select_subset_of_blocks_bruteforce_loops():
    """Selection restricted to a subset of query blocks (given out of order,
    not contiguous), against plain loops: pooled means, scores for c <= b,
    diagonal forced, ranked by (score desc, index asc), first k ascending."""
    rng = np.random.default_rng(12)
    nb, d, k_b = 12, 6, 4
    q = rng.standard_normal((64 * nb, d))
    k = rng.standard_normal((64 * nb, d))
    blocks = [9, 2, 11, 5, 0, 7]
    sc = 0.7
    idx, cnt = orc.bs_select(q, k, sc, k_b, blocks=blocks)
    idx_p, cnt_p = orc.bs_select_pooled(orc.bs_pool(q), orc.bs_pool(k), sc, k_b, blocks=blocks)
    assert np.array_equal(idx, idx_p) and np.array_equal(cnt, cnt_p)
    mean = lambda x, b, t: sum(x[64 * b + r, t] for r in range(64)) / 64
    for row, b in enumerate(blocks):
        cand = []
        for c in range(b + 1):
            s = sc * sum(mean(q, b, t) * mean(k, c, t) for t in range(d))
            cand.append((-math.inf if c == b else -s, c))
        chosen = sorted(c for _, c in sorted(cand)[: min(k_b, b + 1)])
        assert cnt[row] == len(chosen)
        assert idx[row, : cnt[row]].tolist() == chosen, (b, idx[row], chosen)
        assert (idx[row, cnt[row]:] == -1).all()


# ------------------------------------------------------ VS index build

def test_vs_groups_loops():
    s = [0, 10, 74, 75, 140, 205, 206, 400, 464, 529, 1000]
    got = orc.vs_groups(np.array(s)).tolist()
    ref = []
    a = b = s[0]
    for o in s[1:]:
        if o - b <= 64:
            b = o
        else:
            ref.append([a, b])
            a = b = o
    ref.append([a, b])
    assert got == ref


@pytest.mark.parametrize("seed", range(4))
def test_vs_index_reproduces_mask(seed):
    """Index invariants: (groups, per-block verticals) describe exactly the
    definitional VS mask, and no key appears twice in a block."""
    rng = np.random.default_rng(seed)
    N = 64 * 12
    S = np.unique(np.concatenate([[0], rng.choice(N, 25 + 10 * seed, replace=False)]))
    V = np.unique(rng.choice(N, 30, replace=False))
    groups, vcnt, vidx = orc.vs_build_index(V, S, N)
    ref = orc.mask_vs(np.arange(N), N, V, S)
    got = np.zeros((N, N), bool)
    for i in range(N):
        b = i // 64
        r0 = 64 * b
        band = np.zeros(N, bool)
        for a_g, b_g in groups:
            lo, hi = max(0, r0 - b_g), r0 + 63 - a_g
            if hi >= 0:
                band[lo:hi + 1] = True
        vert = np.zeros(N, bool)
        vert[vidx[b, : vcnt[b]]] = True
        assert not (band & vert).any()            # de-duplicated
        got[i] = (band | vert) & (np.arange(N) <= i)
    assert np.array_equal(got, ref)


def test_vs_block_verticals_direct_intervals():
    rng = np.random.default_rng(21)
    N = 64 * 10
    S = np.unique(np.concatenate([[0], rng.choice(N, 30, replace=False)]))
    V = np.unique(rng.choice(N, 40, replace=False))
    groups = orc.vs_groups(S)
    vcnt, vidx = orc.vs_block_verticals(V, groups, N)
    for b in range(N // 64):
        r0 = 64 * b
        ref = [j for j in V if j <= r0 + 63 and
               not any(r0 - bg <= j <= r0 + 63 - ag for ag, bg in groups)]
        assert vidx[b, : vcnt[b]].tolist() == ref


# ------------------------------------------------ element-exact VS variant

def test_vs_exact_mask_bruteforce_loops():
    rng = np.random.default_rng(40)
    N = 48
    S = sorted(set([0] + rng.choice(N, 9, replace=False).tolist()))
    V = sorted(set(rng.choice(N, 6, replace=False).tolist()))
    got = orc.mask_vs_exact(np.arange(N), N, V, S)
    for i in range(N):
        for j in range(N):
            assert got[i, j] == (j <= i and (j in V or (i - j) in S)), (i, j)


def test_vs_exact_mask_closed_forms():
    N = 200
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    assert np.array_equal(orc.mask_vs_exact(np.arange(N), N, [], np.arange(N)), j <= i)
    assert np.array_equal(orc.mask_vs_exact(np.arange(N), N, [], [0]), i == j)
    assert np.array_equal(orc.mask_vs_exact(np.arange(N), N, [7], [0]), (i == j) | ((j == 7) & (i >= 7)))


@pytest.mark.parametrize("seed", range(3))
def test_vs_exact_mask_within_band_mask(seed):
    """The exact diagonals are a subset of the bands they sweep (the band
    reading is a superset)."""
    rng = np.random.default_rng(50 + seed)
    N = 64 * 9
    S = np.unique(np.concatenate([[0], rng.choice(N, 30, replace=False)]))
    V = np.unique(rng.choice(N, 20, replace=False))
    ex = orc.mask_vs_exact(np.arange(N), N, V, S)
    band = orc.mask_vs(np.arange(N), N, V, S)
    assert not (ex & ~band).any()
    assert ex.sum() < band.sum()


@pytest.mark.parametrize("seed", range(3))
def test_vs_exact_index_reproduces_mask(seed):
    """Per 128-row query tile: the key ranges of the offset groups (gap <= 128),
    masked element by element with (i - j in S or j in V), plus the tile's
    vertical list, give exactly the exact mask; the list never repeats a key
    of the ranges."""
    rng = np.random.default_rng(60 + seed)
    N = 128 * 6
    S = np.unique(np.concatenate([[0], rng.choice(N, 40 + 10 * seed, replace=False)]))
    V = np.unique(rng.choice(N, 50, replace=False))
    groups, vcnt, vidx = orc.vs_exact_index(V, S, N)
    sset, vset = set(S.tolist()), set(V.tolist())
    ref = orc.mask_vs_exact(np.arange(N), N, V, S)
    got = np.zeros((N, N), bool)
    for t in range(N // 128):
        R = 128 * t
        rng_keys = set()
        for a_g, b_g in groups:
            rng_keys.update(range(max(0, R - b_g), max(0, R + 128 - a_g)))
        lst = vidx[t, : vcnt[t]].tolist()
        assert not (set(lst) & rng_keys)
        assert lst == sorted(lst)
        for i in range(R, R + 128):
            for j in rng_keys:
                if j <= i and ((i - j) in sset or j in vset):
                    got[i, j] = True
            for j in lst:
                if j <= i:
                    got[i, j] = True
    assert np.array_equal(got, ref)


# ------------------------------------------------- head map and conversion

def test_kv_head_matches_repeat_interleave():
    """GQA reading: expanding the KV heads with repeat_interleave (each KV head
    serving g consecutive query heads, the LLaMA grouping) puts KV head
    kv_head(h) at query head h."""
    for Hq, Hkv in [(32, 8), (8, 2), (4, 4), (6, 1)]:
        expanded = torch.arange(Hkv).repeat_interleave(Hq // Hkv)
        assert [orc.kv_head(h, Hq, Hkv) for h in range(Hq)] == expanded.tolist()


def test_to_f64_is_exact_bf16_decoding():
    """bf16 -> float64 equals decoding the 16 stored bits by hand: sign,
    8-bit exponent, 7-bit fraction, normal and subnormal."""
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 1 << 16, 4096)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]                 # no inf / nan encodings
    x = torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)
    got = orc.to_f64(x)
    for b, g in zip(bits.tolist(), got.tolist()):
        sign = -1.0 if b >> 15 else 1.0
        e, f = (b >> 7) & 0xFF, b & 0x7F
        ref = sign * (f / 128.0 * 2.0 ** -126 if e == 0 else (1 + f / 128.0) * 2.0 ** (e - 127))
        assert g == ref, (b, g, ref)


# ---------------------------------------------------------- kept attention mass
def test_kept_mass_bruteforce_loops_and_closed_forms():
    """The kept share of a row's causal softmax, by plain loops; the full
    causal mask keeps 1, the empty mask 0, a single key its probability, and
    keys past the row do not count."""
    rng = np.random.default_rng(5)
    N, d = 24, 8
    q = rng.normal(size=(N, d))
    k = rng.normal(size=(N, d))
    sc = 0.4
    rows = np.array([0, 3, 11, 23])
    mask = rng.random((rows.size, N)) < 0.4
    got = orc.kept_mass(q[rows], k, rows, mask, sc)
    for a, i in enumerate(rows):
        w = [math.exp(sc * float(q[i] @ k[j])) for j in range(i + 1)]
        kept = sum(w[j] for j in range(i + 1) if mask[a, j])
        assert got[a] == pytest.approx(kept / sum(w), rel=1e-12, abs=1e-15)
    full = np.ones((rows.size, N), bool)
    np.testing.assert_allclose(orc.kept_mass(q[rows], k, rows, full, sc), 1.0, rtol=1e-12)
    assert (orc.kept_mass(q[rows], k, rows, ~full, sc) == 0).all()
    one = np.zeros((rows.size, N), bool)
    one[:, 0] = True
    p0 = [math.exp(sc * float(q[i] @ k[0])) / sum(math.exp(sc * float(q[i] @ k[j])) for j in range(i + 1))
          for i in rows]
    np.testing.assert_allclose(orc.kept_mass(q[rows], k, rows, one, sc), p0, rtol=1e-12)
    past = np.zeros((rows.size, N), bool)
    past[:, -1] = True  # key N-1 is past every row but the last
    np.testing.assert_allclose(orc.kept_mass(q[rows], k, rows, past, sc)[:-1], 0.0)


def test_kept_mass_equals_lse_ratio():
    """For a causal mask M, the kept mass of row i is exp(LSE over M minus the
    dense causal LSE): the identity the pattern search reads off the kernels'
    LSE outputs."""
    rng = np.random.default_rng(6)
    N, d = 40, 16
    q, k, v = rng.normal(size=(N, d)), rng.normal(size=(N, d)), rng.normal(size=(N, d))
    sc = 0.25
    rows = np.arange(N)
    causal = np.arange(N)[None, :] <= rows[:, None]
    mask = (rng.random((N, N)) < 0.5) & causal
    mask[rows, rows] = True  # every row keeps at least its diagonal
    _, lse_s = orc.attention_rows(q, k, v, mask, sc)
    _, lse_d = orc.attention_rows(q, k, v, causal, sc)
    np.testing.assert_allclose(orc.kept_mass(q, k, rows, mask, sc), np.exp(lse_s - lse_d), rtol=1e-12)


# ---------------------------------------------------------------- Grid pattern
def test_grid_with_one_position_is_block_sparse():
    """P = 1: every token is at the same in-frame position, and the Grid
    selection and mask are the Block-Sparse ones."""
    rng = np.random.default_rng(8)
    N, d = 512, 8
    q, k = rng.normal(size=(N, d)), rng.normal(size=(N, d))
    gi, gc = orc.grid_select(q, k, 1, 0.3, 3)
    bi, bc = orc.bs_select(q, k, 0.3, 3)
    assert np.array_equal(gi[0], bi) and np.array_equal(gc[0], bc)
    rows = np.array([0, 70, 200, 511])
    assert np.array_equal(orc.mask_grid(rows, N, 1, gi, gc), orc.mask_bs(rows, N, bi, bc))


def test_grid_mask_bruteforce_loops():
    """Plain loops over (i, j) with the position, causal and block rules."""
    rng = np.random.default_rng(9)
    P, F, d = 3, 256, 4
    N = P * F
    q, k = rng.normal(size=(N, d)), rng.normal(size=(N, d))
    gi, gc = orc.grid_select(q, k, P, 0.5, 2)
    rows = np.array([0, 2, 5, 190, 383, 600, N - 1])
    got = orc.mask_grid(rows, N, P, gi, gc)
    for r, i in enumerate(rows):
        for j in range(N):
            want = False
            if j <= i and j % P == i % P:
                sel = set(int(x) for x in gi[i % P][(i // P) // 64][: gc[i % P][(i // P) // 64]])
                want = ((j // P) // 64) in sel
            assert got[r, j] == want, (i, j)


def test_grid_selection_follows_each_position_sequence():
    """A block pair planted in one position's sequence is selected there and
    not at the other positions; with every block selected the mask is every
    earlier same-position key."""
    rng = np.random.default_rng(10)
    P, F, d = 2, 512, 8
    N = P * F
    q = rng.normal(size=(N, d)) * 0.1
    k = rng.normal(size=(N, d)) * 0.1
    u = np.zeros(d)
    u[0] = 5.0
    # position 1: query block 7 and key block 2 of its frame sequence share a direction
    q[[f * P + 1 for f in range(7 * 64, 8 * 64)]] += u
    k[[f * P + 1 for f in range(2 * 64, 3 * 64)]] += u
    gi, gc = orc.grid_select(q, k, P, 1.0, 2)
    assert 2 in gi[1][7][: gc[1][7]]
    assert 2 not in gi[0][7][: gc[0][7]]
    ai, ac = orc.grid_select(q, k, P, 1.0, F // 64)
    rows = np.array([5, 700, N - 1])
    m = orc.mask_grid(rows, N, P, ai, ac)
    j = np.arange(N)
    for r, i in enumerate(rows):
        assert np.array_equal(m[r], (j <= i) & (j % P == i % P))
