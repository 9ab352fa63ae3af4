"""CPU oracle for pre-fill dynamic sparse attention (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, tables or helpers); it receives the same
seeded bf16 inputs as plain arrays and converts them exactly to float64.

What it computes, and where that comes from ("MInference 1.0: Accelerating
Pre-filling for Long-Context LLMs via Dynamic Sparse Attention", the summary
page and the abstract):

* three per-head patterns, A-shape, Vertical-Slash and Block-Sparse
  (abstract; summary, "Summary");
* Vertical-Slash indices estimated online by scoring the last query vectors
  against all keys (summary, "Key points", second item);
* Block-Sparse indices estimated online from queries and keys mean-pooled in
  64-token blocks (summary, "Key points", second item);
* attention computed only over the estimated indices (summary, "Summary",
  stage 3).

Besides the band reading of a slash (``mask_vs``), ``mask_vs_exact`` and
``vs_exact_index`` give the element-exact variant, where a slash is its
diagonal only.

The pages fix nothing finer.  The readings taken where they are silent
(last 64 queries; natural-exp softmax with scale 1/sqrt(d) before the column
and diagonal sums; forced slash offset 0 and forced diagonal block; ties to
the lowest index; a slash covering the 64-key band it sweeps through a
64-row query block; de-duplicated key sets; GQA head h -> KV head h // g;
no softmax before the Block-Sparse top-k because it is monotone) are listed
with the reasons in the design notes.  Every function below states the
reading it follows.

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_*.py`` (brute force on tiny inputs, a library attention
routine, closed forms, invariants, planted structure, and a full sort).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def to_f64(x) -> np.ndarray:
    """bf16 torch tensor (or any array) -> float64 numpy, exactly."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int) -> float:
    """Softmax temperature 1/sqrt(d) (standard attention; the pages state none)."""
    return 1.0 / np.sqrt(d)


def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """GQA reading: contiguous groups, query head h uses KV head h // (Hq/Hkv)."""
    return h // (Hq // Hkv)


# --------------------------------------------------------------------------
# Vertical-Slash estimation ("Key points": last query vectors vs all keys)
# --------------------------------------------------------------------------

def vs_estimate(q_last: np.ndarray, k: np.ndarray, scale: float, row_chunk: int = 16):
    """Vertical and slash scores of one head.

    ``q_last`` holds the last L query rows (rows N-L .. N-1), ``k`` all N keys.
    For each of those rows i, the causal scores s_ij = scale * q_i . k_j
    (j <= i) are turned into probabilities p_ij by a softmax over j.  Then

        v_j     = sum_i p_ij                  (vertical score of key column j)
        sigma_o = sum_i p_{i, i-o}, i-o >= 0  (slash score of diagonal offset o)

    Both are returned as float64 arrays of length N.
    """
    q_last = np.asarray(q_last, np.float64)
    k = np.asarray(k, np.float64)
    N = k.shape[0]
    L = q_last.shape[0]
    v = np.zeros(N)
    sigma = np.zeros(N)
    cols = np.arange(N)
    for r0 in range(0, L, row_chunk):
        qs = q_last[r0:r0 + row_chunk]
        rows = np.arange(N - L + r0, N - L + r0 + qs.shape[0])
        s = scale * (qs @ k.T)
        causal = cols[None, :] <= rows[:, None]
        s = np.where(causal, s, NEG_INF)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)
        v += p.sum(axis=0)
        offs = rows[:, None] - cols[None, :]
        sigma += np.bincount(offs[causal], weights=p[causal], minlength=N)
    return v, sigma


# --------------------------------------------------------------------------
# Top-k selection (one rule for every pattern)
# --------------------------------------------------------------------------

def select_topk(scores: np.ndarray, k: int, forced=None) -> np.ndarray:
    """Indices of the k best candidates, returned in ascending index order.

    Candidates are ranked by score, higher first, ties going to the lower
    index; a ``forced`` index ranks above every score.  With tau the k-th key
    in that order, the result is every index whose score beats tau plus the
    lowest-index candidates that equal it, which is the first k of a full
    sort by (score desc, index asc).  ``k`` is clamped to the number of
    candidates.
    """
    key = np.array(scores, dtype=np.float64, copy=True)
    n = key.shape[0]
    if forced is not None:
        key[forced] = np.inf
    k = min(int(k), n)
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    tau = np.partition(key, n - k)[n - k]
    gt = key > tau
    eq = key == tau
    need = k - int(gt.sum())
    take_eq = eq & (np.cumsum(eq) <= need)
    return np.nonzero(gt | take_eq)[0].astype(np.int64)


def select_topk_rows(scores: np.ndarray, valid: np.ndarray, k: int, forced_col=None):
    """Row-wise :func:`select_topk` over a 2-D score matrix.

    ``valid[r, c]`` marks candidates; ``forced_col[r]`` (optional) is forced in
    row r.  Returns ``idx`` [R, k] (ascending, padded with -1) and
    ``cnt`` [R] = min(k, number of candidates).
    """
    R, C = scores.shape
    key = np.where(valid, scores, NEG_INF).astype(np.float64)
    if forced_col is not None:
        key[np.arange(R), forced_col] = np.inf
    ncand = valid.sum(axis=1)
    cnt = np.minimum(ncand, k)
    idx = np.full((R, k), -1, dtype=np.int64)
    # rows whose candidates all fit are taken whole
    kk = min(k, C)
    tau = -np.partition(-key, kk - 1, axis=1)[:, kk - 1]
    gt = (key > tau[:, None]) & valid
    eq = (key == tau[:, None]) & valid
    need = cnt - gt.sum(axis=1)
    take = gt | (eq & (np.cumsum(eq, axis=1) <= need[:, None]))
    for r in range(R):
        sel = np.nonzero(take[r])[0]
        idx[r, :sel.shape[0]] = sel
    return idx, cnt.astype(np.int64)


def vs_select(v: np.ndarray, sigma: np.ndarray, k_v: int, k_s: int):
    """Vertical set V = top-k_v of v; slash set S = top-k_s of sigma with
    offset 0 forced (every causal diagonal's main line is always kept)."""
    return select_topk(v, k_v), select_topk(sigma, k_s, forced=0)


# --------------------------------------------------------------------------
# Block-Sparse estimation ("Key points": 64-token mean-pooled Q and K)
# --------------------------------------------------------------------------

def bs_pool(x: np.ndarray, block: int = 64) -> np.ndarray:
    """Mean of each run of ``block`` consecutive rows: [N, d] -> [N/block, d]."""
    x = np.asarray(x, np.float64)
    N, d = x.shape
    return x.reshape(N // block, block, d).mean(axis=1)


def bs_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """t[b, c] = scale * qbar_b . kbar_c (all pairs; causality applied by the caller)."""
    return scale * (qbar @ kbar.T)


def bs_select(q: np.ndarray, k: np.ndarray, scale: float, k_b: int, block: int = 64, blocks=None):
    """Per query block b, the k_b best key blocks c <= b by pooled score,
    with c = b forced.  No softmax: it is monotone within a row, so it cannot
    change the selection.  Returns idx [nb, k_b] (ascending, -1 padded) and
    cnt [nb] = min(b + 1, k_b).  With ``blocks`` given, only those query
    blocks are selected (rows of the result follow ``blocks``)."""
    return bs_select_pooled(bs_pool(q, block), bs_pool(k, block), scale, k_b, blocks)


def bs_select_pooled(qbar: np.ndarray, kbar: np.ndarray, scale: float, k_b: int, blocks=None):
    """The selection of :func:`bs_select` from already pooled queries and
    keys (``qbar``, ``kbar``: [nb, d]).  Row r of the result is query block
    ``blocks[r]`` (every block when ``blocks`` is None): its candidates are
    the key blocks c <= blocks[r], and c = blocks[r] is forced."""
    nb = qbar.shape[0]
    b = np.arange(nb) if blocks is None else np.asarray(blocks, np.int64)
    t = bs_scores(qbar[b], kbar, scale)
    valid = np.arange(nb)[None, :] <= b[:, None]
    return select_topk_rows(t, valid, k_b, forced_col=b)


# --------------------------------------------------------------------------
# Vertical-Slash index: offset groups and per-block vertical lists
# --------------------------------------------------------------------------

def vs_groups(s_idx: np.ndarray, block: int = 64) -> np.ndarray:
    """Merge ascending slash offsets into groups [a_g, b_g].

    In a query block with first row r0, offset o sweeps the key band
    [r0 - o, r0 + block - 1 - o].  Bands of offsets o < o' touch or overlap
    exactly when o' - o <= block, so consecutive offsets closer than that
    belong to one group, whose union band is [r0 - b_g, r0 + block - 1 - a_g].
    """
    s = np.asarray(s_idx, np.int64)
    if s.size == 0:
        return np.zeros((0, 2), np.int64)
    starts = np.concatenate([[True], np.diff(s) > block])
    first = np.nonzero(starts)[0]
    last = np.concatenate([first[1:] - 1, [s.size - 1]])
    return np.stack([s[first], s[last]], axis=1)


def vs_block_verticals(v_idx: np.ndarray, groups: np.ndarray, N: int, block: int = 64):
    """Per query block b (rows r0 .. r0+block-1): the vertical columns that no
    slash group already covers, V_b = {j in V : j <= r0+block-1, j outside
    every band [r0 - b_g, r0 + block - 1 - a_g]}.

    Band membership is tested in the block-offset form: j lies in group g's
    band exactly when u = r0 - j satisfies a_g - (block-1) <= u <= b_g.
    Returns (vcnt [nb], vidx [nb, len(V)] padded with -1), lists ascending.
    """
    v = np.asarray(v_idx, np.int64)
    nb = N // block
    lo = groups[:, 0] - (block - 1) if groups.size else np.zeros(0, np.int64)
    hi = groups[:, 1] if groups.size else np.zeros(0, np.int64)
    vcnt = np.zeros(nb, np.int64)
    vidx = np.full((nb, v.size), -1, np.int64)
    for b in range(nb):
        r0 = b * block
        cand = v[v <= r0 + block - 1]
        u = r0 - cand
        g = np.searchsorted(hi, u, side="left")       # first group with b_g >= u
        inside = np.zeros(cand.shape, bool)
        ok = g < hi.size
        inside[ok] = lo[g[ok]] <= u[ok]
        keep = cand[~inside]
        vcnt[b] = keep.size
        vidx[b, :keep.size] = keep
    return vcnt, vidx


def vs_build_index(v_idx, s_idx, N: int, block: int = 64):
    """The compact Vertical-Slash index of one head: groups and per-block
    vertical lists (see :func:`vs_groups` and :func:`vs_block_verticals`)."""
    groups = vs_groups(s_idx, block)
    vcnt, vidx = vs_block_verticals(v_idx, groups, N, block)
    return groups, vcnt, vidx


# --------------------------------------------------------------------------
# Masks, straight from the set definitions (no groups, no lists)
# --------------------------------------------------------------------------

def mask_dense(rows: np.ndarray, N: int) -> np.ndarray:
    """Causal mask M(i, j) = [j <= i] for the given query rows."""
    return np.arange(N)[None, :] <= np.asarray(rows)[:, None]


def mask_ashape(rows, N: int, n_sink: int, n_local: int) -> np.ndarray:
    """A-shape: causal and (j < n_sink or i - j < n_local); the local window
    holds the diagonal and n_local keys in all."""
    rows = np.asarray(rows)
    j = np.arange(N)[None, :]
    i = rows[:, None]
    return (j <= i) & ((j < n_sink) | (i - j < n_local))


def mask_vs(rows, N: int, v_idx, s_idx, block: int = 64) -> np.ndarray:
    """Vertical-Slash: causal and (j in V or some o in S has
    r0 - o <= j <= r0 + block - 1 - o, r0 the first row of i's block).

    The slash test is evaluated directly on S: with u = r0 - j it asks for
    an offset in [u, u + block - 1].
    """
    rows = np.asarray(rows)
    s = np.sort(np.asarray(s_idx, np.int64))
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    vert = np.zeros(N, bool)
    vert[np.asarray(v_idx, np.int64)] = True
    for r, i in enumerate(rows):
        r0 = (i // block) * block
        u = r0 - j
        n_in = np.searchsorted(s, u + block - 1, side="right") - np.searchsorted(s, u, side="left")
        out[r] = (j <= i) & (vert | (n_in > 0))
    return out


def mask_vs_exact(rows, N: int, v_idx, s_idx) -> np.ndarray:
    """Element-exact Vertical-Slash: causal and (j in V or i - j in S).

    The slashes are the selected diagonals themselves, element by element,
    instead of the 64-key bands they sweep through a 64-row query block
    (:func:`mask_vs`); the exact set is contained in the band set.
    """
    rows = np.asarray(rows)
    vert = np.zeros(N, bool)
    vert[np.asarray(v_idx, np.int64)] = True
    diag = np.zeros(N, bool)
    diag[np.asarray(s_idx, np.int64)] = True
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        o = i - j
        causal = o >= 0
        out[r] = causal & (vert | np.where(causal, diag[np.clip(o, 0, N - 1)], False))
    return out


def vs_exact_index(v_idx, s_idx, N: int, tile: int = 128):
    """Index of the element-exact variant for query tiles of ``tile`` rows:
    the offsets merged at gap <= tile (each group's diagonals sweep the key
    range [R - b_g, R + tile - 1 - a_g] of the tile starting at row R), and
    per tile the verticals outside every such range (they are the only keys
    of V that the ranges do not already hold).  Returns (groups, vcnt, vidx)
    as :func:`vs_build_index` with blocks of ``tile`` rows."""
    groups = vs_groups(s_idx, tile)
    vcnt, vidx = vs_block_verticals(v_idx, groups, N, tile)
    return groups, vcnt, vidx


def mask_bs(rows, N: int, blk_idx, blk_cnt, block: int = 64) -> np.ndarray:
    """Block-Sparse: causal and key block floor(j/64) selected for i's block."""
    rows = np.asarray(rows)
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        b = i // block
        sel = np.zeros(N // block, bool)
        sel[np.asarray(blk_idx[b][: int(blk_cnt[b])], np.int64)] = True
        out[r] = (j <= i) & sel[j // block]
    return out


# --------------------------------------------------------------------------
# Grid pattern (MMInference abstract: video locality gives a Grid pattern,
# handled through a permutation; the pages define no more, the reading is
# stated in the design notes)
# --------------------------------------------------------------------------

def grid_select(q: np.ndarray, k: np.ndarray, P: int, scale: float, k_b: int, block: int = 64):
    """Selection of a Grid head over a video segment of F frames x P tokens
    per frame, tokens frame-major (i = f * P + p).  Reading: the tokens of one
    in-frame position p, taken in frame order (rows p, p + P, p + 2P, ...),
    form a sequence of their own, and each such sequence gets the
    Block-Sparse selection (64-frame mean-pooled blocks, top-k_b per query
    block, diagonal forced).  Returns idx [P, F/64, k_b] and cnt [P, F/64]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    idx, cnt = [], []
    for p in range(P):
        i_, c_ = bs_select(q[p::P], k[p::P], scale, k_b, block)
        idx.append(i_)
        cnt.append(c_)
    return np.stack(idx), np.stack(cnt)


def mask_grid(rows, N: int, P: int, blk_idx, blk_cnt, block: int = 64) -> np.ndarray:
    """Grid: key j is kept for query i when both sit at the same in-frame
    position (j = i mod P), j <= i, and the 64-frame block of j's frame is
    selected for the block of i's frame in that position's sequence."""
    rows = np.asarray(rows)
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        p, f = i % P, i // P
        sel = np.zeros(N // P // block, bool)
        b = f // block
        sel[np.asarray(blk_idx[p][b][: int(blk_cnt[p][b])], np.int64)] = True
        out[r] = (j <= i) & (j % P == p) & sel[(j // P) // block]
    return out


# --------------------------------------------------------------------------
# Masked softmax attention
# --------------------------------------------------------------------------

def attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray,
                   mask: np.ndarray, scale: float):
    """O_i = sum_{j in M(i)} softmax_j(s_ij) v_j with s_ij = scale q_i . k_j, and
    LSE_i = log sum_{j in M(i)} exp(s_ij), in float64.  An empty row gives
    O = 0 and LSE = -inf."""
    q_rows = np.asarray(q_rows, np.float64)
    s = scale * (q_rows @ np.asarray(k, np.float64).T)
    s = np.where(mask, s, NEG_INF)
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(s - m), 0.0)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ np.asarray(v, np.float64)) / np.where(l > 0, l, 1.0)
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = m[:, 0] + np.log(l[:, 0])
    lse[empty] = NEG_INF
    return o, lse


def kept_mass(q_rows: np.ndarray, k: np.ndarray, rows: np.ndarray, mask: np.ndarray, scale: float):
    """The share of each row's dense causal attention that a sparse mask keeps
    (the quality measure of the offline pattern search, "MInference 1.0"
    summary, "Summary", stage 1: a pattern per head chosen offline; the page
    names no measure, and the kept probability mass is the plain reading):
    for row i, the sum over j in M(i) of p_ij, p_ij = exp(s_ij) / sum_{j' <= i}
    exp(s_ij'), s_ij = scale q_i . k_j.  Only the causal part of the mask
    counts."""
    q_rows = np.asarray(q_rows, np.float64)
    rows = np.asarray(rows)
    s = scale * (q_rows @ np.asarray(k, np.float64).T)
    causal = np.arange(k.shape[0])[None, :] <= rows[:, None]
    s = np.where(causal, s, NEG_INF)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return np.where(mask & causal, e, 0.0).sum(axis=1) / e.sum(axis=1)


def attention_head(q, k, v, rows, mask_fn, scale, row_chunk: int = 0):
    """Attention of one head for the given query rows, in row chunks;
    ``mask_fn(rows)`` returns the boolean mask of those rows."""
    rows = np.asarray(rows)
    d = v.shape[1]
    if row_chunk <= 0:
        row_chunk = max(1, min(256, (1 << 23) // k.shape[0]))
    O = np.zeros((rows.size, d))
    L = np.zeros(rows.size)
    for a in range(0, rows.size, row_chunk):
        rr = rows[a:a + row_chunk]
        o, lse = attention_rows(q[rr], k, v, mask_fn(rr), scale)
        O[a:a + rr.size] = o
        L[a:a + rr.size] = lse
    return O, L
