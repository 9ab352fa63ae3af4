"""Planted mistakes in the oracle.

Each mutant below is a plausible slip in one oracle function: a dropped term,
an off-by-one, a wrong sign or index, a transposed operand, a missed forced
index.  With the mutant patched into the oracle module (on the CPU, for the
duration of one test), at least one pin of ``test_oracle_pins.py`` must fail.
A mutant that survives every pin would mean that part of the oracle is not
pinned.
"""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import minf_oracle as orc

_ORIG = {name: getattr(orc, name) for name in dir(orc) if not name.startswith("_")}


def _pin_calls():
    """Every pin of test_oracle_pins with each of its parameter sets."""
    calls = []
    for name in sorted(vars(pins)):
        fn = getattr(pins, name)
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, ()))
            continue
        argnames, argvalues = marks[0].args[0], marks[0].args[1]
        multi = "," in argnames
        for v in argvalues:
            calls.append((name, fn, tuple(v) if multi else (v,)))
    return calls


PIN_CALLS = _pin_calls()


def _some_pin_fails():
    for name, fn, args in PIN_CALLS:
        try:
            fn(*args)
        except AssertionError:
            return name
    return None


# ------------------------------------------------------------------ mutants

def _vs_estimate_variant(q_last, k, scale, row_chunk=16, *, normalise=True, strict=False, slash_row_free=False):
    q_last = np.asarray(q_last, np.float64)
    k = np.asarray(k, np.float64)
    N, L = k.shape[0], q_last.shape[0]
    v = np.zeros(N)
    sigma = np.zeros(N)
    cols = np.arange(N)
    for r0 in range(0, L, row_chunk):
        qs = q_last[r0:r0 + row_chunk]
        rows = np.arange(N - L + r0, N - L + r0 + qs.shape[0])
        s = scale * (qs @ k.T)
        causal = (cols[None, :] < rows[:, None]) if strict else (cols[None, :] <= rows[:, None])
        causal = causal | (cols[None, :] == 0)          # keep every row non-empty
        s = np.where(causal, s, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True) if normalise else e
        v += p.sum(axis=0)
        offs = (N - 1 - cols[None, :] + 0 * rows[:, None]) if slash_row_free else rows[:, None] - cols[None, :]
        sigma += np.bincount(offs[causal], weights=p[causal], minlength=N)
    return v, sigma


def _select_topk_ties_high(scores, k, forced=None):
    key = np.array(scores, dtype=np.float64, copy=True)
    n = key.shape[0]
    if forced is not None:
        key[forced] = np.inf
    k = min(int(k), n)
    order = sorted(range(n), key=lambda j: (-key[j], -j))
    return np.array(sorted(order[:k]), dtype=np.int64)


def _select_topk_rows_score_order(scores, valid, k, forced_col=None):
    idx, cnt = _ORIG["select_topk_rows"](scores, valid, k, forced_col)
    key = np.where(valid, scores, -np.inf)
    if forced_col is not None:
        key[np.arange(scores.shape[0]), forced_col] = np.inf
    for r in range(idx.shape[0]):
        sel = idx[r, : cnt[r]]
        idx[r, : cnt[r]] = sel[np.argsort(-key[r, sel], kind="stable")]
    return idx, cnt


def _bs_select_no_forced(q, k, scale, k_b, block=64, blocks=None):
    qbar, kbar = orc.bs_pool(q, block), orc.bs_pool(k, block)
    nb = qbar.shape[0]
    b = np.arange(nb) if blocks is None else np.asarray(blocks, np.int64)
    t = orc.bs_scores(qbar[b], kbar, scale)
    valid = np.arange(nb)[None, :] <= b[:, None]
    return orc.select_topk_rows(t, valid, k_b, forced_col=None)


def _bs_select_pooled_rows_by_position(qbar, kbar, scale, k_b, blocks=None):
    nb = qbar.shape[0]
    b = np.arange(nb) if blocks is None else np.asarray(blocks, np.int64)
    t = orc.bs_scores(qbar[b], kbar, scale)
    valid = np.arange(nb)[None, :] <= np.arange(len(b))[:, None]      # row position, not block id
    return orc.select_topk_rows(t, valid, k_b, forced_col=b)


def _bs_select_pooled_forced_by_position(qbar, kbar, scale, k_b, blocks=None):
    nb = qbar.shape[0]
    b = np.arange(nb) if blocks is None else np.asarray(blocks, np.int64)
    t = orc.bs_scores(qbar[b], kbar, scale)
    valid = np.arange(nb)[None, :] <= b[:, None]
    return orc.select_topk_rows(t, valid, k_b, forced_col=np.arange(len(b)))   # not following blocks


def _vs_groups_strict(s_idx, block=64):
    s = np.asarray(s_idx, np.int64)
    if s.size == 0:
        return np.zeros((0, 2), np.int64)
    starts = np.concatenate([[True], np.diff(s) >= block])
    first = np.nonzero(starts)[0]
    last = np.concatenate([first[1:] - 1, [s.size - 1]])
    return np.stack([s[first], s[last]], axis=1)


def _vs_block_verticals_no_dedup(v_idx, groups, N, block=64):
    v = np.asarray(v_idx, np.int64)
    nb = N // block
    vcnt = np.zeros(nb, np.int64)
    vidx = np.full((nb, v.size), -1, np.int64)
    for b in range(nb):
        keep = v[v <= b * block + block - 1]
        vcnt[b] = keep.size
        vidx[b, : keep.size] = keep
    return vcnt, vidx


def _mask_vs_variant(rows, N, v_idx, s_idx, block=64, *, widen=0, per_row=False):
    rows = np.asarray(rows)
    s = np.sort(np.asarray(s_idx, np.int64))
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    vert = np.zeros(N, bool)
    vert[np.asarray(v_idx, np.int64)] = True
    for r, i in enumerate(rows):
        r0 = i if per_row else (i // block) * block
        u = r0 - j
        n_in = np.searchsorted(s, u + block - 1 + widen, side="right") - np.searchsorted(s, u, side="left")
        out[r] = (j <= i) & (vert | (n_in > 0))
    return out


def _mask_ashape_inclusive(rows, N, n_sink, n_local):
    rows = np.asarray(rows)
    j = np.arange(N)[None, :]
    i = rows[:, None]
    return (j <= i) & ((j < n_sink) | (i - j <= n_local))


def _mask_bs_no_causal(rows, N, blk_idx, blk_cnt, block=64):
    rows = np.asarray(rows)
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        sel = np.zeros(N // block, bool)
        sel[np.asarray(blk_idx[i // block][: int(blk_cnt[i // block])], np.int64)] = True
        out[r] = sel[j // block]
    return out


def _mask_vs_exact_offsets_as_keys(rows, N, v_idx, s_idx):
    rows = np.asarray(rows)
    vert = np.zeros(N, bool)
    vert[np.asarray(v_idx, np.int64)] = True
    diag = np.zeros(N, bool)
    diag[np.asarray(s_idx, np.int64)] = True
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        out[r] = (j <= i) & (vert | diag[j])           # S read as key columns
    return out


def _attention_rows_variant(q_rows, k, v, mask, scale, *, lse_without_max=False, sum_unmasked=False):
    s_all = scale * (np.asarray(q_rows, np.float64) @ np.asarray(k, np.float64).T)
    s = np.where(mask, s_all, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(s - m), 0.0)
    l = (np.exp(s_all - m).sum(axis=1, keepdims=True) if sum_unmasked else e.sum(axis=1, keepdims=True))
    o = (e @ np.asarray(v, np.float64)) / np.where(l > 0, l, 1.0)
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.log(l[:, 0]) + (0.0 if lse_without_max else m[:, 0])
    lse[empty] = -np.inf
    return o, lse


def _kept_mass_variant(q_rows, k, rows, mask, scale, *, over_mask=False, noncausal=False):
    q_rows = np.asarray(q_rows, np.float64)
    rows = np.asarray(rows)
    s = scale * (q_rows @ np.asarray(k, np.float64).T)
    causal = np.arange(k.shape[0])[None, :] <= rows[:, None]
    sc = np.where(causal, s, -np.inf)
    e = np.exp(sc - sc.max(axis=1, keepdims=True))
    keep = mask if noncausal else (mask & causal)
    if noncausal:
        e = np.exp(s - sc.max(axis=1, keepdims=True))
    den = np.where(mask & causal, e, 0.0).sum(axis=1) if over_mask else np.where(causal, e, 0.0).sum(axis=1)
    return np.where(keep, e, 0.0).sum(axis=1) / den


def _grid_select_contiguous(q, k, P, scale, k_b, block=64):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    F = q.shape[0] // P
    idx, cnt = [], []
    for p in range(P):
        i_, c_ = _ORIG["bs_select"](q[p * F:(p + 1) * F], k[p * F:(p + 1) * F], scale, k_b, block)
        idx.append(i_)
        cnt.append(c_)
    return np.stack(idx), np.stack(cnt)


def _mask_grid_any_position(rows, N, P, blk_idx, blk_cnt, block=64):
    rows = np.asarray(rows)
    j = np.arange(N)
    out = np.zeros((rows.size, N), bool)
    for r, i in enumerate(rows):
        p, f = i % P, i // P
        sel = np.zeros(N // P // block, bool)
        b = f // block
        sel[np.asarray(blk_idx[p][b][: int(blk_cnt[p][b])], np.int64)] = True
        out[r] = (j <= i) & sel[(j // P) // block]
    return out


def _to_f64_via_half(x):
    import torch
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float16).to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


MUTANTS = {
    "vs_estimate: probabilities not normalised": {
        "vs_estimate": lambda q, k, sc, row_chunk=16: _vs_estimate_variant(q, k, sc, row_chunk, normalise=False)},
    "vs_estimate: diagonal key excluded (j < i)": {
        "vs_estimate": lambda q, k, sc, row_chunk=16: _vs_estimate_variant(q, k, sc, row_chunk, strict=True)},
    "vs_estimate: slash offset taken from the key alone": {
        "vs_estimate": lambda q, k, sc, row_chunk=16: _vs_estimate_variant(q, k, sc, row_chunk, slash_row_free=True)},
    "vs_estimate: scale dropped": {
        "vs_estimate": lambda q, k, sc, row_chunk=16: _ORIG["vs_estimate"](q, k, 1.0, row_chunk)},
    "select_topk: ties to the higher index": {"select_topk": _select_topk_ties_high},
    "select_topk: forced index ignored": {
        "select_topk": lambda scores, k, forced=None: _ORIG["select_topk"](scores, k, None)},
    "select_topk_rows: selection left in score order": {"select_topk_rows": _select_topk_rows_score_order},
    "vs_select: slash offset 0 not forced": {
        "vs_select": lambda v, s, kv, ks: (_ORIG["select_topk"](v, kv), _ORIG["select_topk"](s, ks))},
    "bs_pool: block sum instead of mean": {
        "bs_pool": lambda x, block=64: _ORIG["bs_pool"](x, block) * block},
    "bs_scores: operands transposed": {"bs_scores": lambda qb, kb, sc: sc * (kb @ qb.T)},
    "bs_select: diagonal block not forced": {"bs_select": _bs_select_no_forced},
    "bs_select_pooled: causal limit from the row position": {"bs_select_pooled": _bs_select_pooled_rows_by_position},
    "bs_select_pooled: forced block from the row position": {
        "bs_select_pooled": _bs_select_pooled_forced_by_position},
    "vs_groups: offsets exactly 64 apart not merged": {"vs_groups": _vs_groups_strict},
    "vs_block_verticals: verticals inside bands kept": {"vs_block_verticals": _vs_block_verticals_no_dedup},
    "mask_vs: band one key too wide": {
        "mask_vs": lambda rows, N, V, S, block=64: _mask_vs_variant(rows, N, V, S, block, widen=1)},
    "mask_vs: band anchored at the row, not the block": {
        "mask_vs": lambda rows, N, V, S, block=64: _mask_vs_variant(rows, N, V, S, block, per_row=True)},
    "mask_ashape: local window one key too long": {"mask_ashape": _mask_ashape_inclusive},
    "mask_bs: causal limit missing": {"mask_bs": _mask_bs_no_causal},
    "mask_vs_exact: slash offsets read as key columns": {"mask_vs_exact": _mask_vs_exact_offsets_as_keys},
    "attention_rows: LSE without the row max": {
        "attention_rows": lambda q, k, v, m, sc: _attention_rows_variant(q, k, v, m, sc, lse_without_max=True)},
    "attention_rows: softmax sum over unmasked keys": {
        "attention_rows": lambda q, k, v, m, sc: _attention_rows_variant(q, k, v, m, sc, sum_unmasked=True)},
    "default_scale: 1/d instead of 1/sqrt(d)": {"default_scale": lambda d: 1.0 / d},
    "kv_head: interleaved instead of contiguous groups": {"kv_head": lambda h, Hq, Hkv: h % Hkv},
    "to_f64: converted through float16": {"to_f64": _to_f64_via_half},
    "kept_mass: normalised over the mask": {
        "kept_mass": lambda q, k, r, m, sc: _kept_mass_variant(q, k, r, m, sc, over_mask=True)},
    "grid_select: positions taken as contiguous runs": {"grid_select": _grid_select_contiguous},
    "mask_grid: other in-frame positions kept": {"mask_grid": _mask_grid_any_position},
    "kept_mass: keys past the row counted": {
        "kept_mass": lambda q, k, r, m, sc: _kept_mass_variant(q, k, r, m, sc, noncausal=True)},
}


@pytest.mark.parametrize("label", sorted(MUTANTS))
def test_pins_catch_mutant(label, monkeypatch):
    for name, fn in MUTANTS[label].items():
        assert name in _ORIG, name
        monkeypatch.setattr(orc, name, fn)
    caught = _some_pin_fails()
    assert caught is not None, f"no pin fails with the mutant '{label}'"


def test_pins_pass_unmutated():
    assert _some_pin_fails() is None
