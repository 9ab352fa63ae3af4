"""Offline, kernel-aware pattern search: one pattern and setting per head
("MInference 1.0" summary, "Summary", stage 1: an offline search assigns
A-shape, Vertical-Slash or Block-Sparse to every head).

The page gives the step in one sentence; this module takes its plainest
reading:

* cost is kernel-aware: the 128 x 128 key tiles that this library's attention
  kernel executes for the head under a candidate setting, counted on the
  device during the run (4 * 128 * 128 * d FLOP each), not the mask's size;
* quality is the share of the head's dense causal attention that the
  candidate keeps, averaged over query rows: for row i,
  sum over the kept keys j of softmax_j(s_ij) = exp(LSE_sparse(i) - LSE_dense(i)),
  both LSEs from this library's kernels (the sparse kernels' LSE runs over the
  kept keys only);
* the budget of a head is the cost of a reference setting on the same head
  (Vertical-Slash with 1000 verticals and 6096 slashes by default); per
  pattern the largest candidate setting that fits the budget competes, and
  the head takes the pattern whose candidate keeps the most mass, ties going
  to the cheaper.

Every estimation and attention step runs in the library's kernels; this
module sequences the calls and averages the per-row shares.
"""
from __future__ import annotations

import argparse
import json
from dataclasses import dataclass, field

import torch

from . import minf

PATTERNS = ("a_shape", "vertical_slash", "block_sparse")

# candidate settings per pattern, cheapest first
DEFAULT_CANDIDATES = {
    "a_shape": [(128, 1024), (128, 2048), (128, 4096), (128, 8192), (128, 16384), (128, 32768)],
    "vertical_slash": [(250, 1524), (500, 3048), (1000, 6096), (2000, 12192)],
    "block_sparse": [25, 50, 100, 200, 400],
}
DEFAULT_REFERENCE = ("vertical_slash", (1000, 6096))


@dataclass
class Trial:
    """One candidate setting evaluated on one head."""
    pattern: str
    setting: object
    tiles: int          # executed 128 x 128 key tiles (device counter)
    kept: float         # mean kept share of the dense attention


@dataclass
class HeadChoice:
    head: int
    budget_tiles: int
    choice: Trial | None
    trials: list = field(default_factory=list)


def _clamp(pattern, setting, N):
    """A candidate setting limited to what a prompt of N tokens holds."""
    if pattern == "a_shape":
        n_sink, n_local = setting
        return (min(n_sink, N), min(n_local, N))
    if pattern == "vertical_slash":
        k_v, k_s = setting
        return (min(k_v, N), min(k_s, N))
    return min(int(setting), N // 64)


def choose(trials, budget_tiles):
    """Per pattern the largest fitting candidate (trials of a pattern are
    cheapest first), then the one keeping the most mass, ties to the cheaper.
    None when no candidate fits."""
    best = []
    for pat in PATTERNS:
        fit = [t for t in trials if t.pattern == pat and t.tiles <= budget_tiles]
        if fit:
            best.append(max(reversed(fit), key=lambda t: t.tiles))  # the later of equal costs
    if not best:
        return None
    return max(best, key=lambda t: (t.kept, -t.tiles))


class Evaluator:
    """Runs one head under candidate settings through the library's kernels
    and reports (executed tiles, mean kept share)."""

    def __init__(self, q, k, v, rows=None):
        self.q, self.k, self.v = q, k, v
        self.shape = minf.shape_of(q, k)
        self.N = self.shape.N
        _, self.lse_dense = minf.minf_dense_attn(q, k, v)
        self.rows = None if rows is None else torch.as_tensor(rows, device=q.device, dtype=torch.long)
        self.o = torch.empty_like(q)
        self.lse = torch.empty_like(self.lse_dense)

    def _kept(self, head):
        ls, ld = self.lse[:, head], self.lse_dense[:, head]
        if self.rows is not None:
            ls, ld = ls[:, self.rows], ld[:, self.rows]
        return float(torch.exp((ls - ld).double()).mean().item())

    def run(self, head, pattern, setting):
        q, k, v, shp = self.q, self.k, self.v, self.shape
        hd = [head]
        if pattern == "a_shape":
            n_sink, n_local = setting
            ws = minf.workspace(minf.OP_ATTN_ASHAPE, shp, 1, device=q.device)
            minf.minf_attn_ashape(q, k, v, hd, n_sink, n_local, o=self.o, lse=self.lse, ws=ws)
        elif pattern == "vertical_slash":
            k_v, k_s = setting
            v_idx, s_idx = minf.minf_estimate_vs(q, k, hd, k_v, k_s)
            index = minf.minf_build_index(shp, v_idx, s_idx)
            ws = minf.workspace(minf.OP_SPARSE_ATTN_VS, shp, 1, device=q.device)
            minf.minf_sparse_attn_vs(q, k, v, hd, index, o=self.o, lse=self.lse, ws=ws)
        elif pattern == "block_sparse":
            blk_idx, blk_cnt = minf.minf_estimate_bs(q, k, hd, int(setting))
            ws = minf.workspace(minf.OP_SPARSE_ATTN_BS, shp, 1, device=q.device)
            minf.minf_sparse_attn_bs(q, k, v, hd, blk_idx, blk_cnt, o=self.o, lse=self.lse, ws=ws)
        else:
            raise ValueError(f"unknown pattern {pattern!r}")
        code = minf.minf_get_device_status(ws)
        if code:
            raise minf.MinfError(f"{pattern} attention", code)
        tiles, _ = minf.attn_counters(ws)
        return tiles, self._kept(head)


def search_patterns(q, k, v, heads=None, candidates=None, reference=DEFAULT_REFERENCE, rows=None):
    """The pattern and setting of every head of one layer's pre-fill inputs
    (q [B, Hq, N, d], k and v [B, Hkv, N, d], bf16 on the GPU).  ``rows``
    restricts the kept-share average to some query rows.  Returns a list of
    HeadChoice, one per head."""
    candidates = candidates or DEFAULT_CANDIDATES
    ev = Evaluator(q, k, v, rows)
    N = ev.N
    heads = list(range(q.shape[1])) if heads is None else list(heads)
    out = []
    for h in heads:
        ref_pat, ref_set = reference
        budget, _ = ev.run(h, ref_pat, _clamp(ref_pat, ref_set, N))
        trials = []
        for pat in PATTERNS:
            seen = set()
            for st in candidates.get(pat, []):
                st = _clamp(pat, st, N)
                if st in seen:
                    continue
                seen.add(st)
                tiles, kept = ev.run(h, pat, st)
                trials.append(Trial(pat, st, tiles, kept))
        out.append(HeadChoice(h, budget, choose(trials, budget), trials))
    return out


def main(argv=None):
    """Searches one seeded synthetic layer and prints the table as JSON."""
    from . import workloads as wl
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--N", type=int, default=None)
    ap.add_argument("--heads", type=int, nargs="*", default=None)
    args = ap.parse_args(argv)
    w = wl.config(args.config, N=args.N)
    q, k, v = wl.make_qkv(w, "cuda")
    res = search_patterns(q, k, v, heads=args.heads)
    for r in res:
        c = r.choice
        print(json.dumps({"head": r.head, "budget_tiles": r.budget_tiles,
                          "pattern": c.pattern if c else None, "setting": c.setting if c else None,
                          "tiles": c.tiles if c else None, "kept": c.kept if c else None}))


if __name__ == "__main__":
    main()
