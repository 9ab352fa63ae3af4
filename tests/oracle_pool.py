"""Oracle checks of one full-size attention layer, one query head per task,
run in a process pool (started with spawn, before or after CUDA use alike).

The parent puts the layer's bf16 inputs (raw bits) and the GPU's large index
arrays into shared memory; each worker converts what its head needs to
float64 and runs the oracle on it.  Workers use only numpy and the oracle.
"""
from __future__ import annotations

import os
from dataclasses import dataclass
from multiprocessing import shared_memory

import numpy as np

from oracle import minf_oracle as orc
from tests.parity import GAP, LSE_ABS, MAX_ABS, MEAN_ABS, tile_list_errors


@dataclass
class Shared:
    name: str
    shape: tuple
    dtype: str

    def attach(self):
        shm = shared_memory.SharedMemory(name=self.name)
        return shm, np.ndarray(self.shape, dtype=np.dtype(self.dtype), buffer=shm.buf)


def share(arr: np.ndarray, keep: list) -> Shared:
    shm = shared_memory.SharedMemory(create=True, size=max(arr.nbytes, 1))
    view = np.ndarray(arr.shape, dtype=arr.dtype, buffer=shm.buf)
    view[...] = arr
    keep.append(shm)
    return Shared(shm.name, arr.shape, arr.dtype.str)


def bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact: a bf16 value is the top half of the float32 with the same bits."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _index_set_errors(got, ref, scores, forced=None):
    """Indices that differ from the oracle's set beyond the score-gap rule."""
    got = np.asarray(got, np.int64)
    ref = np.asarray(ref, np.int64)
    if got.shape != ref.shape:
        return -1, "shape"
    if np.array_equal(got, ref):
        return 0, ""
    if not np.all(np.diff(got) > 0):
        return -1, "not ascending"
    sc = np.array(scores, np.float64, copy=True)
    if forced is not None:
        sc[forced] = np.inf
    tau = np.sort(sc[ref])[0]
    diff = np.setxor1d(got, ref)
    bad = diff[np.abs(sc[diff] - tau) >= GAP]
    return int(diff.size), ("" if bad.size == 0 else f"{bad.size} beyond gap, e.g. {bad[:4].tolist()}")


def _attention_rows(q_rows, k64, v64, rows, mask_fn, sc):
    """The oracle's masked attention on sampled rows, a few rows at a time."""
    step = max(1, min(64, (1 << 23) // k64.shape[0]))
    O = np.zeros((rows.size, v64.shape[1]))
    L = np.zeros(rows.size)
    for a in range(0, rows.size, step):
        O[a:a + step], L[a:a + step] = orc.attention_rows(q_rows[a:a + step], k64, v64,
                                                          mask_fn(rows[a:a + step]), sc)
    return O, L


def check_head(task: dict) -> dict:
    """One query head: its index estimation (full), index build (full) and
    attention on the sampled rows, against the oracle."""
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    h, kv, pat = task["head"], task["kv"], task["pattern"]
    N, d = task["N"], task["d"]
    sc = orc.default_scale(d)
    out = {"head": h, "pattern": pat, "errors": [], "flips": 0}
    shms = []
    try:
        s_q, Q = task["Q"].attach(); shms.append(s_q)
        s_k, K = task["K"].attach(); shms.append(s_k)
        s_v, V = task["V"].attach(); shms.append(s_v)
        k64 = bf16_bits_to_f64(K[kv])
        v64 = bf16_bits_to_f64(V[kv])
        rows = np.asarray(task["rows"])
        if pat == "vs":
            q_last = bf16_bits_to_f64(Q[h, N - task["last_q"]:])
            rv, rs = orc.vs_estimate(q_last, k64, sc)
            ov, os_ = orc.vs_select(rv, rs, task["k_v"], task["k_s"])
            gv, gs = task["v_idx"], task["s_idx"]
            n1, e1 = _index_set_errors(gv, ov, rv)
            n2, e2 = _index_set_errors(gs, os_, rs, forced=0)
            out["flips"] += max(n1, 0) + max(n2, 0)
            if e1:
                out["errors"].append(f"vertical: {e1}")
            if e2:
                out["errors"].append(f"slash: {e2}")
            # index build on the GPU's own sets: bit-exact
            groups, vcnt, vidx = orc.vs_build_index(gv, gs, N)
            if not np.array_equal(task["grp"], groups):
                out["errors"].append("groups differ")
            if not np.array_equal(task["tgrp"], orc.vs_groups(gs, block=128)):
                out["errors"].append("tile groups differ")
            s_vi, VI = task["vidx"].attach(); shms.append(s_vi)
            gcnt = task["vcnt"]
            if not np.array_equal(gcnt, vcnt):
                out["errors"].append("vcnt differs")
            else:
                bad = [b for b in range(N // 64) if not np.array_equal(VI[task["slot"], b, :vcnt[b]], vidx[b, :vcnt[b]])]
                if bad:
                    out["errors"].append(f"vidx differs in {len(bad)} blocks, e.g. {bad[:4]}")
            if "tvidx" in task:
                s_tv, TV = task["tvidx"].attach(); shms.append(s_tv)
                bad = tile_list_errors(task["tvcnt"], TV[task["slot"]], vcnt, vidx)
                if bad:
                    out["errors"].append(f"tile gather lists differ in {len(bad)} tiles, e.g. {bad[:4]}")
            mask_fn = lambda r: orc.mask_vs(r, N, gv, gs)
            if "ox_rows" in task:
                # element-exact variant on the same sets: its per-tile vertical
                # lists bit-exactly, its outputs on the sampled rows
                _, xcnt, xidx = orc.vs_exact_index(gv, gs, N)
                s_xi, XI = task["xidx"].attach(); shms.append(s_xi)
                if not np.array_equal(task["xcnt"], xcnt):
                    out["errors"].append("exact vcnt differs")
                else:
                    bad = [t for t in range(N // 128)
                           if not np.array_equal(XI[task["slot"], t, :xcnt[t]], xidx[t, :xcnt[t]])]
                    if bad:
                        out["errors"].append(f"exact vidx differs in {len(bad)} tiles, e.g. {bad[:4]}")
                q_rows = bf16_bits_to_f64(Q[h, rows])
                OX, LX = _attention_rows(q_rows, k64, v64, rows, lambda r: orc.mask_vs_exact(r, N, gv, gs), sc)
                ex = np.abs(task["ox_rows"].astype(np.float64) - OX)
                out["x_max_abs"] = float(ex.max())
                if not np.isfinite(task["ox_rows"]).all() or ex.max() > MAX_ABS or ex.mean() > MEAN_ABS:
                    out["errors"].append(f"exact attention error max {ex.max():.3g} mean {ex.mean():.3g}")
                lx = np.abs(task["lsex_rows"] - LX)
                if lx[np.isfinite(LX)].max() > LSE_ABS:
                    out["errors"].append(f"exact lse error {lx[np.isfinite(LX)].max():.3g}")
        elif pat == "bs":
            qh = bf16_bits_to_f64(Q[h])
            qbar, kbar = orc.bs_pool(qh), orc.bs_pool(k64)
            del qh
            nb = N // 64
            gi, gc = task["blk_idx"], task["blk_cnt"]
            step = 512
            for b0 in range(0, nb, step):
                b = np.arange(b0, min(nb, b0 + step))
                ri, rc = orc.bs_select_pooled(qbar, kbar, sc, task["k_b"], blocks=b)
                t = orc.bs_scores(qbar[b], kbar, sc)      # the scores the gap rule reads
                if not np.array_equal(rc, gc[b]):
                    out["errors"].append(f"blk_cnt differs near block {b0}")
                    break
                for a, bb in enumerate(b):
                    n3, e3 = _index_set_errors(gi[bb, :gc[bb]], ri[a, :rc[a]], t[a, :bb + 1], forced=bb)
                    out["flips"] += max(n3, 0)
                    if e3:
                        out["errors"].append(f"block {bb}: {e3}")
                        break
                if out["errors"]:
                    break
            mask_fn = lambda r: orc.mask_bs(r, N, gi, gc)
        else:
            mask_fn = lambda r: orc.mask_ashape(r, N, task["n_sink"], task["n_local"])
        q_rows = bf16_bits_to_f64(Q[h, rows])
        O, L = _attention_rows(q_rows, k64, v64, rows, mask_fn, sc)
        err = np.abs(task["o_rows"].astype(np.float64) - O)
        out["max_abs"] = float(err.max())
        out["mean_abs"] = float(err.mean())
        lerr = np.abs(task["lse_rows"] - L)
        out["lse_abs"] = float(lerr[np.isfinite(L)].max())
        if not np.isfinite(task["o_rows"]).all():
            out["errors"].append("non-finite output")
        if out["max_abs"] > MAX_ABS or out["mean_abs"] > MEAN_ABS:
            out["errors"].append(f"attention error max {out['max_abs']:.3g} mean {out['mean_abs']:.3g}")
        if out["lse_abs"] > LSE_ABS:
            out["errors"].append(f"lse error {out['lse_abs']:.3g}")
    except Exception as exc:  # report, do not hang the pool
        out["errors"].append(f"exception: {exc!r}")
    finally:
        for s in shms:
            s.close()
    return out
