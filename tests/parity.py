"""Comparison helpers shared by the GPU parity tests (no method arithmetic:
the expected values always come from the oracle)."""
import numpy as np

MAX_ABS = 2e-2     # attention outputs, bf16 with fp32 accumulation
MEAN_ABS = 2e-3
LSE_ABS = 1e-2
GAP = 1e-5         # index sets may differ only where the oracle's score is this close to the cut


def check_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3g}"


def check_lse(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got)), what
    if fin.any():
        err = np.abs(got[fin] - ref[fin]).max()
        assert err <= LSE_ABS, f"{what}: lse err {err:.3g}"


def check_index_set(got, ref, scores, forced=None, gap=GAP, what=""):
    """Bit-exact index sets, except that an index may swap across the cut when
    the oracle's score of it is within `gap` of the k-th score."""
    got = np.asarray(got, np.int64)
    ref = np.asarray(ref, np.int64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.diff(got) > 0), f"{what}: not strictly ascending"
    if np.array_equal(got, ref):
        return 0
    sc = np.array(scores, np.float64, copy=True)
    if forced is not None:
        sc[forced] = np.inf
    tau = np.sort(sc[ref])[0]
    diff = np.setxor1d(got, ref)
    bad = diff[np.abs(sc[diff] - tau) >= gap]
    assert bad.size == 0, f"{what}: {diff.size} differing indices, {bad.size} beyond the gap rule: {bad[:8]}"
    return diff.size


def tile_gather_lists(vcnt, vidx):
    """The per-128-row-tile gather lists, composed from per-64-row-block
    vertical lists (vcnt [nb], vidx [nb, k_v], the oracle's): for tile t the
    columns of block 2t + 1's list in order, each flagged with the blocks that
    list it (bit 30: block 2t, bit 31: block 2t + 1), then the columns of block
    2t's list that block 2t + 1 does not list (bit 30).  Returns (count [nt],
    list of uint32 arrays)."""
    nb = len(vcnt)
    cnts, lists = [], []
    for t in range(nb // 2):
        l0 = np.asarray(vidx[2 * t, :vcnt[2 * t]], np.uint64)
        l1 = np.asarray(vidx[2 * t + 1, :vcnt[2 * t + 1]], np.uint64)
        first = l1 | (np.isin(l1, l0).astype(np.uint64) << 30) | np.uint64(1 << 31)
        second = l0[~np.isin(l0, l1)] | np.uint64(1 << 30)
        e = np.concatenate([first, second]).astype(np.uint32)
        cnts.append(len(e))
        lists.append(e)
    return np.asarray(cnts, np.int64), lists


def tile_list_errors(gcnt, gidx, vcnt, vidx):
    """Tiles whose GPU gather list (gcnt [nt], gidx [nt, k_v] int32) differs
    from the one composed from the oracle's block lists."""
    cnts, lists = tile_gather_lists(vcnt, vidx)
    gidx = np.asarray(gidx).view(np.uint32)
    return [t for t in range(len(cnts))
            if gcnt[t] != cnts[t] or not np.array_equal(gidx[t, :cnts[t]], lists[t])]
