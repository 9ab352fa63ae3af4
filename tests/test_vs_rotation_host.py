"""Index arithmetic of the Vertical-Slash pass-2 diagonal sums, on the CPU.

Pass 2 holds one key per thread (key 32 w + L of the tile in lane L of warp
w) and query row q in register q.  At step q lane L reads row q of lane
(q - L) mod 32 and adds it to the sum of the warp-local diagonal
q - ((q - L) mod 32), one of L - 32, L, L + 32, kept in slot diagonal + 32 of
96; the tile diagonal kd (entries (q, key q - kd + 127)) is slot
kd - 95 + 32 w of warp w.  These checks restate that mapping and show that
every entry of the 64 x 128 tile lands in exactly one slot and every slot in
exactly one tile diagonal, the one the entry belongs to."""
import numpy as np

LANES, ROWS, WARPS, SLOTS = 32, 64, 4, 96


def _received():
    """(warp, lane, step) -> (source lane, slot) of the value lane L receives."""
    out = {}
    for w in range(WARPS):
        for L in range(LANES):
            for q in range(ROWS):
                src = (q - L) % LANES
                out[(w, L, q)] = (src, q - src + 32)
    return out


def test_every_entry_taken_once_by_the_right_slot():
    seen = np.zeros((WARPS * LANES, ROWS), int)
    for (w, L, q), (src, slot) in _received().items():
        key = 32 * w + src
        seen[key, q] += 1
        diag = q - src  # warp-local diagonal: row minus key within the warp
        assert diag in (L - 32, L, L + 32)
        assert slot == diag + 32 and 0 <= slot < SLOTS
    assert (seen == 1).all()


def test_slots_combine_into_tile_diagonals():
    rng = np.random.default_rng(3)
    p = rng.random((WARPS * LANES, ROWS))  # p[key, row]
    part = np.zeros((WARPS, SLOTS))
    for (w, L, q), (src, slot) in _received().items():
        part[w, slot] += p[32 * w + src, q]
    ref = np.zeros(191)
    for key in range(WARPS * LANES):
        for q in range(ROWS):
            ref[q - key + 127] += p[key, q]
    got = np.zeros(191)
    for kd in range(191):
        for w in range(WARPS):
            sl = kd - 95 + 32 * w
            if 0 <= sl < SLOTS:
                got[kd] += part[w, sl]
    np.testing.assert_allclose(got, ref, rtol=1e-12)
    assert not part[:, 0].any()  # the slot of diagonal -32 never receives a value


def test_each_slot_lies_in_one_tile_diagonal():
    owner = {}
    for kd in range(191):
        for w in range(WARPS):
            sl = kd - 95 + 32 * w
            if 0 <= sl < SLOTS:
                assert (w, sl) not in owner
                owner[(w, sl)] = kd
    # every slot is read by exactly one diagonal, except slot 0 of the last
    # warp, whose diagonal (-1) lies outside the tile; slot 0 always holds 0
    assert sorted(owner) == [(w, s) for w in range(WARPS) for s in range(SLOTS) if (w, s) != (WARPS - 1, 0)]
