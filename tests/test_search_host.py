"""Host logic of the offline pattern search: which candidate a head takes
from measured (tiles, kept share) pairs."""
from dynamic_sparse_attention_minf_b200.search import Trial, choose, _clamp


def T(p, s, tiles, kept):
    return Trial(p, s, tiles, kept)


def test_largest_fitting_setting_per_pattern_then_most_kept():
    trials = [T("a_shape", 1, 10, 0.50), T("a_shape", 2, 20, 0.70), T("a_shape", 3, 40, 0.95),
              T("vertical_slash", 1, 15, 0.80), T("vertical_slash", 2, 30, 0.90),
              T("block_sparse", 1, 12, 0.60), T("block_sparse", 2, 25, 0.85)]
    # budget 30: a_shape 2 (0.70), vertical_slash 2 (0.90), block_sparse 2 (0.85)
    c = choose(trials, 30)
    assert (c.pattern, c.setting) == ("vertical_slash", 2)
    # budget 25: vertical_slash 1 (0.80) loses to block_sparse 2 (0.85)
    c = choose(trials, 25)
    assert (c.pattern, c.setting) == ("block_sparse", 2)
    # a larger budget lets the long A-shape window win
    c = choose(trials, 40)
    assert (c.pattern, c.setting) == ("a_shape", 3)


def test_ties_go_to_the_cheaper_and_nothing_fits():
    trials = [T("a_shape", 1, 20, 0.9), T("vertical_slash", 1, 10, 0.9), T("block_sparse", 1, 30, 0.99)]
    c = choose(trials, 25)
    assert (c.pattern, c.tiles) == ("vertical_slash", 10)
    assert choose(trials, 5) is None


def test_the_most_expensive_fitting_setting_competes_even_if_it_keeps_less():
    # within a pattern the budget decides, not the measured share
    trials = [T("block_sparse", 1, 10, 0.9), T("block_sparse", 2, 20, 0.8)]
    assert choose(trials, 20).setting == 2


def test_settings_clamped_to_the_prompt():
    assert _clamp("a_shape", (128, 32768), 4096) == (128, 4096)
    assert _clamp("vertical_slash", (2000, 12192), 4096) == (2000, 4096)
    assert _clamp("block_sparse", 400, 4096) == 64
