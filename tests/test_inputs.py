"""Host checks of the seeded input recipes: the block-mask generators that the
GPU tests and the bench share, checked position by position against the
oracle's expansion of a block mask and its causal filter."""
import numpy as np
import pytest

import oracle
from seeded_inputs import block_mask, block_mask_pairs


@pytest.mark.parametrize("n", [128, 300, 1024])
def test_causal_recipe_is_the_causal_filter(n):
    keep = oracle.block_mask_keep(block_mask("causal", n), n)
    assert np.array_equal(keep, oracle.keep_mask(n, n, True))
    assert np.array_equal(oracle.block_mask_keep(block_mask("full", n), n),
                          oracle.keep_mask(n, n, False))


@pytest.mark.parametrize("n,w", [(640, 1), (640, 3), (1000, 2), (512, 9)])
def test_window_recipe_keeps_the_last_w_tiles_causally(n, w):
    keep = oracle.block_mask_keep(block_mask(f"window:{w}", n), n)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    assert np.array_equal(keep, (j <= i) & (i // 128 - j // 128 < w))


def test_random_recipe_is_seeded_and_causal():
    a = block_mask("random:0.5:7", 2048)
    assert np.array_equal(a, block_mask("random:0.5:7", 2048))
    assert not np.array_equal(a, block_mask("random:0.5:8", 2048))
    assert np.all(np.diag(a) == 2)
    assert np.all(np.triu(a, 1) == 0)
    assert set(np.unique(np.tril(a, -1))) <= {0, 1}
    assert np.all(block_mask("random:1:0", 1024) == block_mask("causal", 1024))


def test_pair_count_follows_the_causal_convention():
    n = 16384
    assert block_mask_pairs(block_mask("causal", n)) == n * n / 2
    assert block_mask_pairs(block_mask("full", n)) == n * n
    # window of W tiles: W - 1 full tiles and a half per query tile, fewer at the start
    t, w = n // 128, 16
    full_tiles = sum(min(r, w - 1) for r in range(t))
    assert block_mask_pairs(block_mask(f"window:{w}", n)) == 128 * 128 * (full_tiles + t / 2)


def test_bad_specs_are_rejected():
    for spec in ("window:0", "diagonal", "window"):
        with pytest.raises((ValueError, IndexError)):
            block_mask(spec, 256)


def test_two_tile_window_is_local_to_three_tiles():
    # the reasoning the long-mask GPU test relies on: under window:2, query
    # tile t's O, LSE, dQ and key tile t's dK, dV depend only on tiles t-1..t+1
    from seeded_inputs import draw, as_f64
    T, d = 6, 8
    N = T * 128 - 50
    q, k, v, do = (as_f64(x) for x in draw(1, 1, N, d, 5, "f32"))
    full = oracle.backward(q, k, v, do, d ** -0.5, keep=oracle.block_mask_keep(block_mask("window:2", N), N))
    for t in (1, 3, T - 2):
        lo, hi = 128 * (t - 1), min(N, 128 * (t + 2))
        n = hi - lo
        keep = oracle.block_mask_keep(block_mask("window:2", n), n)
        loc = oracle.backward(*(x[:, :, lo:hi] for x in (q, k, v, do)), d ** -0.5, keep=keep)
        for name in ("O", "LSE", "dQ", "dK", "dV"):
            np.testing.assert_allclose(loc[name][0, 0, 128:256], full[name][0, 0, lo + 128:lo + 256],
                                       rtol=1e-12, atol=1e-13)
