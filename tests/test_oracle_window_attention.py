"""Pins for the sliding-window attention oracle against facts that are not
the oracle: torch's scaled-dot-product attention (a library routine) with an
explicit band mask, its causal special case, and closed forms."""
import numpy as np
import pytest
import torch

from oracle import sliding_window_attention


def _rand(B=2, H=3, N=40, d=8, seed=0):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, N, d)), r.standard_normal((B, H, N, d)),
            r.standard_normal((B, H, N, d)))


def _sdpa(q, k, v, mask=None, causal=False):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))  # noqa: E731
    with torch.no_grad():
        o = torch.nn.functional.scaled_dot_product_attention(
            t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
            is_causal=causal)
    return o.numpy()


@pytest.mark.parametrize("window", [1, 2, 7, 16, 39])
def test_equals_library_attention_with_a_band_mask(window):
    q, k, v = _rand()
    N = q.shape[2]
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    band = (j <= i) & (j > i - window)          # True = attend
    ref = _sdpa(q, k, v, mask=band)
    np.testing.assert_allclose(sliding_window_attention(q, k, v, window), ref, rtol=0, atol=1e-12)


def test_window_covering_the_sequence_is_causal_attention():
    q, k, v = _rand(N=33, seed=1)
    ref = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(sliding_window_attention(q, k, v, 33), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sliding_window_attention(q, k, v, 1000), ref, rtol=0, atol=1e-12)


def test_window_of_one_returns_the_values():
    q, k, v = _rand(seed=2)
    assert np.array_equal(sliding_window_attention(q, k, v, 1), v)


def test_constant_values_pass_through():
    # the weights of every row sum to one
    q, k, _ = _rand(seed=3)
    v = np.broadcast_to(np.arange(8.0), q.shape)
    np.testing.assert_allclose(sliding_window_attention(q, k, v, 5), v, rtol=0, atol=1e-12)


def test_planted_window_off_by_one_is_caught():
    q, k, v = _rand(seed=4)
    N = q.shape[2]
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    ref = _sdpa(q, k, v, mask=(j <= i) & (j > i - 8))
    assert np.abs(sliding_window_attention(q, k, v, 9) - ref).max() > 1e-3


def test_sampled_positions_match_the_full_computation():
    q, k, v = _rand(N=50, seed=5)
    full = sliding_window_attention(q, k, v, 9)
    idx = [0, 8, 9, 31, 49]
    np.testing.assert_array_equal(sliding_window_attention(q, k, v, 9, t_index=idx), full[:, :, idx])
