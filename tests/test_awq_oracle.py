"""Pins of the AWQ scale-search oracle (dingiv.github.io "量化" page, section
AWQ) against closed forms, special cases and the page's stated effect.

Each pin is chosen so that a plausible mistake fails it: a sum in place of
the mean, a missing absolute value, a wrong exponent or grid, a missing
division by s (the equivalent transform), a wrong loss.
"""
import numpy as np
import pytest

from oracle import awq_oracle as A
from oracle import gptq_oracle as O


def test_channel_scale_closed_form():
    x = np.array([[1.0, -2.0, 0.0], [3.0, 4.0, 0.0], [-2.0, 0.0, 0.0]])
    np.testing.assert_array_equal(A.channel_scale(x), [2.0, 2.0, 0.0])


def test_alpha_grid_is_twenty_points_over_the_closed_interval():
    g = A.alpha_grid()
    assert len(g) == 20 and g[0] == 0.0 and g[-1] == 1.0
    np.testing.assert_allclose(np.diff(g), 1.0 / 19, rtol=1e-12)
    assert g[7] == 7 / 19  # written as a / 19 exactly


def test_scales_closed_form_and_silent_channels():
    sx = np.array([4.0, 0.25, 0.0, 1.0])
    np.testing.assert_array_equal(A.scales_for(sx, 0.5), [2.0, 0.5, 1.0, 1.0])
    np.testing.assert_array_equal(A.scales_for(sx, 0.0), [1.0, 1.0, 1.0, 1.0])
    np.testing.assert_array_equal(A.scales_for(sx, 1.0), [4.0, 0.25, 1.0, 1.0])


def _layer(seed=0, d_row=24, d_col=256, n=600, outliers=()):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((d_row, d_col)) * 0.02
    x = rng.standard_normal((n, d_col))
    for k, f in outliers:
        x[:, k] *= f
    return w, x


@pytest.mark.parametrize("group", [0, 64, 128])
def test_alpha_zero_is_round_to_nearest(group):
    w, x = _layer(1)
    r = A.quantize_scaled(w, A.scales_for(A.channel_scale(x), 0.0), 4, group)
    ref = O.rtn(w, 4, group)
    assert np.array_equal(r["codes"], ref["codes"])
    np.testing.assert_array_equal(r["scales"], ref["scales"])
    np.testing.assert_array_equal(r["w_hat"], ref["w_hat"])


@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_uniform_power_of_two_activations_make_every_alpha_equal(dtype):
    """s_X = 2^3 on every channel: W diag(s) = 2^(3 alpha) W; the min-max
    quantizer is scale-equivariant, so the codes and zero points are those of
    RTN and, once divided by s, W^ is RTN's W^ exactly, for every alpha."""
    w, _ = _layer(2)
    h = 2.0 * np.eye(w.shape[1])
    sx = np.full(w.shape[1], 8.0)
    res = A.search(w, h, sx, 4, 128, dtype=dtype)
    rt = O.rtn(w, 4, 128)
    for alpha in res["alphas"]:
        s = A.scales_for(sx, alpha, dtype)
        if not np.all(np.log2(s) == np.round(np.log2(s))):
            continue  # only exact powers of two scale without rounding
        r = A.quantize_scaled(w, s, 4, 128, dtype)
        assert np.array_equal(r["codes"], O.rtn(w.astype(dtype), 4, 128, dtype=dtype)["codes"])
        np.testing.assert_allclose(r["w_hat"], O.rtn(w.astype(dtype), 4, 128, dtype=dtype)["w_hat"],
                                   rtol=0, atol=0)
    if dtype == np.float64:
        assert res["best"] == 0
        np.testing.assert_allclose(res["losses"][0], O.layer_loss_hessian(w, rt["w_hat"], h),
                                   rtol=1e-14)


def test_losses_equal_the_direct_output_error():
    """The search's H-form loss equals ||W X - W^ X||^2 computed from X."""
    w, x = _layer(3, outliers=[(5, 20.0), (77, 8.0)])
    h = O.hessian(x)
    res = A.search(w, h, A.channel_scale(x), 4, 64)
    for a in (0, 7, 19):
        s = A.scales_for(A.channel_scale(x), res["alphas"][a])
        r = A.quantize_scaled(w, s, 4, 64)
        direct = O.layer_loss_direct(w, r["w_hat"], x)
        assert res["losses"][a] == pytest.approx(direct, rel=1e-9)
    assert res["losses"][res["best"]] == res["losses"].min()
    assert res["best"] == int(np.flatnonzero(res["losses"] == res["losses"].min())[0])


def test_scaling_salient_channels_beats_plain_rounding():
    """The page's claim on a layer with a few large-activation channels: some
    alpha > 0 lowers the output error below round-to-nearest (alpha = 0)."""
    w, x = _layer(4, d_row=64, d_col=512, n=2000,
                  outliers=[(3, 40.0), (100, 25.0), (300, 60.0), (411, 30.0)])
    h = O.hessian(x)
    res = A.search(w, h, A.channel_scale(x), 4, 128)
    assert res["best"] > 0
    assert res["losses"][res["best"]] < 0.9 * res["losses"][0]
    # the reported quantization is the one at the best alpha
    s = A.scales_for(A.channel_scale(x), res["alphas"][res["best"]])
    assert np.array_equal(res["codes"], A.quantize_scaled(w, s, 4, 128)["codes"])
    np.testing.assert_array_equal(res["s"], s)
