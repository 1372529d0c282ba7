"""The tie-aware row check of ``gptq_parity`` on the CPU, with the oracle's
own layers: it accepts the oracle's layer and a row that flipped its tightest
decision (a tie at fp32 resolution) and then follows on from different
values; it rejects a flipped decision far from its boundary, a code two steps
away and too many tie rows.  The flips are planted by moving one weight
across its rounding boundary: column q's running weight depends only on
columns <= q, so the row is the oracle's up to that column and then the
cascade the method gives from there."""
import numpy as np
import pytest

from gptq_parity import TIE_MARGIN, check_layer_up_to_ties, decision_margins
from oracle import gptq_oracle as O


@pytest.fixture(scope="module")
def layer():
    rng = np.random.default_rng(17)
    w = rng.standard_normal((64, 512)) * 0.02
    x = rng.standard_normal((2048, 512))
    x[:, rng.permutation(512)[:4]] *= 20.0
    hd, _ = O.dampen(O.hessian(x), 0.01)
    u = O.hinv_cholesky_upper(hd)
    ref = O.gptq_quantize(w, u, 4, 0, False, 128)
    margins = decision_margins(ref[3], ref[4], np.diag(u), ref[1], 0)
    return w, u, ref, margins


def _nudged(layer, r, c, steps):
    """The layer with W[r, c] moved so that its running weight x (in units
    of s) lands just past the nearer rounding boundary (steps = 1) or
    `steps` codes away on that side."""
    w, u, ref, _ = layer
    s = ref[1][r, 0]
    x = (ref[3][r, c] + ref[4][r, c] * u[c, c]) / s
    k = np.rint(x)
    side = 1.0 if x >= k else -1.0
    target = k + side * (steps - 0.5 + 1e-3)
    w2 = w.copy()
    w2[r, c] += (target - x) * s
    out = O.gptq_quantize(w2, u, 4, 0, False, 128)
    assert np.array_equal(out[1], ref[1])   # the row's range is unchanged
    return out


def _interior(layer, order):
    """The (row, column) of the first decision in `order` whose weight is
    not its row's extreme (moving an extreme would move the per-channel
    range) and whose code has two steps of room on both sides."""
    w, _, ref, margins = layer
    for k in order:
        r, c = np.unravel_index(k, margins.shape)
        if w[r, c] not in (w[r].min(), w[r].max()) and 2 <= ref[0][r, c] <= 13:
            return int(r), int(c)
    raise AssertionError("no interior decision")


def test_decision_margins_closed_form():
    """With U = cI nothing propagates: the running weights are the weights."""
    rng = np.random.default_rng(3)
    w = rng.standard_normal((8, 64)) * 0.02
    u = np.eye(64) / np.sqrt(3.0)
    codes, sc, ze, wh, err = O.gptq_quantize(w, u, 3, 16, False, 32)
    m = decision_margins(wh, err, np.diag(u), sc, 16)
    x = w / sc[:, np.arange(64) // 16]
    np.testing.assert_allclose(m, np.abs(x - np.floor(x) - 0.5), atol=1e-12)


def test_accepts_the_oracle_layer(layer):
    _, _, ref, margins = layer
    assert check_layer_up_to_ties(ref[0], ref[1], ref[2], ref[0], ref[1], ref[2], margins, 0) == []


def test_accepts_a_tie_and_its_cascade(layer):
    _, _, ref, margins = layer
    r, c = _interior(layer, np.argsort(margins, axis=None))
    assert margins[r, c] < TIE_MARGIN
    out = _nudged(layer, r, c, 1)
    assert (out[0][r] != ref[0][r]).sum() >= 1
    ties = check_layer_up_to_ties(out[0], out[1], out[2], ref[0], ref[1], ref[2], margins, 0)
    assert [(t[0], t[1]) for t in ties] == [(r, c)]


def test_rejects_a_flip_far_from_its_boundary(layer):
    _, _, ref, margins = layer
    order = np.argsort(margins, axis=None)[::-1]   # decisions far from a boundary first
    r, c = _interior(layer, order)
    assert margins[r, c] > 0.4
    out = _nudged(layer, r, c, 1)
    with pytest.raises(AssertionError, match="from the tie"):
        check_layer_up_to_ties(out[0], out[1], out[2], ref[0], ref[1], ref[2], margins, 0)


def test_rejects_a_code_two_steps_away(layer):
    _, _, ref, margins = layer
    r, c = _interior(layer, np.argsort(margins, axis=None))
    out = _nudged(layer, r, c, 2)
    assert abs(out[0][r, c] - ref[0][r, c]) == 2
    with pytest.raises(AssertionError, match="off by more than 1"):
        check_layer_up_to_ties(out[0], out[1], out[2], ref[0], ref[1], ref[2], margins, 0)


def test_rejects_more_tie_rows_than_allowed(layer):
    _, _, ref, margins = layer
    r, c = _interior(layer, np.argsort(margins, axis=None))
    out = _nudged(layer, r, c, 1)
    with pytest.raises(AssertionError, match="rows met a tie"):
        check_layer_up_to_ties(out[0], out[1], out[2], ref[0], ref[1], ref[2], margins, 0,
                               max_tie_rows=0)
