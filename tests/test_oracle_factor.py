"""Pins of the factor route's reading (CPU, no GPU).

Section GPTQ of the dingiv.github.io "量化" page subtracts e_q U[q, k] from
every later column, with e_q = (w_q - w^_q) / U_qq.  So W = W^ + E U (pinned
in test_oracle.test_gptq_error_identity), E = (W - W^) V with V = U^-1, and
the running weights at the start of a 128-column block b are
W_b + sum_{a<b} (W - W^)_a V_ab U_bb.  ``O.factor_blocks`` holds U_bb on the
diagonal blocks and V_ab U_bb right of them.  Here a plain fp64 sweep through
that F must give the oracle's layer exactly (up to fp64 rounding), and F with
a planted mistake must not.
"""
import numpy as np
import pytest

from oracle import gptq_oracle as O


def _layer(seed, d_row, d_col, n, outliers=4, dead=()):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((d_row, d_col)) * 0.02
    x = rng.standard_normal((n, d_col))
    x[:, rng.permutation(d_col)[:outliers]] *= 20.0
    x[:, list(dead)] = 0.0
    hd, dead_mask = O.dampen(O.hessian(x), 0.01)
    return w, hd, dead_mask


def _sweep_factor(w, f, bits, group, sym, block=128, dead=None):
    """Quantize through F: inside a block as through U (its diagonal block),
    across blocks W[:, right] += (W - W^)[:, block] F[block, right]."""
    w = np.array(w, dtype=np.float64, copy=True)
    if dead is not None:
        w[:, np.asarray(dead, dtype=bool)] = 0.0
    wo = w.copy()
    d_row, d_col = w.shape
    g = group or d_col
    n_groups = d_col // g if group else 1
    codes = np.zeros((d_row, d_col), dtype=np.int64)
    scales = np.zeros((d_row, n_groups))
    zeros = np.zeros((d_row, n_groups))
    w_hat = np.zeros_like(w)
    if group == 0:
        scales[:, 0], zeros[:, 0] = O.quant_params(wo, bits, sym)
    for j0 in range(0, d_col, block):
        j1 = min(j0 + block, d_col)
        for q in range(j0, j1):
            gi = q // g if group else 0
            if group and q % g == 0:
                scales[:, gi], zeros[:, gi] = O.quant_params(w[:, q:q + g], bits, sym)
            s, z = scales[:, gi], zeros[:, gi]
            c = O.quantize(w[:, q], s, z, bits)
            wq = O.dequantize(c, s, z)
            e = (w[:, q] - wq) / f[q, q]
            w[:, q + 1:j1] -= np.outer(e, f[q, q + 1:j1])
            codes[:, q], w_hat[:, q] = c, wq
        if j1 < d_col:
            w[:, j1:] += (wo[:, j0:j1] - w_hat[:, j0:j1]) @ f[j0:j1, j1:]
    return codes, scales, zeros, w_hat


CASES = [  # seed, d_row, d_col, bits, group, sym
    (1, 24, 512, 4, 0, False),
    (2, 24, 512, 4, 128, False),
    (3, 16, 384, 3, 32, True),
    (4, 16, 416, 2, 32, False),     # ragged last block (416 = 3 * 128 + 32)
    (5, 8, 640, 8, 128, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[1:])))
def test_sweep_through_f_is_the_oracle_layer(case):
    seed, d_row, d_col, bits, group, sym = case
    w, hd, _ = _layer(seed, d_row, d_col, 4 * d_col)
    u = O.hinv_cholesky_upper(hd)
    f = O.factor_blocks(u)
    ref = O.gptq_quantize(w, u, bits, group, sym, 128)
    got = _sweep_factor(w, f, bits, group, sym)
    assert np.array_equal(got[0], ref[0])
    np.testing.assert_allclose(got[1], ref[1], rtol=1e-12)
    assert np.array_equal(got[2], ref[2])
    np.testing.assert_allclose(got[3], ref[3], rtol=1e-12, atol=1e-15)


def test_sweep_through_f_with_dead_channels():
    w, hd, dead = _layer(9, 16, 384, 1536, dead=(3, 130, 300))
    assert dead.sum() == 3
    u = O.hinv_cholesky_upper(hd)
    ref = O.gptq_quantize(w, u, 4, 128, False, 128, dead=dead)
    got = _sweep_factor(w, O.factor_blocks(u), 4, 128, False, dead=dead)
    assert np.array_equal(got[0], ref[0])
    np.testing.assert_allclose(got[1], ref[1], rtol=1e-12)


@pytest.mark.parametrize("plant", ["no_diag_factor", "diag_transposed", "row_block_factor"])
def test_sweep_rejects_planted_mistakes(plant):
    """F_ab = V_ab (U_bb dropped), V_ab U_bb^T (transposed), or U_aa V_ab (the
    row block's factor on the left): each changes the layer."""
    w, hd, _ = _layer(2, 24, 512, 2048)
    u = O.hinv_cholesky_upper(hd)
    v = np.linalg.inv(u)
    f = O.factor_blocks(u)
    bad = f.copy()
    for b0 in range(128, 512, 128):
        ub = u[b0:b0 + 128, b0:b0 + 128]
        for a0 in range(0, b0, 128):
            vab = v[a0:a0 + 128, b0:b0 + 128]
            if plant == "no_diag_factor":
                bad[a0:a0 + 128, b0:b0 + 128] = vab
            elif plant == "diag_transposed":
                bad[a0:a0 + 128, b0:b0 + 128] = vab @ ub.T
            else:
                bad[a0:a0 + 128, b0:b0 + 128] = u[a0:a0 + 128, a0:a0 + 128] @ vab
    ref = O.gptq_quantize(w, u, 4, 128, False, 128)
    got = _sweep_factor(w, bad, 4, 128, False)
    assert not np.array_equal(got[0], ref[0])


def test_factor_blocks_against_reversed_cholesky():
    """V from the reversed Cholesky of H' (no inverse of U) gives the same
    off-diagonal blocks V_ab U_bb, and U_bb V_bb = I on the diagonal."""
    _, hd, _ = _layer(6, 1, 416, 1600)
    d = hd.shape[0]
    u = O.hinv_cholesky_upper(hd)
    f = O.factor_blocks(u)
    rev = np.arange(d)[::-1]
    v = np.linalg.cholesky(hd[np.ix_(rev, rev)])[np.ix_(rev, rev)]  # H' = V V^T, V upper
    assert np.allclose(np.tril(v, -1), 0.0)
    np.testing.assert_allclose(v @ v.T, hd, rtol=1e-12, atol=1e-12 * np.abs(hd).max())
    for b0 in range(0, d, 128):
        b1 = min(b0 + 128, d)
        np.testing.assert_allclose(f[b0:b1, b0:b1] @ v[b0:b1, b0:b1], np.eye(b1 - b0),
                                   atol=1e-10)
        if b0 == 0:
            continue
        ref = v[:b0, b0:b1] @ u[b0:b1, b0:b1]
        np.testing.assert_allclose(f[:b0, b0:b1], ref, rtol=1e-8,
                                   atol=1e-10 * max(1.0, np.abs(ref).max()))
    assert np.all(np.tril(f, -1) == 0.0)


def test_factor_blocks_closed_forms():
    c = 5.0
    hd, _ = O.dampen(c * np.eye(300), 0.01)
    f = O.factor_blocks(O.hinv_cholesky_upper(hd))
    np.testing.assert_allclose(f, np.eye(300) / np.sqrt(1.01 * c), rtol=1e-14)
    # H' block diagonal in 128-blocks: nothing couples the blocks
    rng = np.random.default_rng(3)
    h = np.zeros((256, 256))
    for b0 in (0, 128):
        a = rng.standard_normal((128, 400))
        h[b0:b0 + 128, b0:b0 + 128] = a @ a.T
    u = O.hinv_cholesky_upper(h)
    f = O.factor_blocks(u)
    assert np.abs(f[:128, 128:]).max() < 1e-12 * np.abs(u).max()
    np.testing.assert_allclose(f[128:, 128:], u[128:, 128:], rtol=1e-14)


@pytest.mark.parametrize("d", [200, 416, 640])
def test_factor_rows_match_blocks(d):
    _, hd, _ = _layer(d, 1, d, 4 * d)
    u = O.hinv_cholesky_upper(hd)
    f = O.factor_blocks(u)
    rows = np.array([0, 1, 127, 128, d // 2, d - 33, d - 1])
    got = O.factor_rows(u, rows)
    np.testing.assert_allclose(got, f[rows], rtol=1e-9, atol=1e-12 * np.abs(f).max())


def test_groups_wider_than_a_block_need_the_running_weights_of_g():
    """Why the factor route takes only group sizes that divide 128: a group
    of 256 reads its parameters at its first column from the running weights
    of both its blocks, and right of the current block F gives other partial
    sums than U (only the full sums at a block start agree).  The scales of
    the second group of 256 then differ from the oracle's."""
    w, hd, _ = _layer(8, 24, 512, 2048)
    u = O.hinv_cholesky_upper(hd)
    ref = O.gptq_quantize(w, u, 4, 256, False, 128)
    got = _sweep_factor(w, O.factor_blocks(u), 4, 256, False)
    np.testing.assert_allclose(got[1][:, 0], ref[1][:, 0], rtol=1e-12)  # read from W itself
    assert np.abs(got[1][:, 1] - ref[1][:, 1]).max() > 1e-6 * np.abs(ref[1][:, 1]).max()
