"""Pins for the CPU oracle: each test checks it against something other than
itself (hand-worked cases, closed forms, linear-algebra identities, an
independent unblocked OBS procedure, exhaustive search)."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import gptq_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rand_layer(rng, d_row, d_col, n, outliers=2):
    w = rng.standard_normal((d_row, d_col)) * 0.02
    x = rng.standard_normal((n, d_col))
    x[:, rng.permutation(d_col)[:outliers]] *= 20.0
    return w, x


# --------------------------------------------------------------- quantizer
@pytest.mark.parametrize("case", _load("quantizer_cases.json")["cases"],
                         ids=lambda c: c["id"])
def test_quantizer_hand_cases(case):
    x = np.array([case["x"]])
    s, z = O.quant_params(x, case["bits"], case["sym"])
    assert s[0] == pytest.approx(case["scale"], rel=1e-15)
    assert z[0] == case["zero"]
    q = O.quantize(x[0], s[0], z[0], case["bits"])
    assert q.tolist() == case["codes"]
    np.testing.assert_allclose(O.dequantize(q, s[0], z[0]), case["dequant"],
                               rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("case", _load("quantizer_cases.json")["zero_tie_cases"],
                         ids=lambda c: c["id"])
@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_zero_point_ties(case, dtype):
    """An exact tie in -xmin/s is rounded half to even, in either decision
    precision (the quotient is formed with s exact)."""
    _, z = O.quant_params(np.array([case["x"]]), case["bits"], False, dtype=dtype)
    assert z[0] == case["zero"]


@pytest.mark.parametrize("case", _load("quantizer_cases.json")["clip_cases"],
                         ids=lambda c: c["id"])
def test_quantizer_clip(case):
    q = O.quantize(np.array([case["x"]]), case["scale"], case["zero"],
                   case["bits"])
    assert q.tolist() == [case["code"]]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_quantizer_error_bound(bits, sym):
    """Inside the fitted range the rounding error is at most s/2."""
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((64, 128))
    s, z = O.quant_params(x, bits, sym)
    xh = np.zeros_like(x)
    for k in range(x.shape[1]):
        xh[:, k] = O.dequantize(O.quantize(x[:, k], s, z, bits), s, z)
    err = np.abs(x - xh)
    # both quantizers fit the range to the data, so nothing clips here
    bound = np.broadcast_to(s[:, None] / 2, x.shape) * (1 + 1e-12)
    assert np.all(err <= bound)


def test_quantizer_f32_decisions_match_f64_off_ties():
    """Taking the integer decision in float32 changes codes only at ties."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((256, 128)).astype(np.float32).astype(np.float64)
    s64, z64 = O.quant_params(x, 4, False, np.float64)
    s32, z32 = O.quant_params(x, 4, False, np.float32)
    np.testing.assert_allclose(s32, s64, rtol=1e-6)
    assert np.array_equal(z32, z64)
    q64 = np.stack([O.quantize(x[:, k], s64, z64, 4) for k in range(128)], 1)
    q32 = np.stack([O.quantize(x[:, k], s32, z32, 4, np.float32)
                    for k in range(128)], 1)
    assert np.mean(q64 != q32) < 1e-3
    assert np.max(np.abs(q64 - q32)) <= 1


# ----------------------------------------------------------------- packing
@pytest.mark.parametrize("case", _load("pack_cases.json")["cases"],
                         ids=lambda c: c["id"])
def test_pack_hand_cases(case):
    codes = np.array([case["codes"]])
    words = O.pack_codes(codes, case["bits"])
    assert words[0].tolist() == case["words"]
    back = O.unpack_codes(words, case["bits"], codes.shape[1])
    assert back.tolist() == codes.tolist()


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip_random(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, size=(7, 256))
    words = O.pack_codes(codes, bits)
    assert words.shape == (7, 256 * bits // 32)
    assert np.array_equal(O.unpack_codes(words, bits, 256), codes)


def test_pack_size_matches_bytes_per_param():
    """A 4-bit code costs 0.5 bytes per parameter (youleyou.com, section 一,
    memory per 1e9 parameters: int4 0.5G)."""
    codes = np.zeros((16, 1024), dtype=np.int64)
    assert O.pack_codes(codes, 4).nbytes == codes.size // 2


# ----------------------------------------------------------------- Hessian
def test_hessian_one_hot_tokens():
    """Tokens that are unit vectors give H = 2 * diag(token counts)."""
    d = 6
    ids = np.array([0, 2, 2, 5, 5, 5, 1])
    x = np.eye(d)[ids]
    h = O.hessian(x, chunk=3)
    np.testing.assert_array_equal(h, 2.0 * np.diag(np.bincount(ids, minlength=d)))


def test_hessian_loss_identity():
    """||dW X||_F^2 == 1/2 sum_r dW_r H dW_r^T fixes H = 2 X X^T (factor and
    transpose) independently of how H is computed."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((300, 24))
    dw = rng.standard_normal((5, 24))
    h = O.hessian(x, chunk=64)
    direct = O.layer_loss_direct(dw, np.zeros_like(dw), x)
    via_h = O.layer_loss_hessian(dw, np.zeros_like(dw), h)
    assert via_h == pytest.approx(direct, rel=1e-12)


def test_hessian_rows_one_hot_and_agreement():
    """hessian_rows: unit-vector tokens give 2 * counts on the diagonal and
    zeros elsewhere; on random input it returns exactly the requested rows
    of the full H (row order kept, repeats allowed)."""
    d = 7
    ids = np.array([3, 3, 0, 6, 6, 6, 2, 3])
    x = np.eye(d)[ids]
    r = O.hessian_rows(x, [3, 6, 1], chunk=3)
    want = 2.0 * np.diag(np.bincount(ids, minlength=d))[[3, 6, 1]]
    np.testing.assert_array_equal(r, want)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1000, 33))
    rows = [32, 0, 5, 5]
    np.testing.assert_allclose(O.hessian_rows(x, rows, chunk=128),
                               O.hessian(x, chunk=256)[rows], rtol=1e-12, atol=1e-9)


# ------------------------------------------------------ damping and factor
def test_dampen_closed_form_and_dead():
    h = np.diag([4.0, 0.0, 8.0])
    h[0, 2] = h[2, 0] = 1.0
    hd, dead = O.dampen(h, 0.03)
    lam = 0.03 * 4.0  # mean(diag) = 12/3
    assert dead.tolist() == [False, True, False]
    assert hd[0, 0] == pytest.approx(4.0 + lam)
    assert hd[1, 1] == 1.0
    assert hd[2, 2] == pytest.approx(8.0 + lam)
    assert hd[0, 2] == 1.0


@pytest.mark.parametrize("d", [1, 5, 33, 130])
def test_hinv_factor_defining_property(d):
    rng = np.random.default_rng(d)
    _, x = _rand_layer(rng, 1, d, 4 * d + 3)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    u = O.hinv_cholesky_upper(hd)
    assert np.allclose(np.tril(u, -1), 0.0)
    assert np.all(np.diag(u) > 0)
    np.testing.assert_allclose(u.T @ u @ hd, np.eye(d), atol=1e-9)
    u2 = O.hinv_cholesky_upper_reversed(hd)
    np.testing.assert_allclose(u2, u, rtol=1e-9, atol=1e-12 * np.abs(u).max())


def test_hinv_factor_scaled_identity():
    c, damp = 3.0, 0.01
    hd, _ = O.dampen(c * np.eye(7), damp)
    u = O.hinv_cholesky_upper(hd)
    np.testing.assert_allclose(u, np.eye(7) / np.sqrt(c * (1 + damp)),
                               rtol=1e-14)


def test_hinv_factor_trailing_block_is_schur_inverse():
    """U[q:,q:]^T U[q:,q:] is the inverse of H'[q:,q:]: row q of U is the OBS
    update direction for the remaining set."""
    rng = np.random.default_rng(5)
    _, x = _rand_layer(rng, 1, 12, 80)
    hd, _ = O.dampen(O.hessian(x), 0.01)
    u = O.hinv_cholesky_upper(hd)
    for q in range(12):
        uf = u[q:, q:]
        np.testing.assert_allclose(uf.T @ uf @ hd[q:, q:], np.eye(12 - q),
                                   atol=1e-9)


# -------------------------------------------------------------------- GPTQ
def test_gptq_hand_case():
    c = _load("gptq_hand_case.json")
    w, h = np.array(c["w"]), np.array(c["h"])
    r = O.gptq(w, h, bits=c["bits"], group=c["group"], sym=c["sym"],
               block=c["block"], damp_rel=c["damp_rel"])
    assert r["scales"][0, 0] == c["scale"] and r["zeros"][0, 0] == c["zero"]
    assert r["codes"][0].tolist() == c["gptq_codes"]
    np.testing.assert_allclose(r["w_hat"][0], c["gptq_dequant"], rtol=1e-15)
    assert O.layer_loss_hessian(w, r["w_hat"], h) == pytest.approx(
        c["gptq_loss_half_dWHdW"], rel=1e-12)
    rt = O.rtn(w, bits=c["bits"], group=c["group"], sym=c["sym"])
    assert rt["codes"][0].tolist() == c["rtn_codes"]
    assert O.layer_loss_hessian(w, rt["w_hat"], h) == pytest.approx(
        c["rtn_loss_half_dWHdW"], rel=1e-12)


@pytest.mark.parametrize("group", [0, 16, 64])
@pytest.mark.parametrize("sym", [False, True])
def test_gptq_scaled_identity_is_rtn(group, sym):
    """With H = cI the factor is diagonal, nothing propagates, and GPTQ is
    exactly round-to-nearest."""
    rng = np.random.default_rng(11)
    w = rng.standard_normal((40, 128)) * 0.02
    r = O.gptq(w, 5.0 * np.eye(128), bits=3, group=group, sym=sym, block=32)
    rt = O.rtn(w, bits=3, group=group, sym=sym)
    assert np.array_equal(r["codes"], rt["codes"])
    assert np.array_equal(r["scales"], rt["scales"])
    assert np.array_equal(r["zeros"], rt["zeros"])


@pytest.mark.parametrize("group,block", [(0, 128), (0, 32), (128, 128),
                                          (32, 128), (256, 128)])
def test_gptq_block1_equals_blocked(group, block):
    """Lazy batching only re-associates sums: block size 1 and the blocked
    run agree to 1e-10 (relative) and give the same codes."""
    rng = np.random.default_rng(7)
    w, x = _rand_layer(rng, 24, 512, 2048, outliers=6)
    h = O.hessian(x)
    a = O.gptq(w, h, bits=4, group=group, block=1)
    b = O.gptq(w, h, bits=4, group=group, block=block)
    assert np.array_equal(a["codes"], b["codes"])
    np.testing.assert_allclose(b["w_hat"], a["w_hat"], rtol=1e-10, atol=0)
    np.testing.assert_allclose(b["err"], a["err"], rtol=1e-10,
                               atol=1e-10 * np.abs(a["err"]).max())


@pytest.mark.parametrize("d", [2, 3, 5, 8])
@pytest.mark.parametrize("bits,sym,group", [(2, False, 0), (3, True, 0),
                                            (4, False, 0), (2, False, 2)])
def test_gptq_matches_unblocked_obs(d, bits, sym, group):
    """On tiny layers the Cholesky/blocked form equals OBS with the inverse
    Hessian of the remaining columns recomputed after every column."""
    if group and d % group:
        pytest.skip("group must divide d")
    rng = np.random.default_rng(100 + d)
    w, x = _rand_layer(rng, 8, d, 6 * d, outliers=1)
    h = O.hessian(x)
    r = O.gptq(w, h, bits=bits, group=group, sym=sym, block=2)
    codes, w_hat = O.obs_unblocked(w, r["h_damped"], bits, group, sym)
    assert np.array_equal(r["codes"], codes)
    np.testing.assert_allclose(r["w_hat"], w_hat, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("group", [0, 32])
def test_gptq_error_identity(group):
    """Algebraic consequence of the update rule: the total weight change is
    dW = E U, so 1/2 dW H' dW^T = 1/2 sum E^2 row by row, whatever codes
    were chosen.  A wrong row, sign or index in the propagation breaks it."""
    rng = np.random.default_rng(21)
    w, x = _rand_layer(rng, 16, 256, 1024, outliers=4)
    r = O.gptq(w, O.hessian(x), bits=3, group=group, block=64)
    dw = w - r["w_hat"]
    np.testing.assert_allclose(dw, r["err"] @ r["u"], rtol=1e-9,
                               atol=1e-12 * np.abs(dw).max())
    lhs = 0.5 * np.sum((dw @ r["h_damped"]) * dw, axis=1)
    np.testing.assert_allclose(lhs, 0.5 * np.sum(r["err"] ** 2, axis=1),
                               rtol=1e-8)


def test_gptq_loss_not_above_rtn_on_seeded_layers():
    """Section GPTQ's claim that error feedback beats plain rounding, checked
    on the seeded small layers (an empirical invariant, not a theorem)."""
    for seed in range(4):
        rng = np.random.default_rng(seed)
        w, x = _rand_layer(rng, 64, 128, 1024, outliers=3)
        h = O.hessian(x)
        for bits in (2, 3, 4):
            g = O.gptq(w, h, bits=bits)
            rt = O.rtn(w, bits=bits)
            assert (O.layer_loss_hessian(w, g["w_hat"], h)
                    <= O.layer_loss_hessian(w, rt["w_hat"], h))


def test_gptq_loss_bounded_by_exhaustive_search():
    """For d = 4 and 2-bit codes, enumerate all 4^4 code vectors per row with
    the same scale and zero: no code vector beats the minimum, and GPTQ sits
    between that minimum and RTN in total."""
    rng = np.random.default_rng(9)
    w, x = _rand_layer(rng, 12, 4, 32, outliers=1)
    h = O.hessian(x)
    g = O.gptq(w, h, bits=2, damp_rel=0.0)
    rt = O.rtn(w, bits=2)
    allq = np.array(list(itertools.product(range(4), repeat=4)), dtype=float)
    best = 0.0
    for r_ in range(w.shape[0]):
        s, z = g["scales"][r_, 0], g["zeros"][r_, 0]
        dw = w[r_][None, :] - s * (allq - z)
        best += float(np.min(0.5 * np.sum((dw @ h) * dw, axis=1)))
    lg = O.layer_loss_hessian(w, g["w_hat"], h)
    assert best <= lg + 1e-15
    assert lg <= O.layer_loss_hessian(w, rt["w_hat"], h)


def test_gptq_dead_channel():
    """An input channel that never fires contributes nothing to W X: its
    weights are zeroed and coded as the zero point."""
    rng = np.random.default_rng(4)
    w, x = _rand_layer(rng, 6, 16, 64, outliers=0)
    x[:, 5] = 0.0
    r = O.gptq(w, O.hessian(x), bits=4, group=8)
    assert r["dead"].tolist() == [k == 5 for k in range(16)]
    assert np.all(r["w_hat"][:, 5] == 0.0)
    assert np.array_equal(r["codes"][:, 5], r["zeros"][:, 0].astype(int))


def test_small_256_layer_end_to_end():
    """The 256x256, 2048-token layer: direct and Hessian losses agree, GPTQ
    beats RTN, and the blocked run equals block size 1."""
    from post_weight_quantization_26_b200 import synth
    spec = synth.SMALL_256
    w = synth.gen_weight(spec).numpy()
    x = synth.gen_tokens(spec).float().numpy()
    h = O.hessian(x)
    r = O.gptq(w, h, bits=4, group=0, block=128, damp_rel=0.01)
    ld = O.layer_loss_direct(w, r["w_hat"], x)
    assert O.layer_loss_hessian(w, r["w_hat"], h) == pytest.approx(ld, rel=1e-10)
    assert ld < O.layer_loss_direct(w, O.rtn(w, 4)["w_hat"], x)
    r1 = O.gptq(w, h, bits=4, group=0, block=1, damp_rel=0.01)
    assert np.array_equal(r1["codes"], r["codes"])


def test_dequantized_matmul_closed_forms():
    """Codes equal to the zero point give Y = 0; unit scales, zero points 0
    and all-ones codes give the row sums of X; a single code 3 at (r, k)
    with scale 0.5 gives Y[:, r] = 1.5 X[:, k].  Grouped parameters pick
    the right group (the second group's scale doubles its columns)."""
    rng = np.random.default_rng(9)
    bits, rows, cols = 4, 3, 64
    x = rng.standard_normal((2, cols))
    z = np.full((rows, 1), 5.0)
    y0 = O.dequantized_matmul(O.pack_codes(np.full((rows, cols), 5), bits), np.ones((rows, 1)),
                              z, x, bits, 0)
    assert np.all(y0 == 0.0)
    y1 = O.dequantized_matmul(O.pack_codes(np.ones((rows, cols), int), bits), np.ones((rows, 1)),
                              np.zeros((rows, 1)), x, bits, 0)
    np.testing.assert_allclose(y1, np.repeat(x.sum(1, keepdims=True), rows, 1), rtol=1e-12)
    codes = np.zeros((rows, cols), int)
    codes[1, 17] = 3
    y2 = O.dequantized_matmul(O.pack_codes(codes, bits), np.full((rows, 1), 0.5),
                              np.zeros((rows, 1)), x, bits, 0)
    np.testing.assert_allclose(y2[:, 1], 1.5 * x[:, 17], rtol=1e-12)
    assert np.all(y2[:, [0, 2]] == 0.0)
    s = np.ones((rows, 2)); s[:, 1] = 2.0
    y3 = O.dequantized_matmul(O.pack_codes(np.ones((rows, cols), int), bits), s,
                              np.zeros((rows, 2)), x, bits, 32)
    want = x[:, :32].sum(1) + 2.0 * x[:, 32:].sum(1)
    np.testing.assert_allclose(y3, np.repeat(want[:, None], rows, 1), rtol=1e-12)
