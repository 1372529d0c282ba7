"""GPU parity of the factor route (gptq_prepare_factor, then
gptq_quantize_layer_factor) against the fp64 oracle.

gptq_prepare_factor's F is compared element by element with the oracle's
``factor_blocks`` of its own U (H given to both as the same fp32 matrix),
including widths that are not a multiple of 128 (the factorization then
starts with the ragged block) and widths with lazy windows (d >= 8192).  The
layer that gptq_quantize_layer_factor writes from F is compared with the
oracle's sweep through U (``gptq_quantize``, the page's form), under the bars
of ``gptq_parity``: the same layer, reached with the sums regrouped.
"""
import numpy as np
import pytest
import torch

from gptq_parity import check_layer, check_layer_up_to_ties, check_loss, decision_margins
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_26_b200 import build, gptq
    build.build()
    gptq.load_library()
    return gptq


def _sym32(h64):
    """The fp32 matrix the GPU sees (upper triangle stored), as fp64."""
    h32 = np.triu(h64).astype(np.float32).astype(np.float64)
    return h32 + np.triu(h32, 1).T


def _gpu_prepare_factor(G, h64, damp):
    d = h64.shape[0]
    h = torch.from_numpy(np.triu(h64).astype(np.float32)).cuda()
    f = torch.empty((d, d), dtype=torch.float32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(64, max(32, (d + 31) // 32 * 32), G.make_config(block=128))
    piv = G.gptq_prepare_factor(h, damp, f, dead, ws)
    return f, dead.cpu().numpy(), piv


def _check_f(f_gpu, f_ref):
    assert np.all(np.tril(f_gpu, -1) == 0)
    np.testing.assert_allclose(f_gpu, f_ref, rtol=1e-5, atol=1e-6 * np.abs(f_ref).max())


@pytest.mark.parametrize("d", [256, 136, 520, 1000, 1024, 8, 64])
def test_prepare_factor_matches_oracle(G, d):
    spec = synth.tiny_spec(8, d, 4 * d + 100, seed=d)
    h64 = O.hessian(synth.gen_tokens(spec).float().numpy())
    f, dead, piv = _gpu_prepare_factor(G, h64, 0.01)
    assert piv == -1 and not dead.any()
    hd, _ = O.dampen(_sym32(h64), 0.01)
    _check_f(f.cpu().numpy(), O.factor_blocks(O.hinv_cholesky_upper(hd)))


@pytest.mark.parametrize("d", [8192, 8200])
def test_prepare_factor_wide_windows(G, d):
    """Lazy windows of 8 panels; d = 8200 also starts with a ragged block of
    8 columns and ends its last window part-full."""
    spec = synth.tiny_spec(8, d, d + 512, seed=d)
    h64 = O.hessian(synth.gen_tokens(spec).float().numpy())
    f, _, piv = _gpu_prepare_factor(G, h64, 0.01)
    assert piv == -1
    hd, _ = O.dampen(_sym32(h64), 0.01)
    u = O.hinv_cholesky_upper(hd)
    rows = np.array([0, 1, 127, 128, 4095, 4096, d - 129, d - 9, d - 8, d - 1])
    f_rows = f[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    ref = O.factor_rows(u, rows)
    np.testing.assert_allclose(f_rows, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def test_prepare_factor_errors_and_dead(G):
    h = np.eye(64) * 4.0
    h[5, 5] = -10.0
    with pytest.raises(G.GptqError, match="NOT_SPD") as ei:
        _gpu_prepare_factor(G, h, 0.01)
    assert "bad_pivot=5" in str(ei.value)
    h = np.eye(64)
    h[7, 7] = np.nan
    with pytest.raises(G.GptqError, match="NONFINITE"):
        _gpu_prepare_factor(G, h, 0.01)
    d = 296   # 2 blocks + a ragged 40, dead channels in two blocks
    x = synth.gen_tokens(synth.tiny_spec(8, d, 1200, seed=3)).float().numpy()
    x[:, [17, 200]] = 0.0
    h64 = O.hessian(x)
    f, dead, piv = _gpu_prepare_factor(G, h64, 0.01)
    assert piv == -1 and np.nonzero(dead)[0].tolist() == [17, 200]
    hd, _ = O.dampen(_sym32(h64), 0.01)
    _check_f(f.cpu().numpy(), O.factor_blocks(O.hinv_cholesky_upper(hd)))


# ------------------------------------------------------------- the sweep
def _run_factor(G, w, f32, bits, group, sym, dead=None):
    d_row, d_col = w.shape
    cfg = G.make_config(bits=bits, group_size=group, sym=sym, block=128)
    wt = torch.from_numpy(w.astype(np.float32)).cuda()
    ft = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32)).cuda()
    dm = None if dead is None else torch.from_numpy(dead.astype(np.uint8)).cuda()
    qw, sc, ze = G.alloc_outputs(d_row, d_col, cfg)
    ws = G.alloc_workspace(d_row, d_col, cfg)
    G.gptq_quantize_layer_factor(wt, ft, dm, cfg, qw, sc, ze, ws)
    torch.cuda.synchronize()
    assert G.gptq_device_status() == 0
    codes = O.unpack_codes(qw.cpu().numpy().view(np.uint32), bits, d_col)
    return codes, sc.cpu().numpy(), ze.cpu().numpy()


FCASES = [  # d_row, d_col, bits, group, sym
    (256, 256, 4, 0, False),
    (64, 512, 3, 128, False),
    (96, 512, 2, 32, False),
    (64, 384, 4, 64, False),
    (40, 320, 3, 0, True),       # ragged last block of 64
    (33, 160, 4, 32, False),     # ragged last block of 32, rows not a multiple of 32
    (1, 32, 4, 0, False),
    (130, 640, 4, 128, True),
    (64, 384, 8, 0, False),
    (40, 288, 5, 32, False),
    (96, 1024, 4, 128, False),
]


@pytest.mark.parametrize("case", FCASES, ids=lambda c: "x".join(map(str, c)))
def test_quantize_factor_matches_oracle(G, case):
    d_row, d_col, bits, group, sym = case
    spec = synth.tiny_spec(d_row, d_col, 4 * d_col, seed=d_row + d_col + bits)
    w = synth.gen_weight(spec).numpy()
    hd, _ = O.dampen(O.hessian(synth.gen_tokens(spec).float().numpy()), 0.01)
    u = O.hinv_cholesky_upper(hd)
    codes, sc, ze = _run_factor(G, w, O.factor_blocks(u), bits, group, sym)
    ref = O.gptq_quantize(w.astype(np.float64), u, bits, group, sym, 128)
    check_layer(codes, sc, ze, ref[0], ref[1], ref[2], group)


_WIDE = {}


def _wide(d_col):
    if d_col not in _WIDE:
        spec = synth.tiny_spec(8, d_col, d_col + 512, seed=d_col)
        hd, _ = O.dampen(O.hessian(synth.gen_tokens(spec).float().numpy()), 0.01)
        u = O.hinv_cholesky_upper(hd)
        _WIDE[d_col] = (u, O.factor_blocks(u))
    return _WIDE[d_col]


@pytest.mark.parametrize("case", [(48, 8448, 4, 128, False), (40, 8448, 3, 0, False),
                                  (24, 8448, 4, 32, True), (32, 8224, 4, 0, False)],
                         ids=lambda c: "x".join(map(str, c)))
def test_quantize_factor_wide_layers_lazy_windows(G, case):
    """Windows of 4 blocks: inside one, each block's errors reach the
    window's later blocks; the window's errors reach the rest at once.
    8224 columns end in a ragged block of 32 inside a part-full window.
    Layers of 24 to 48 rows: one row is 2-4% of the items, so a single tie
    at fp32 resolution (about one per million decisions on either route)
    would spend the pooled budget by itself.  Each row is therefore held to
    the oracle's exactly unless its first difference is such a tie (the
    24 x 8448 g = 32 layer has one 1.8e-6 s from it, the tightest of its
    202752 decisions, which the inverse route with round-to-nearest TF32
    splits also flips)."""
    d_row, d_col, bits, group, sym = case
    w = synth.gen_weight(synth.tiny_spec(d_row, d_col, 8, seed=d_row + bits)).numpy()
    u, f = _wide(d_col)
    codes, sc, ze = _run_factor(G, w, f, bits, group, sym)
    ref = O.gptq_quantize(w.astype(np.float64), u, bits, group, sym, 128)
    margins = decision_margins(ref[3], ref[4], np.diag(u), ref[1], group)
    check_layer_up_to_ties(codes, sc, ze, ref[0], ref[1], ref[2], margins, group)


def test_quantize_factor_dead_columns(G):
    """Dead columns read as zero weights: their errors, w^ - w, are zero."""
    spec = synth.tiny_spec(32, 384, 1536, seed=9)
    w = synth.gen_weight(spec).numpy()
    x = synth.gen_tokens(spec).float().numpy()
    x[:, [3, 130, 300]] = 0.0
    hd, dead = O.dampen(O.hessian(x), 0.01)
    u = O.hinv_cholesky_upper(hd)
    codes, sc, ze = _run_factor(G, w, O.factor_blocks(u), 4, 128, False, dead=dead)
    ref = O.gptq_quantize(w.astype(np.float64), u, 4, 128, False, 128, dead=dead)
    check_layer(codes, sc, ze, ref[0], ref[1], ref[2], 128)
    for c in (3, 130, 300):
        assert np.array_equal(codes[:, c], ze[:, c // 128].astype(np.int64))


@pytest.mark.parametrize("group", [0, 32, 128])
def test_quantize_factor_degenerate_rows(G, group):
    """The rows of the degenerate-row test of the other route: zero, constant,
    a spike in the last group, a zero half, and rows scaled by 1e-4 and 1e4."""
    d_row, d_col = 40, 256
    spec = synth.tiny_spec(d_row, d_col, 4 * d_col, seed=900 + group)
    w = synth.gen_weight(spec).numpy().astype(np.float64)
    w[0] = 0.0
    w[1] = 0.03
    w[2] = -0.02
    w[3] = 0.0
    w[3, d_col - 5] = 0.5
    w[4] *= 1e-4
    w[5] *= 1e4
    w[6, :128] = 0.0
    w = w.astype(np.float32)
    hd, _ = O.dampen(O.hessian(synth.gen_tokens(spec).float().numpy()), 0.01)
    u = O.hinv_cholesky_upper(hd)
    codes, sc, ze = _run_factor(G, w, O.factor_blocks(u), 4, group, False)
    ref = O.gptq_quantize(w.astype(np.float64), u, 4, group, False, 128)
    check_layer(codes, sc, ze, ref[0], ref[1], ref[2], group)
    assert np.all(np.isfinite(sc)) and np.all(sc > 0)
    assert np.all(codes[0] == ze[0, 0])


@pytest.mark.parametrize("block,group", [(64, 0), (32, 32), (128, 256)])
def test_quantize_factor_rejects_unsupported_configs(G, block, group):
    d_row, d_col = 8, 512
    cfg = G.make_config(bits=4, group_size=group, block=block)
    w = torch.zeros((d_row, d_col), device="cuda")
    f = torch.eye(d_col, device="cuda")
    qw, sc, ze = G.alloc_outputs(d_row, d_col, cfg)
    ws = G.alloc_workspace(d_row, d_col, cfg)
    with pytest.raises(G.GptqError, match="INVALID"):
        G.gptq_quantize_layer_factor(w, f, None, cfg, qw, sc, ze, ws)


# ------------------------------------------------------------ end to end
@pytest.mark.parametrize("bits,group,sym", [(4, 0, False), (3, 128, False), (4, 32, True)])
def test_factor_route_end_to_end(G, bits, group, sym):
    """Accumulate, prepare_factor, quantize_layer_factor and the loss check
    on one layer, against the whole oracle (its own H, U and sweep)."""
    spec = synth.tiny_spec(192, 640, 3000, seed=bits * 7 + group).with_(
        bits=bits, group=group, sym=sym)
    w_cpu, x_cpu = synth.gen_weight(spec), synth.gen_tokens(spec)
    d = spec.d_col
    cfg = G.make_config(bits=bits, group_size=group, sym=sym, block=128)
    x, w = x_cpu.cuda(), w_cpu.cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    f = torch.empty_like(h)
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(spec.d_row, d, cfg)
    qw, sc, ze = G.alloc_outputs(spec.d_row, d, cfg)
    G.gptq_hessian_accumulate(h, x)
    assert G.gptq_prepare_factor(h, spec.damp, f, dead, ws) == -1
    G.gptq_quantize_layer_factor(w, f, dead, cfg, qw, sc, ze, ws)
    loss = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, ws=ws)
    assert G.gptq_device_status() == 0
    xn, wn = x_cpu.float().numpy(), w_cpu.numpy().astype(np.float64)
    ref = O.gptq(wn, O.hessian(xn), bits=bits, group=group, sym=sym, block=128,
                 damp_rel=spec.damp)
    codes = O.unpack_codes(qw.cpu().numpy().view(np.uint32), bits, d)
    check_layer(codes, sc.cpu().numpy(), ze.cpu().numpy(), ref["codes"], ref["scales"],
                ref["zeros"], group)
    check_loss(loss, O.layer_loss_direct(wn, ref["w_hat"], xn))
