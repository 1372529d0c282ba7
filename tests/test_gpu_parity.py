"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle
on the same seeded inputs.

Tolerances (the workload's stated bars): H within 1e-5 relative Frobenius;
at most 0.1% of codes differ from the oracle's and only by +-1; scales
within 1e-5 relative and zero points equal (with the reading for groups
after a differing code in ``gptq_parity``); layer loss within 0.5%.  The
oracle takes its integer decisions in fp64, as the method defines them.
"""
import numpy as np
import pytest
import torch

from gptq_parity import check_layer, check_loss
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


def _upper_rel_fro(h_gpu, h_ref):
    iu = np.triu_indices(h_ref.shape[0])
    a, b = h_gpu[iu].astype(np.float64), h_ref[iu]
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _gpu_hessian(G, x_cpu, chunks=1, ldx_pad=0):
    n, d = x_cpu.shape
    if ldx_pad:
        buf = torch.zeros((n, d + ldx_pad), dtype=torch.bfloat16, device="cuda")
        buf[:, :d] = x_cpu.cuda()
        x = buf[:, :d]
    else:
        x = x_cpu.cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    bounds = np.linspace(0, n, chunks + 1).astype(int)
    for a, b in zip(bounds[:-1], bounds[1:]):
        G.gptq_hessian_accumulate(h, x[a:b])
    assert G.gptq_device_status() == 0
    return h.cpu().numpy()


def _tokens(d, n, seed):
    return synth.gen_tokens(synth.tiny_spec(8, d, n, seed=seed))


# ------------------------------------------------------------------ Hessian
@pytest.mark.parametrize("d,n", [(256, 2048), (136, 1000), (8, 5), (1024, 4096),
                                 (520, 777), (384, 64), (64, 1)])
def test_hessian_matches_oracle(G, d, n):
    x = _tokens(d, n, seed=d + n)
    h = _gpu_hessian(G, x)
    ref = O.hessian(x.float().numpy())
    assert _upper_rel_fro(h, ref) <= 1e-5
    assert np.all(np.tril(h, -1) == 0.0), "strict lower triangle must stay untouched"


def test_hessian_chunked_and_strided(G):
    x = _tokens(264, 3000, seed=3)
    ref = O.hessian(x.float().numpy())
    h1 = _gpu_hessian(G, x, chunks=3)
    h2 = _gpu_hessian(G, x, chunks=1, ldx_pad=40)
    assert _upper_rel_fro(h1, ref) <= 1e-5
    assert _upper_rel_fro(h2, ref) <= 1e-5


def test_hessian_empty_is_noop(G):
    h = torch.full((64, 64), 3.0, device="cuda")
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    G.gptq_hessian_accumulate(h, x)
    assert torch.all(h == 3.0)


# ------------------------------------------------------------ prepare (G)
def _oracle_h(d, n, seed):
    x = _tokens(d, n, seed)
    return O.hessian(x.float().numpy())


def _gpu_prepare(G, h64, damp):
    d = h64.shape[0]
    h = torch.from_numpy(np.triu(h64).astype(np.float32)).cuda()
    g = torch.empty((d, d), dtype=torch.float32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    cfg = G.make_config(block=128)
    ws = G.alloc_workspace(64, max(32, (d + 31) // 32 * 32), cfg)
    piv = G.gptq_prepare_hinv(h, damp, g, dead, ws)
    return g.cpu().numpy(), dead.cpu().numpy(), piv, h


@pytest.mark.parametrize("d", [256, 136, 520, 1024, 8])
def test_prepare_matches_oracle(G, d):
    h64 = _oracle_h(d, 4 * d + 100, seed=d)
    h32 = np.triu(h64).astype(np.float32).astype(np.float64)
    h32 = h32 + np.triu(h32, 1).T  # the exact fp32 matrix the GPU sees
    g, dead, piv, _ = _gpu_prepare(G, h64, 0.01)
    assert piv == -1 and not dead.any()
    hd, _ = O.dampen(h32, 0.01)
    u = O.hinv_cholesky_upper(hd)
    assert np.all(np.tril(g, -1) == 0)
    np.testing.assert_allclose(g, u, rtol=1e-5, atol=1e-6 * np.abs(u).max())
    res = g.astype(np.float64).T @ g.astype(np.float64) @ hd - np.eye(d)
    assert np.abs(res).max() < 1e-4


def test_prepare_detects_non_spd(G):
    d = 64
    h = np.eye(d) * 4.0
    h[5, 5] = -10.0
    with pytest.raises(G.GptqError, match="NOT_SPD") as ei:
        _gpu_prepare(G, h, 0.01)
    assert "bad_pivot=5" in str(ei.value)


def test_prepare_detects_nonfinite(G):
    h = np.eye(64)
    h[7, 7] = np.nan
    with pytest.raises(G.GptqError, match="NONFINITE"):
        _gpu_prepare(G, h, 0.01)


def test_prepare_dead_channel(G):
    d = 136
    x = _tokens(d, 900, seed=2).float().numpy()
    x[:, 17] = 0.0
    x[:, 100] = 0.0
    h64 = O.hessian(x)
    g, dead, piv, _ = _gpu_prepare(G, h64, 0.01)
    assert piv == -1
    assert np.nonzero(dead)[0].tolist() == [17, 100]
    hd, odead = O.dampen(h64.astype(np.float32).astype(np.float64), 0.01)
    assert np.nonzero(odead)[0].tolist() == [17, 100]
    u = O.hinv_cholesky_upper(hd)
    np.testing.assert_allclose(g, u, rtol=1e-5, atol=1e-6 * np.abs(u).max())


# -------------------------------------------------------- quantize (stage)
QCASES = [  # d_row, d_col, bits, group, sym, block
    (256, 256, 4, 0, False, 128),
    (64, 512, 3, 128, False, 128),
    (96, 512, 2, 32, False, 128),
    (64, 384, 4, 64, False, 64),
    (40, 320, 3, 0, True, 32),
    (64, 512, 4, 256, False, 128),
    (33, 160, 4, 32, False, 128),
    (70, 256, 2, 0, True, 64),
    (1, 32, 4, 0, False, 128),
    (130, 640, 4, 128, True, 128),
    (48, 256, 3, 64, False, 128),
    (64, 384, 8, 0, False, 128),      # INT8, per channel
    (96, 512, 8, 128, True, 128),     # INT8 symmetric, g = 128
    (40, 320, 5, 32, False, 32),      # an odd width: codes straddle words
    (64, 256, 6, 64, True, 64),
]


def _run_quantize(G, w, u32, bits, group, sym, block, dead=None):
    d_row, d_col = w.shape
    cfg = G.make_config(bits=bits, group_size=group, sym=sym, block=block)
    wt = torch.from_numpy(w.astype(np.float32)).cuda()
    gt = torch.from_numpy(np.ascontiguousarray(u32, dtype=np.float32)).cuda()
    dm = None if dead is None else torch.from_numpy(dead.astype(np.uint8)).cuda()
    qw, sc, ze = G.alloc_outputs(d_row, d_col, cfg)
    ws = G.alloc_workspace(d_row, d_col, cfg)
    G.gptq_quantize_layer(wt, gt, dm, cfg, qw, sc, ze, ws)
    torch.cuda.synchronize()
    assert G.gptq_device_status() == 0
    words = qw.cpu().numpy().view(np.uint32)
    codes = O.unpack_codes(words, bits, d_col)
    return codes, sc.cpu().numpy(), ze.cpu().numpy(), (qw, sc, ze, cfg, wt)


@pytest.mark.parametrize("case", QCASES, ids=lambda c: "x".join(map(str, c)))
def test_quantize_matches_oracle(G, case):
    d_row, d_col, bits, group, sym, block = case
    spec = synth.tiny_spec(d_row, d_col, 4 * d_col, seed=d_row + d_col + bits)
    w = synth.gen_weight(spec).numpy()
    h = O.hessian(synth.gen_tokens(spec).float().numpy())
    hd, _ = O.dampen(h, 0.01)
    u32 = O.hinv_cholesky_upper(hd).astype(np.float32)
    codes, sc, ze, _ = _run_quantize(G, w, u32, bits, group, sym, block)
    ref_codes, ref_s, ref_z, _, _ = O.gptq_quantize(
        w.astype(np.float64), u32.astype(np.float64), bits, group, sym, block)
    check_layer(codes, sc, ze, ref_codes, ref_s, ref_z, group)


_WIDE = {}


def _wide_factor(d_col):
    """The oracle's fp32-rounded factor for a wide test layer (computed once)."""
    if d_col not in _WIDE:
        spec = synth.tiny_spec(8, d_col, d_col + 512, seed=d_col)
        hd, _ = O.dampen(O.hessian(synth.gen_tokens(spec).float().numpy()), 0.01)
        _WIDE[d_col] = np.ascontiguousarray(O.hinv_cholesky_upper(hd), dtype=np.float32)
    return _WIDE[d_col]


@pytest.mark.parametrize("case", [(48, 8448, 4, 128, False, 128), (40, 8448, 3, 0, False, 64),
                                  (24, 8448, 4, 256, True, 128)],
                         ids=lambda c: "x".join(map(str, c)))
def test_quantize_wide_layers_lazy_windows(G, case):
    """Layers of 8192 columns or more sweep in lazy-update windows of blocks
    (the errors of a window reach the columns right of it at once, and the
    next window's first block takes them in its own step); here the last
    window is partial (66 or 132 blocks) and g = 256 spans two blocks."""
    d_row, d_col, bits, group, sym, block = case
    w = synth.gen_weight(synth.tiny_spec(d_row, d_col, 8, seed=d_row + bits)).numpy()
    u32 = _wide_factor(d_col)
    codes, sc, ze, _ = _run_quantize(G, w, u32, bits, group, sym, block)
    ref_codes, ref_s, ref_z, _, _ = O.gptq_quantize(
        w.astype(np.float64), u32.astype(np.float64), bits, group, sym, block)
    check_layer(codes, sc, ze, ref_codes, ref_s, ref_z, group)


@pytest.mark.parametrize("group", [0, 32, 128])
def test_quantize_degenerate_rows(G, group):
    """Rows the quantizer treats specially or that stress fp32 range: all zero
    (min = max, the +-1 range of the quantizer's rule), constant of either
    sign, one spike after zeros, a zero first half, and whole rows scaled by
    1e-4 and by 1e4, quantized with a real factor, against the plain fp64
    oracle.  (A group that holds nothing but the rounding residue of an
    earlier column has parameters fitted to that residue, which fp32 and
    fp64 leave at unrelated magnitudes; no row here makes one.)"""
    d_row, d_col = 40, 256
    spec = synth.tiny_spec(d_row, d_col, 4 * d_col, seed=900 + group)
    w = synth.gen_weight(spec).numpy().astype(np.float64)
    w[0] = 0.0
    w[1] = 0.03
    w[2] = -0.02
    w[3] = 0.0
    w[3, d_col - 5] = 0.5             # a spike in the last group: no group to its
                                      # right holds only its rounding residue
    w[4] *= 1e-4
    w[5] *= 1e4
    w[6, : d_col // 2] = 0.0          # a zero first half, then ordinary values
    w = w.astype(np.float32)
    h = O.hessian(synth.gen_tokens(spec).float().numpy())
    hd, _ = O.dampen(h, 0.01)
    u32 = np.ascontiguousarray(O.hinv_cholesky_upper(hd), dtype=np.float32)
    codes, sc, ze, _ = _run_quantize(G, w, u32, 4, group, False, 128)
    ref_codes, ref_s, ref_z, _, _ = O.gptq_quantize(
        w.astype(np.float64), u32.astype(np.float64), 4, group, False, 128)
    check_layer(codes, sc, ze, ref_codes, ref_s, ref_z, group)
    assert np.all(np.isfinite(sc)) and np.all(sc > 0)
    # an all-zero row stays at its zero point: nothing to propagate
    assert np.all(codes[0] == ze[0, 0])


def test_quantize_scaled_identity_is_rtn(G):
    """With G = c I nothing propagates: GPU output equals round-to-nearest."""
    spec = synth.tiny_spec(64, 256, 16)
    w = synth.gen_weight(spec).numpy()
    u32 = (np.eye(256) / np.sqrt(5.05)).astype(np.float32)
    codes, sc, ze, _ = _run_quantize(G, w, u32, 4, 64, False, 128)
    r = O.rtn(w.astype(np.float64), 4, 64, False)
    check_layer(codes, sc, ze, r["codes"], r["scales"], r["zeros"], 64)
    assert np.array_equal(codes, r["codes"]) and np.array_equal(ze, r["zeros"])


@pytest.mark.parametrize("bits,group", [(2, 0), (3, 0), (4, 0), (8, 0), (4, 64), (3, 128)])
def test_quantize_zero_point_ties(G, bits, group):
    """Every row (or group) has a symmetric range of bf16 values, max = -min,
    so -min/s lies exactly on a half-integer and the zero point is the
    half-to-even one.  With G = c I nothing propagates, so the parameters of
    every group come from these values."""
    rng = np.random.default_rng(100 + bits)
    w = torch.tensor(rng.standard_normal((64, 256)) * 0.02).to(torch.bfloat16).float().numpy()
    g = group or 256
    for c0 in range(0, 256, g):
        a = np.abs(w[:, c0:c0 + g]).max(axis=1)
        w[:, c0] = -a
        w[:, c0 + 1] = a
    u32 = (np.eye(256) / np.sqrt(5.05)).astype(np.float32)
    codes, sc, ze, _ = _run_quantize(G, w, u32, bits, group, False, 128)
    r = O.rtn(w.astype(np.float64), bits, group, False)
    assert np.array_equal(ze, r["zeros"])
    assert np.all(r["zeros"] == 2 ** (bits - 1))   # the tie (2^b - 1)/2 rounds up to even
    np.testing.assert_allclose(sc, r["scales"], rtol=1e-5)
    # A code whose exact quotient w/s = (2^b - 1) w / (xmax - xmin) is itself
    # a half-integer (-a / s = -(2^b - 1)/2 always is, and some bf16 values
    # are) is a tie decided by how s rounded (fp32 here, fp64 there): one
    # step either way.  Every other code is the oracle's.
    gcol = np.arange(256) // g
    span = (np.maximum(w.reshape(64, -1, g).max(2), 0) -
            np.minimum(w.reshape(64, -1, g).min(2), 0)).astype(np.float64)[:, gcol]
    exact = (2 ** bits - 1) * w.astype(np.float64) / span
    ties = np.abs(exact - np.floor(exact) - 0.5) < 1e-9
    assert ties[:, 0].all()
    assert np.abs(codes[ties] - r["codes"][ties]).max() <= 1
    np.testing.assert_array_equal(codes[~ties], r["codes"][~ties])


def test_quantize_dead_columns(G):
    spec = synth.tiny_spec(32, 128, 512, seed=9)
    w = synth.gen_weight(spec).numpy()
    x = synth.gen_tokens(spec).float().numpy()
    x[:, 3] = 0.0
    h = O.hessian(x)
    hd, dead = O.dampen(h, 0.01)
    u32 = O.hinv_cholesky_upper(hd).astype(np.float32)
    codes, sc, ze, _ = _run_quantize(G, w, u32, 4, 0, False, 128, dead=dead)
    ref_codes, ref_s, ref_z, _, _ = O.gptq_quantize(
        w.astype(np.float64), u32.astype(np.float64), 4, 0, False, 128, dead=dead)
    check_layer(codes, sc, ze, ref_codes, ref_s, ref_z, 0)
    assert np.array_equal(codes[:, 3], ze[:, 0].astype(np.int64))


# ------------------------------------------------------------- end to end
def _full_gpu(G, spec, x_cpu, w_cpu):
    d = spec.d_col
    cfg = G.make_config(bits=spec.bits, group_size=spec.group, sym=spec.sym,
                        block=spec.block, damp_rel=spec.damp)
    x = x_cpu.cuda()
    w = w_cpu.cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    g = torch.empty_like(h)
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(spec.d_row, d, cfg)
    qw, sc, ze = G.alloc_outputs(spec.d_row, d, cfg)
    G.gptq_hessian_accumulate(h, x)
    G.gptq_prepare_hinv(h, spec.damp, g, dead, ws)
    G.gptq_quantize_layer(w, g, dead, cfg, qw, sc, ze, ws)
    w_hat = torch.empty_like(w)
    loss = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat, ws=ws)
    assert G.gptq_device_status() == 0
    return dict(h=h, g=g, qw=qw, sc=sc, ze=ze, w_hat=w_hat, loss=loss, cfg=cfg)


def test_end_to_end_small_256(G):
    spec = synth.SMALL_256
    w = synth.gen_weight(spec)
    x = synth.gen_tokens(spec)
    r = _full_gpu(G, spec, x, w)
    xn, wn = x.float().numpy(), w.numpy().astype(np.float64)
    href = O.hessian(xn)
    assert _upper_rel_fro(r["h"].cpu().numpy(), href) <= 1e-5
    ref = O.gptq(wn, href, bits=4, group=0, sym=False, block=128, damp_rel=0.01)
    codes = O.unpack_codes(r["qw"].cpu().numpy().view(np.uint32), 4, 256)
    check_layer(codes, r["sc"].cpu().numpy(), r["ze"].cpu().numpy(), ref["codes"],
                ref["scales"], ref["zeros"], 0)
    ref_loss = O.layer_loss_direct(wn, ref["w_hat"], xn)
    check_loss(r["loss"], ref_loss)
    # the GPU loss check agrees with the oracle's loss of the GPU's own codes
    w_hat_ref = O.dequantize(codes, r["sc"].cpu().numpy().astype(np.float64),
                             r["ze"].cpu().numpy().astype(np.float64))
    np.testing.assert_allclose(r["w_hat"].cpu().numpy(), w_hat_ref, rtol=1e-6,
                               atol=1e-7)
    own = O.layer_loss_direct(wn, r["w_hat"].cpu().numpy(), xn)
    assert r["loss"] == pytest.approx(own, rel=1e-4)
    assert r["loss"] < O.layer_loss_direct(wn, O.rtn(wn, 4)["w_hat"], xn)


@pytest.mark.parametrize("bits,group,sym", [(3, 128, False), (2, 0, True),
                                            (4, 64, False), (8, 0, False),
                                            (8, 128, True)])
def test_end_to_end_variants(G, bits, group, sym):
    spec = synth.tiny_spec(192, 512, 3000, seed=bits * 7 + group).with_(
        bits=bits, group=group, sym=sym)
    w = synth.gen_weight(spec)
    x = synth.gen_tokens(spec)
    r = _full_gpu(G, spec, x, w)
    xn, wn = x.float().numpy(), w.numpy().astype(np.float64)
    ref = O.gptq(wn, O.hessian(xn), bits=bits, group=group, sym=sym,
                 block=128, damp_rel=0.01)
    codes = O.unpack_codes(r["qw"].cpu().numpy().view(np.uint32), bits, 512)
    check_layer(codes, r["sc"].cpu().numpy(), r["ze"].cpu().numpy(), ref["codes"],
                ref["scales"], ref["zeros"], group)
    ref_loss = O.layer_loss_direct(wn, ref["w_hat"], xn)
    check_loss(r["loss"], ref_loss)
