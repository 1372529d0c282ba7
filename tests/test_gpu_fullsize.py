"""Parity at the workloads' full layer sizes, in the launch configuration the
benchmark times: one accumulate call over all calibration tokens, then
prepare, then quantize (and the dequantize/loss check).  The oracle is the
plain fp64 one (integer decisions in fp64); the bars are those of
``gptq_parity``.

* q_proj 4096 x 4096 (262144 tokens) and down_proj 4096 x 11008 (g = 128):
  the whole oracle runs on the same seeded inputs, and H, every code, scale
  and zero point, and the layer loss are compared.
* the LLaMA-7B-shaped decoder block (7 layers, 4 Hessians) at 3 and 4 bits,
  and the 65B-scale gate/up projections (H of 8192^2) at 4 and 3 bits: the
  oracle forms each input's H from the tokens and its factor, then
  quantizes sampled rows (the first, the last and random ones; rows are
  independent given the factor), which are compared code by code with their
  loss; every H is compared whole.
* the 65B-scale down projection (H of 22016^2 from 131072 tokens, the
  default benchmark layer) at 4 and 3 bits: the same, with the oracle's H
  (1.3e14 fp64 flops on the host) and its factor of that size.
Every returned G is also checked by U^T U H' v = v on random vectors v.
The q_proj, down_proj and 65B down projection layers are also quantized
through the factor route (gptq_prepare_factor, gptq_quantize_layer_factor)
and held to the same oracle layer, and rows of that route's F to the
oracle's.
"""
import numpy as np
import pytest
import torch

from gptq_parity import check_layer, check_loss
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth

pytestmark = pytest.mark.gpu

G_RESID = 1e-5     # ||U^T U H' v - v|| / ||v|| (fp32 rounding of U alone gives ~1e-7)


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_26_b200 import build, gptq
    build.build()
    gptq.load_library()
    return gptq


class _Tokens:
    """Token-major bf16 host tensor seen by the oracle as fp32 numpy slices."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, sl):
        return self.t[sl].float().numpy()


def _inputs(spec):
    x = torch.empty((spec.n_tokens, spec.d_col), dtype=torch.bfloat16)
    synth.gen_tokens(spec, out=x)
    return x, synth.gen_weight(spec)


def _cfg(G, spec):
    return G.make_config(bits=spec.bits, group_size=spec.group, sym=spec.sym,
                         block=spec.block, damp_rel=spec.damp)


def _gpu_hessian(G, x_host):
    d = x_host.shape[1]
    x = x_host.cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(h, x)
    del x
    assert G.gptq_device_status() == 0
    return h


def _gpu_prepare(G, h, spec, d_row_max):
    d = spec.d_col
    g = torch.empty_like(h)
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(d_row_max, d, _cfg(G, spec))
    piv = G.gptq_prepare_hinv(h, spec.damp, g, dead, ws)
    assert piv == -1
    assert not bool(dead.any())
    return g, dead, ws


def _gpu_prepare_factor(G, h, spec, ws):
    f = torch.empty_like(h)
    dead = torch.empty(spec.d_col, dtype=torch.uint8, device="cuda")
    assert G.gptq_prepare_factor(h, spec.damp, f, dead, ws) == -1
    assert not bool(dead.any())
    return f, dead


def _gpu_quantize(G, spec, w_host, g, dead, ws, h, factor=False):
    cfg = _cfg(G, spec)
    w = w_host.cuda()
    qw, sc, ze = G.alloc_outputs(spec.d_row, spec.d_col, cfg)
    quantize = G.gptq_quantize_layer_factor if factor else G.gptq_quantize_layer
    quantize(w, g, dead, cfg, qw, sc, ze, ws)
    w_hat = torch.empty_like(w)
    loss = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat, ws=ws)
    assert G.gptq_device_status() == 0
    return dict(qw=qw, sc=sc, ze=ze, w_hat=w_hat, loss=loss)


def _sym_upper_matmul(hu, v, chunk=2048):
    """H v for H symmetric, given its upper triangle hu (strict lower zero);
    v is [d] or [d][k]; fp64 accumulation over fp32 storage."""
    d = hu.shape[0]
    out = np.zeros(v.shape, dtype=np.float64)
    for r0 in range(0, d, chunk):
        b = hu[r0:r0 + chunk].astype(np.float64)
        out[r0:r0 + chunk] += b @ v
        out += b.T @ v[r0:r0 + chunk]
        idx = np.arange(r0, min(d, r0 + chunk))
        out[idx] -= (b[np.arange(idx.size), idx] * v[idx].T).T
    return out


def _upper_matmul(gu, v, transpose=False, chunk=2048):
    d = gu.shape[0]
    out = np.zeros(v.shape, dtype=np.float64)
    for r0 in range(0, d, chunk):
        b = gu[r0:r0 + chunk].astype(np.float64)
        if transpose:
            out += b.T @ v[r0:r0 + chunk]
        else:
            out[r0:r0 + chunk] = b @ v
    return out


def _check_g_property(h_dev, g_dev, damp, seed):
    d = h_dev.shape[0]
    assert float(torch.tril(g_dev, -1).abs().max()) == 0.0
    assert bool((torch.diagonal(g_dev) > 0).all())
    hu = h_dev.cpu().numpy()
    gu = g_dev.cpu().numpy()
    lam = damp * float(np.mean(np.diag(hu).astype(np.float64)))
    v = np.random.default_rng(seed).standard_normal((d, 2))
    hv = _sym_upper_matmul(hu, v) + lam * v
    r = _upper_matmul(gu, _upper_matmul(gu, hv), transpose=True) - v
    rel = np.linalg.norm(r, axis=0) / np.linalg.norm(v, axis=0)
    assert rel.max() <= G_RESID, f"U^T U H' v - v: rel {rel.max():.2e}"
    return hu, gu


def _check_f_property(h_dev, f_dev, damp, seed, block=128):
    """F from gptq_prepare_factor holds G_bb on its diagonal blocks and
    V_ab G_bb right of them (H' = V V^T, G = V^-1).  G is applied through F
    without forming it, as the sweep does, and G H' G^T v = v is checked on
    random vectors v (the check of G above, in the form G H' G^T = I):
      x = G^T v:  x_b = F_bb^T v_b - F[:b0, b]^T x[:b0]  (block columns, forward)
      z = G y:    w_b = y_b - F[b, >b] w[>b],  z_b = F_bb w_b  (block rows, backward)"""
    d = h_dev.shape[0]
    assert float(torch.tril(f_dev, -1).abs().max()) == 0.0
    assert bool((torch.diagonal(f_dev) > 0).all())
    hu = h_dev.cpu().numpy()
    fu = f_dev.cpu().numpy()
    lam = damp * float(np.mean(np.diag(hu).astype(np.float64)))
    v = np.random.default_rng(seed).standard_normal((d, 2))
    starts = list(range(0, d, block))
    x = np.zeros_like(v)
    for b0 in starts:
        b1 = min(b0 + block, d)
        x[b0:b1] = (fu[b0:b1, b0:b1].astype(np.float64).T @ v[b0:b1]
                    - fu[:b0, b0:b1].astype(np.float64).T @ x[:b0])
    y = _sym_upper_matmul(hu, x) + lam * x
    del hu
    w = np.zeros_like(v)
    z = np.zeros_like(v)
    for b0 in reversed(starts):
        b1 = min(b0 + block, d)
        w[b0:b1] = y[b0:b1] - fu[b0:b1, b1:].astype(np.float64) @ w[b1:]
        z[b0:b1] = fu[b0:b1, b0:b1].astype(np.float64) @ w[b0:b1]
    rel = np.linalg.norm(z - v, axis=0) / np.linalg.norm(v, axis=0)
    assert rel.max() <= G_RESID, f"G H' G^T v - v through F: rel {rel.max():.2e}"


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _check_h_whole(h_dev, h_ref):
    hu = h_dev.cpu().numpy()
    iu = np.triu_indices(h_ref.shape[0])
    rel = np.linalg.norm(hu[iu] - h_ref[iu]) / np.linalg.norm(h_ref[iu])
    assert rel <= 1e-5, f"H rel Frobenius {rel:.2e}"
    return hu


def _codes(out, spec, rows=None):
    qw = out["qw"] if rows is None else out["qw"][torch.as_tensor(rows, device=out["qw"].device)]
    return O.unpack_codes(qw.cpu().numpy().view(np.uint32), spec.bits, spec.d_col)


def _rows(out, key, rows):
    t = out[key][torch.as_tensor(rows, device=out[key].device)]
    return t.double().cpu().numpy()


def _sample_rows(d_row, seed, n=48):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, d_row - 1], rng.choice(d_row, n, replace=False)]))


def _check_sampled_rows(spec, w_host, out, u, dead, h_ref, seed):
    """The oracle quantizes the sampled rows with its own factor; they are
    compared with the GPU's rows code by code, and their loss (through the
    oracle's H) within the loss bar.  `out` may be a list of GPU layers (the
    two routes), all checked against the one oracle sweep."""
    rows = _sample_rows(spec.d_row, seed)
    w0 = w_host[torch.as_tensor(rows)].double().numpy()
    codes, scales, zeros, w_hat, _ = O.gptq_quantize(
        w0, u, spec.bits, spec.group, spec.sym, spec.block, dead=dead)
    loss_ref = O.layer_loss_hessian(w0, w_hat, h_ref)
    res = []
    for o in (out if isinstance(out, list) else [out]):
        res.append(check_layer(_codes(o, spec, rows), _rows(o, "sc", rows), _rows(o, "ze", rows),
                               codes, scales, zeros, spec.group))
        check_loss(O.layer_loss_hessian(w0, _rows(o, "w_hat", rows), h_ref), loss_ref)
    return res


def _check_f_rows(f_dev, u, seed, n=24):
    """Sampled rows of the GPU's F (gptq_prepare_factor) against the
    oracle's rows of F from its own U."""
    d = u.shape[0]
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, 127, 128, d - 1], rng.choice(d, n, replace=False)]))
    got = f_dev[torch.as_tensor(rows, device=f_dev.device)].double().cpu().numpy()
    ref = O.factor_rows(u, rows)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


# ------------------------------------- q_proj and down_proj: the whole oracle
@pytest.mark.parametrize("spec", [synth.Q_PROJ_7B, synth.DOWN_PROJ_7B], ids=lambda s: s.name)
def test_full_size_against_whole_oracle(G, spec):
    """Both routes (G, and F from gptq_prepare_factor) against the whole
    oracle; F itself against the oracle's F of its own U."""
    x, w = _inputs(spec)
    h = _gpu_hessian(G, x)
    g, dead, ws = _gpu_prepare(G, h, spec, spec.d_row)
    out = _gpu_quantize(G, spec, w, g, dead, ws, h)
    _check_g_property(h, g, spec.damp, seed=1)
    del g
    f, dead_f = _gpu_prepare_factor(G, h, spec, ws)
    out_f = _gpu_quantize(G, spec, w, f, dead_f, ws, h, factor=True)
    h_ref = O.hessian(_Tokens(x))
    del x
    _check_h_whole(h, h_ref)
    del h, dead, dead_f, ws
    _free()
    ref = O.gptq(w.double().numpy(), h_ref, bits=spec.bits, group=spec.group,
                 sym=spec.sym, block=spec.block, damp_rel=spec.damp)
    loss_ref = O.layer_loss_hessian(w.double().numpy(), ref["w_hat"], h_ref)
    for o in (out, out_f):
        check_layer(_codes(o, spec), o["sc"].cpu().numpy(), o["ze"].cpu().numpy(),
                    ref["codes"], ref["scales"], ref["zeros"], spec.group)
        check_loss(o["loss"], loss_ref)
    _check_f_rows(f, ref["u"], seed=2)
    del out, out_f, f
    _free()


# ----------------------------------------------- the decoder block, 3 and 4 bits
def test_decoder_block_all_layers_3_and_4_bits(G):
    """All seven layers of the block, at 3 and 4 bits: one accumulate and one
    prepare per input (q/k/v share one, gate/up another), every layer
    quantized with its input's G; sampled rows of every layer against the
    oracle, which forms each input's H from the tokens."""
    by_bits = {b: synth.decoder_block_7b(b) for b in (3, 4)}
    inputs = sorted({xin for _, xin in by_bits[4]})
    for xin in inputs:
        layers = {b: [s for s, i in by_bits[b] if i == xin] for b in (3, 4)}
        s0 = layers[4][0]
        x, _ = _inputs(s0)
        h = _gpu_hessian(G, x)
        g, dead, ws = _gpu_prepare(G, h, s0, max(s.d_row for s in layers[4]))
        _check_g_property(h, g, s0.damp, seed=20 + xin)
        h_ref = O.hessian(_Tokens(x))
        del x
        _check_h_whole(h, h_ref)
        hd, dead_ref = O.dampen(h_ref, s0.damp)
        u = O.hinv_cholesky_upper(hd)
        del hd
        for b in (3, 4):
            for k, spec in enumerate(layers[b]):
                w = synth.gen_weight(spec)
                out = _gpu_quantize(G, spec, w, g, dead, ws, h)
                assert np.isfinite(out["loss"]) and out["loss"] > 0
                _check_sampled_rows(spec, w, out, u, dead_ref, h_ref, seed=100 * b + 10 * xin + k)
                del out
        del h, g, dead, ws, h_ref, u
        _free()


# -------------------------------------------------------- the 65B-scale MLP
def test_mlp_65b_gate_up_against_oracle(G):
    """gate and up (22016 x 8192) share one input: one H of 8192^2 from
    131072 tokens; both layers at 4 and 3 bits, sampled rows against the
    oracle, H whole."""
    specs = {b: [s for s, i in synth.mlp_65b(b) if i == 0] for b in (4, 3)}
    s0 = specs[4][0]
    x, _ = _inputs(s0)
    h = _gpu_hessian(G, x)
    g, dead, ws = _gpu_prepare(G, h, s0, s0.d_row)
    _check_g_property(h, g, s0.damp, seed=30)
    h_ref = O.hessian(_Tokens(x))
    del x
    _check_h_whole(h, h_ref)
    hd, dead_ref = O.dampen(h_ref, s0.damp)
    u = O.hinv_cholesky_upper(hd)
    del hd
    for b in (4, 3):
        for k, spec in enumerate(specs[b]):
            w = synth.gen_weight(spec)
            out = _gpu_quantize(G, spec, w, g, dead, ws, h)
            _check_sampled_rows(spec, w, out, u, dead_ref, h_ref, seed=300 + 10 * b + k)
            del out
    del h, g, dead, ws
    _free()


def test_mlp_65b_down_proj_4_and_3_bits(G):
    """The 65B down projection (H of 22016^2, the default benchmark layer):
    one accumulate on the GPU, both prepares (G and F), then the layer at 4
    and at 3 bits through each.  The oracle forms its own H from the tokens
    (checked whole against the GPU's), its own factor, rows of F from it,
    and quantizes sampled rows of both widths, checked against both
    routes."""
    spec4 = [s for s, i in synth.mlp_65b(4) if i == 1][0]
    spec3 = [s for s, i in synth.mlp_65b(3) if i == 1][0]
    x, w = _inputs(spec4)
    h = _gpu_hessian(G, x)
    g, dead, ws = _gpu_prepare(G, h, spec4, spec4.d_row)
    _check_g_property(h, g, spec4.damp, seed=44)
    outs = {spec.bits: [_gpu_quantize(G, spec, w, g, dead, ws, h)] for spec in (spec4, spec3)}
    del g
    f, dead_f = _gpu_prepare_factor(G, h, spec4, ws)
    _check_f_property(h, f, spec4.damp, seed=46)
    for spec in (spec4, spec3):
        outs[spec.bits].append(_gpu_quantize(G, spec, w, f, dead_f, ws, h, factor=True))
    h_ref = O.hessian(_Tokens(x))
    del x
    _check_h_whole(h, h_ref)
    del h, dead, dead_f, ws
    _free()
    hd, dead_ref = O.dampen(h_ref, spec4.damp)
    u = O.hinv_cholesky_upper(hd)
    del hd
    _check_f_rows(f, u, seed=45)
    del f
    for spec in (spec4, spec3):
        _check_sampled_rows(spec, w, outs[spec.bits], u, dead_ref, h_ref, seed=440 + spec.bits)
    del outs, u, h_ref
    _free()