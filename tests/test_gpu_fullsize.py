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
* the 65B-scale down projection (H of 22016^2 from 131072 tokens, 1.3e14
  fp64 flops on the host, longer than a test can take): sampled rows of H
  from the tokens, and properties that hold at any size:
  - U^T U H' v = v for the returned G on random vectors v;
  - on sampled rows of W, that each code is the rounding GPTQ prescribes.
    For every row the updates make W - W^ = e U, where e_q is the scaled
    error of column q; so e is recovered from the output by one triangular
    solve, the value column q held when it was quantized is W^_q + e_q U_qq,
    and its code must be that value's nearest grid point (or the clip
    bound), with the group's scale and zero the min-max parameters of the
    values the group held at its first column;
  - the sampled rows' loss is below round-to-nearest's.
"""
import numpy as np
import pytest
import torch
from scipy.linalg import solve_triangular

from gptq_parity import CODE_FRAC, check_layer, check_loss
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


def _gpu_quantize(G, spec, w_host, g, dead, ws, h):
    cfg = _cfg(G, spec)
    w = w_host.cuda()
    qw, sc, ze = G.alloc_outputs(spec.d_row, spec.d_col, cfg)
    G.gptq_quantize_layer(w, g, dead, cfg, qw, sc, ze, ws)
    w_hat = torch.empty_like(w)
    loss = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat, ws=ws)
    assert G.gptq_device_status() == 0
    return dict(qw=qw, sc=sc, ze=ze, w_hat=w_hat, loss=loss)


def _h_row(h_dev, i):
    """Row i of the symmetric H from the stored upper triangle."""
    return torch.cat([h_dev[:i, i], h_dev[i, i:]]).double().cpu().numpy()


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


def _check_h_rows(h_dev, x_host, spec, seed):
    rng = np.random.default_rng(seed)
    d = spec.d_col
    out_ch = synth.outlier_channels(spec)
    rows = [0, d - 1, int(out_ch[0])] + rng.choice(d, 3, replace=False).tolist()
    ref = O.hessian_rows(_Tokens(x_host), rows)
    for k, i in enumerate(rows):
        got = _h_row(h_dev, i)
        rel = np.linalg.norm(got - ref[k]) / np.linalg.norm(ref[k])
        assert rel <= 1e-5, f"H row {i}: rel {rel:.2e}"


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


def _check_rows_property(spec, w_host, out, gu, hu, seed, n_rows=24):
    """Codes, scales and zeros of sampled rows against the rounding GPTQ
    prescribes given the returned U; and the rows' loss against RTN's."""
    d_row, d = spec.d_row, spec.d_col
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, d_row - 1], rng.choice(d_row, n_rows, replace=False)]))
    maxq = 2 ** spec.bits - 1
    codes = O.unpack_codes(out["qw"][rows].cpu().numpy().view(np.uint32), spec.bits, d)
    s = out["sc"][rows].double().cpu().numpy()
    z = out["ze"][rows].double().cpu().numpy()
    w_hat = out["w_hat"][rows].double().cpu().numpy()
    w0 = w_host[rows].double().numpy()
    assert codes.min() >= 0 and codes.max() <= maxq
    g = spec.group or d
    col_group = np.arange(d) // g
    # the check kernel's W^ is s (q - z)
    np.testing.assert_allclose(w_hat, s[:, col_group] * (codes - z[:, col_group]),
                               rtol=1e-6, atol=1e-12)
    u = gu.astype(np.float64)
    e = solve_triangular(u, (w0 - w_hat).T, lower=False, trans="T").T
    w_at_q = w_hat + e * np.diag(u)[None, :]
    # scales and zeros: per-channel from the original rows, group-wise from
    # the values the group held when its first column was reached
    ns, nz = [], []
    for k0 in range(0, d, g):
        if spec.group:
            wg = w0[:, k0:k0 + g] - e[:, :k0] @ u[:k0, k0:k0 + g]
        else:
            wg = w0
        si, zi = O.quant_params(wg, spec.bits, spec.sym)
        ns.append(si)
        nz.append(zi)
    ref_s, ref_z = np.stack(ns, 1), np.stack(nz, 1)
    np.testing.assert_allclose(s, ref_s, rtol=1e-5)
    zdiff = np.abs(z - ref_z)
    assert zdiff.max() <= 1 and np.mean(zdiff != 0) <= CODE_FRAC
    r = np.clip(w_at_q / s[:, col_group] + z[:, col_group], 0, maxq)
    m = np.abs(r - codes)
    assert m.max() <= 1.5, f"a code is off by {m.max():.2f} grid steps"
    frac = float(np.mean(m > 0.5 + 1e-3))
    assert frac <= CODE_FRAC, f"{frac:.2e} of codes are not the prescribed rounding"
    # the rows' loss (1/2 dW H dW^T, undamped H) is below round-to-nearest's
    rw = O.rtn(w0, spec.bits, spec.group, spec.sym)["w_hat"]
    dq = (w0 - w_hat).T
    dr = (w0 - rw).T
    lq = 0.5 * float(np.sum(_sym_upper_matmul(hu, dq) * dq))
    lr = 0.5 * float(np.sum(_sym_upper_matmul(hu, dr) * dr))
    assert lq < lr, f"GPTQ rows' loss {lq:.4e} not below RTN's {lr:.4e}"
    return lq, lr


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
    oracle's H) within the loss bar."""
    rows = _sample_rows(spec.d_row, seed)
    w0 = w_host[torch.as_tensor(rows)].double().numpy()
    codes, scales, zeros, w_hat, _ = O.gptq_quantize(
        w0, u, spec.bits, spec.group, spec.sym, spec.block, dead=dead)
    res = check_layer(_codes(out, spec, rows), _rows(out, "sc", rows), _rows(out, "ze", rows),
                      codes, scales, zeros, spec.group)
    loss_ref = O.layer_loss_hessian(w0, w_hat, h_ref)
    loss_gpu = O.layer_loss_hessian(w0, _rows(out, "w_hat", rows), h_ref)
    check_loss(loss_gpu, loss_ref)
    return res


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ------------------------------------- q_proj and down_proj: the whole oracle
@pytest.mark.parametrize("spec", [synth.Q_PROJ_7B, synth.DOWN_PROJ_7B], ids=lambda s: s.name)
def test_full_size_against_whole_oracle(G, spec):
    x, w = _inputs(spec)
    h = _gpu_hessian(G, x)
    g, dead, ws = _gpu_prepare(G, h, spec, spec.d_row)
    out = _gpu_quantize(G, spec, w, g, dead, ws, h)
    _check_g_property(h, g, spec.damp, seed=1)
    h_ref = O.hessian(_Tokens(x))
    del x
    _check_h_whole(h, h_ref)
    del h, g, dead, ws
    _free()
    ref = O.gptq(w.double().numpy(), h_ref, bits=spec.bits, group=spec.group,
                 sym=spec.sym, block=spec.block, damp_rel=spec.damp)
    check_layer(_codes(out, spec), out["sc"].cpu().numpy(), out["ze"].cpu().numpy(),
                ref["codes"], ref["scales"], ref["zeros"], spec.group)
    loss_ref = O.layer_loss_hessian(w.double().numpy(), ref["w_hat"], h_ref)
    check_loss(out["loss"], loss_ref)
    del out
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


def _run_property_layer(G, spec, x, w, seed, h=None, g=None, dead=None, ws=None):
    if h is None:
        h = _gpu_hessian(G, x)
        _check_h_rows(h, x, spec, seed)
        g, dead, ws = _gpu_prepare(G, h, spec, spec.d_row)
    hu, gu = _check_g_property(h, g, spec.damp, seed)
    out = _gpu_quantize(G, spec, w, g, dead, ws, h)
    assert np.isfinite(out["loss"]) and out["loss"] > 0
    _check_rows_property(spec, w, out, gu, hu, seed)
    return h, g, dead, ws


def test_mlp_65b_down_proj_4_and_3_bits(G):
    """The 65B down projection (H of 22016^2): one accumulate and prepare,
    then the layer at 4 and at 3 bits; sampled H rows from the tokens and the
    properties above."""
    spec4 = [s for s, i in synth.mlp_65b(4) if i == 1][0]
    x, w = _inputs(spec4)
    h, g, dead, ws = _run_property_layer(G, spec4, x, w, seed=44)
    del x
    spec3 = [s for s, i in synth.mlp_65b(3) if i == 1][0]
    _run_property_layer(G, spec3, None, w, seed=43, h=h, g=g, dead=dead, ws=ws)
    del h, g, dead, ws
    _free()
