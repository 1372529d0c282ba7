"""GPU parity of the dequant-fused matmul (gptq_w4a16_matmul, through the C
ABI) against the oracle's fp64 ``dequantized_matmul`` on the same seeded
packed layers and activations.

Tolerance, from the arithmetic: the kernel's products (q - z) x are exact in
fp32 and only additions round.  Each output is a chain of at most
``8 ceil(n_chunks / 8)`` mma accumulations (128-column chunks split over 8
warps), one scale multiply per region, and an 8-term sum over the warps;
taking every step as a truncating fp32 add (2^-23 relative, the tensor cores'
accumulator may truncate) and 32 steps of slack gives
``|Y - Y_ref| <= (8 ceil(n_chunks / 8) + 32) 2^-23 sum_k |x_k| |w^_rk|``.
"""
import math

import numpy as np
import pytest
import torch

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


def _abs_bound(words, scales, zeros, x, group):
    """(8 ceil(n_chunks/8) + 32) 2^-23 |X| |W^|^T, the error bound above."""
    d_col = x.shape[1]
    q = O.unpack_codes(np.asarray(words).view(np.uint32), 4, d_col).astype(np.float64)
    gi = np.arange(d_col) // (group if group else d_col)
    s = np.asarray(scales, np.float64)[:, gi]
    z = np.asarray(zeros, np.float64)[:, gi]
    steps = 8 * math.ceil(math.ceil(d_col / 128) / 8) + 32
    return steps * 2.0 ** -23 * (np.abs(np.asarray(x, np.float64)) @ np.abs(s * (q - z)).T)


def _run(G, words, scales, zeros, x, group):
    cfg = G.make_config(bits=4, group_size=group)
    batch, d_row = x.shape[0], words.shape[0]
    y_full = torch.full((batch + 1, d_row), float("nan"), device="cuda")
    y = G.gptq_w4a16_matmul(words.cuda(), scales.cuda(), zeros.cuda(), cfg,
                            x.cuda(), Y=y_full[:batch])
    torch.cuda.synchronize()
    yf = y_full.cpu().numpy()
    assert np.isnan(yf[batch]).all(), "wrote past the batch rows"
    return yf[:batch].astype(np.float64)


def _check(y, words, scales, zeros, x, group, rows=None):
    w, s, z = words.numpy(), scales.numpy(), zeros.numpy()
    if rows is not None:
        w, s, z, y = w[rows], s[rows], z[rows], y[:, rows]
    xf = x.float().numpy()
    ref = O.dequantized_matmul(w.view(np.uint32), s, z, xf, 4, group)
    bound = _abs_bound(w, s, z, xf, group)
    err = np.abs(y - ref)
    assert np.all(np.isfinite(y))
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
    return float(np.max(err / bound))


# d_row, d_col, group, batch: per channel and g = 32/64/128/256 (the three
# column layouts of the kernel), ragged row tiles, partial 128-column chunks,
# every batch width from 1 to 8
CASES = [
    (64, 256, 0, 1), (64, 256, 0, 8), (33, 160, 0, 3), (128, 512, 128, 5),
    (48, 384, 64, 2), (40, 320, 32, 7), (16, 32, 32, 1), (300, 1024, 256, 4),
    (17, 4096, 128, 8), (80, 2080, 0, 6), (1, 32, 0, 8), (96, 1536, 64, 8),
    (24, 2048, 32, 4),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_w4a16_matches_oracle(G, case):
    d_row, d_col, group, batch = case
    seed = d_row + 3 * d_col + group + batch
    words, scales, zeros = synth.gen_packed_layer(d_row, d_col, group, seed)
    x = synth.gen_activations(batch, d_col, seed)
    y = _run(G, words, scales, zeros, x, group)
    _check(y, words, scales, zeros, x, group)


def test_w4a16_oracle_quantized_layer(G):
    """The matmul of a layer the oracle quantized (packed by the oracle)."""
    spec = synth.tiny_spec(96, 512, 2048, seed=5).with_(group=128)
    w = synth.gen_weight(spec).numpy().astype(np.float64)
    ref = O.gptq(w, O.hessian(synth.gen_tokens(spec).float().numpy()), bits=4,
                 group=128, sym=False, block=128, damp_rel=0.01)
    words = torch.from_numpy(O.pack_codes(ref["codes"], 4).view(np.int32))
    scales = torch.from_numpy(np.asarray(ref["scales"], np.float32))
    zeros = torch.from_numpy(np.asarray(ref["zeros"]).astype(np.uint8))
    x = synth.gen_activations(4, 512, seed=5)
    y = _run(G, words, scales, zeros, x, 128)
    _check(y, words, scales, zeros, x, 128)
    # and it is X W^T of the oracle's own dequantized layer
    np.testing.assert_allclose(y, x.double().numpy() @ ref["w_hat"].T,
                               rtol=1e-4, atol=1e-4 * np.abs(y).max())


def test_w4a16_gpu_quantized_layer(G):
    """Chained on the GPU: quantize, then multiply; equals X W^T for the W^
    that gptq_dequant_check reconstructs from the same packed layer."""
    spec = synth.tiny_spec(128, 768, 3000, seed=2).with_(group=128)
    d = spec.d_col
    cfg = G.make_config(bits=4, group_size=128)
    xt, w = synth.gen_tokens(spec).cuda(), synth.gen_weight(spec).cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    g = torch.empty_like(h)
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(spec.d_row, d, cfg)
    qw, sc, ze = G.alloc_outputs(spec.d_row, d, cfg)
    G.gptq_hessian_accumulate(h, xt)
    G.gptq_prepare_hinv(h, 0.01, g, dead, ws)
    G.gptq_quantize_layer(w, g, dead, cfg, qw, sc, ze, ws)
    w_hat = torch.empty_like(w)
    G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat, ws=ws)
    x = synth.gen_activations(8, d, seed=2).cuda()
    y = G.gptq_w4a16_matmul(qw, sc, ze, cfg, x)
    assert G.gptq_device_status() == 0
    ref = x.double() @ w_hat.double().T
    bound = _abs_bound(qw.cpu(), sc.cpu(), ze.cpu(), x.cpu().float(), 128)
    err = (y.double() - ref).abs().cpu().numpy()
    assert np.all(err <= bound + 1e-6 * np.abs(ref.cpu().numpy()))


# full-size layers (LLaMA-65B MLP, LLaMA-7B attention), checked on sampled
# rows that include the first and the last row tile
FULL = [
    (22016, 8192, 128, 1), (22016, 8192, 128, 8), (8192, 22016, 0, 1),
    (8192, 22016, 128, 4), (4096, 4096, 0, 8),
]


@pytest.mark.parametrize("case", FULL, ids=lambda c: "x".join(map(str, c)))
def test_w4a16_full_size_sampled(G, case):
    d_row, d_col, group, batch = case
    words, scales, zeros = synth.gen_packed_layer(d_row, d_col, group, seed=11)
    x = synth.gen_activations(batch, d_col, seed=11)
    y = _run(G, words, scales, zeros, x, group)
    rng = np.random.default_rng(d_row + d_col)
    rows = np.unique(np.concatenate([np.arange(16), np.arange(d_row - 16, d_row),
                                     rng.choice(d_row, 32, replace=False)]))
    _check(y, words, scales, zeros, x, group, rows=rows)


def test_w4a16_rejects_other_widths(G):
    words, scales, zeros = synth.gen_packed_layer(16, 64, 0)
    x = synth.gen_activations(1, 64).cuda()
    with pytest.raises(G.GptqError):
        G.gptq_w4a16_matmul(words.cuda(), scales.cuda(), zeros.cuda(),
                            G.make_config(bits=3), x)
