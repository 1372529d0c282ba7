"""gptq_dequant_check_noalloc: the loss check for callers that cannot
allocate device memory (no workspace argument; the library's fixed device
array is the scratch).  Its results must match gptq_dequant_check, which
takes a caller workspace, on two calls in a row (the shared scratch keeps the
previous call's contents, so a second call checks that nothing stale leaks
into the result).  Kept in its own file, collected last."""
import numpy as np
import pytest
import torch

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


def _quantized_layer(G, spec):
    d = spec.d_col
    cfg = G.make_config(bits=spec.bits, group_size=spec.group, sym=spec.sym,
                        block=spec.block, damp_rel=spec.damp)
    x = synth.gen_tokens(spec).cuda()
    w = synth.gen_weight(spec).cuda()
    h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
    g = torch.empty_like(h)
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(spec.d_row, d, cfg)
    qw, sc, ze = G.alloc_outputs(spec.d_row, d, cfg)
    G.gptq_hessian_accumulate(h, x)
    G.gptq_prepare_hinv(h, spec.damp, g, dead, ws)
    G.gptq_quantize_layer(w, g, dead, cfg, qw, sc, ze, ws)
    return cfg, w, h, qw, sc, ze, ws


@pytest.mark.parametrize("shape", [(256, 256, 0, 4), (200, 384, 128, 4), (192, 512, 128, 3),
                                   (130, 256, 0, 8)])
def test_noalloc_matches_workspace_version_twice(G, shape):
    d_row, d_col, group, bits = shape
    spec = synth.tiny_spec(d_row, d_col, 1024, seed=d_row).with_(group=group, bits=bits)
    cfg, w, h, qw, sc, ze, ws = _quantized_layer(G, spec)
    w_hat_ref = torch.empty_like(w)
    loss_ref = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat_ref, ws=ws)
    assert np.isfinite(loss_ref) and loss_ref > 0
    for _ in range(2):
        w_hat = torch.full_like(w, float("nan"))
        loss = G.gptq_dequant_check_noalloc(qw, sc, ze, w, h, cfg, W_hat=w_hat)
        assert loss == pytest.approx(loss_ref, rel=1e-12)
        torch.testing.assert_close(w_hat, w_hat_ref, rtol=0, atol=0)
    assert G.gptq_device_status() == 0


def test_noalloc_after_a_larger_call(G):
    """A smaller layer after a larger one must not read the larger call's
    leftover partial sums."""
    big = synth.tiny_spec(512, 512, 1024, seed=5)
    small = synth.tiny_spec(128, 128, 1024, seed=6)
    cfg_b, w_b, h_b, qw_b, sc_b, ze_b, _ = _quantized_layer(G, big)
    cfg_s, w_s, h_s, qw_s, sc_s, ze_s, ws_s = _quantized_layer(G, small)
    G.gptq_dequant_check_noalloc(qw_b, sc_b, ze_b, w_b, h_b, cfg_b)
    ref = G.gptq_dequant_check(qw_s, sc_s, ze_s, w_s, h_s, cfg_s, ws=ws_s)
    got = G.gptq_dequant_check_noalloc(qw_s, sc_s, ze_s, w_s, h_s, cfg_s)
    assert got == pytest.approx(ref, rel=1e-12)


def test_noalloc_many_tiles(G):
    """A 16384 x 4096 layer: 4096 tiles of 128 x 128, so the scratch holds
    thousands of partial sums; twice in a row, against the workspace
    version.  The packed layer is a seeded random one in the quantizer's
    format (only the format matters to the check)."""
    d_row, d_col = 16384, 4096
    words, scales, zeros = synth.gen_packed_layer(d_row, d_col, 128, seed=9)
    cfg = G.make_config(bits=4, group_size=128)
    spec = synth.tiny_spec(d_row, d_col, 8192, seed=9)
    w = synth.gen_weight(spec).cuda()
    x = synth.gen_tokens(spec).cuda()
    h = torch.zeros((d_col, d_col), dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(h, x)
    qw, sc, ze = words.cuda(), scales.cuda(), zeros.cuda()
    ws = G.alloc_workspace(d_row, d_col, cfg)
    w_hat_ref = torch.empty_like(w)
    loss_ref = G.gptq_dequant_check(qw, sc, ze, w, h, cfg, W_hat=w_hat_ref, ws=ws)
    assert np.isfinite(loss_ref) and loss_ref > 0
    for _ in range(2):
        w_hat = torch.full_like(w, float("nan"))
        loss = G.gptq_dequant_check_noalloc(qw, sc, ze, w, h, cfg, W_hat=w_hat)
        assert loss == pytest.approx(loss_ref, rel=1e-12)
        torch.testing.assert_close(w_hat, w_hat_ref, rtol=0, atol=0)
    assert G.gptq_device_status() == 0


def test_noalloc_rejects_layers_beyond_its_scratch(G):
    """More than GPTQ_NOALLOC_MAX_TILES 128x128 tiles is an argument error,
    raised before anything runs (the pointers below are never read)."""
    import ctypes
    lib = G.load_library()
    cfg = G.make_config(bits=4)
    fake = ctypes.c_void_p(0x7F0000000000)
    out = ctypes.c_double()
    rows = 128 * (G.NOALLOC_MAX_TILES // 256 + 1)  # with d_col = 256*128 columns
    st = lib.gptq_dequant_check_noalloc(fake, fake, fake, fake, fake, rows, 256 * 128,
                                        ctypes.byref(cfg), None, ctypes.byref(out), None)
    assert st == 1  # GPTQ_ERR_INVALID
