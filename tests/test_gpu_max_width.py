"""The largest width the calls accept, d = 65536: H, its factor and the column
sweep, where d^2 = 4.3e9 elements and every index into H, G or the fp64
working copies needs 64 bits.

* Hessian: sampled rows against the oracle's rows of H from the tokens.
* Factor: U^T U H' v = v on random vectors (the oracle cannot factor a
  65536^2 matrix in a test's time), and for the factor route's F the same
  identity with G applied through F.
* Sweep: with G = c I nothing propagates, so the layer is round-to-nearest:
  within the stated bars of the fp64 oracle's, and exactly the oracle's
  when that takes its decisions in fp32 as the kernel does.
"""
import numpy as np
import pytest
import torch

import test_gpu_fullsize as T
from gptq_parity import check_layer
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth

pytestmark = pytest.mark.gpu

D = 65536


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_26_b200 import build, gptq
    build.build()
    gptq.load_library()
    return gptq


def _sym_row(h_dev, i):
    """Row i of the symmetric H from the stored upper triangle."""
    return torch.cat([h_dev[:i, i], h_dev[i, i:]]).double().cpu().numpy()


def test_max_width_hessian_and_factor(G):
    torch.cuda.empty_cache()
    spec = synth.tiny_spec(8, D, 2048, seed=65)
    x = synth.gen_tokens(spec)
    h = torch.zeros((D, D), dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(h, x.cuda())
    torch.cuda.synchronize()
    assert G.gptq_device_status() == 0
    rows = [0, 1, 4095, 32768, D - 2, D - 1]
    ref = O.hessian_rows(T._Tokens(x), rows)
    for k, i in enumerate(rows):
        got = _sym_row(h, i)
        rel = np.linalg.norm(got - ref[k]) / np.linalg.norm(ref[k])
        assert rel <= 1e-5, f"H row {i}: rel {rel:.2e}"
    del x
    cfg = G.make_config()
    ws = G.alloc_workspace(8, D, cfg)
    g = torch.empty_like(h)
    dead = torch.empty(D, dtype=torch.uint8, device="cuda")
    assert G.gptq_prepare_hinv(h, 0.01, g, dead, ws) == -1
    assert G.gptq_device_status() == 0
    del ws
    torch.cuda.empty_cache()
    T._check_g_property(h, g, 0.01, seed=65)
    del g
    torch.cuda.empty_cache()
    # the factor route's F at the same width
    ws = G.alloc_workspace(8, D, cfg)
    f = torch.empty_like(h)
    assert G.gptq_prepare_factor(h, 0.01, f, dead, ws) == -1
    assert G.gptq_device_status() == 0
    del ws
    torch.cuda.empty_cache()
    T._check_f_property(h, f, 0.01, seed=66)
    del h, f, dead
    torch.cuda.empty_cache()


@pytest.mark.parametrize("route", ["inverse", "factor"])
def test_max_width_sweep_identity_is_rtn(G, route):
    """G = cI (and F = cI, the factor route's matrix for H' = c^-2 I)."""
    torch.cuda.empty_cache()
    d_row = 40
    spec = synth.tiny_spec(d_row, D, 8, seed=66)
    w = synth.gen_weight(spec).numpy()
    c = 1.0 / np.sqrt(5.05)
    g = torch.eye(D, dtype=torch.float32, device="cuda") * c
    quantize = G.gptq_quantize_layer_factor if route == "factor" else G.gptq_quantize_layer
    for bits, group in ((4, 128), (3, 0)):
        cfg = G.make_config(bits=bits, group_size=group)
        qw, sc, ze = G.alloc_outputs(d_row, D, cfg)
        ws = G.alloc_workspace(d_row, D, cfg)
        quantize(torch.from_numpy(w).cuda(), g, None, cfg, qw, sc, ze, ws)
        torch.cuda.synchronize()
        assert G.gptq_device_status() == 0
        codes = O.unpack_codes(qw.cpu().numpy().view(np.uint32), bits, D)
        sc_h, ze_h = sc.cpu().numpy(), ze.cpu().numpy()
        # the plain fp64 oracle, under the stated bars (a near-tie of x / s
        # may round the other way in fp32, and nothing propagates from it)
        r64 = O.rtn(w.astype(np.float64), bits, group, False)
        check_layer(codes, sc_h, ze_h, r64["codes"], r64["scales"], r64["zeros"], group)
        # the same decisions taken in fp32, as the kernel takes them: exact
        r32 = O.rtn(w.astype(np.float64), bits, group, False, dtype=np.float32)
        assert np.array_equal(codes, r32["codes"])
        assert np.array_equal(ze_h, np.rint(r32["zeros"]).astype(np.uint8))
        np.testing.assert_allclose(sc_h, r32["scales"], rtol=1e-6)
        del qw, sc, ze, ws
        torch.cuda.empty_cache()
    del g
    torch.cuda.empty_cache()
