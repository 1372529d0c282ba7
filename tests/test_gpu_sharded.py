"""The sharded one-layer sequence on one GPU (a single rank): cuda_steps runs
the library's kernels in the order of quantize_layer_sharded.  With one
rank the collectives are no-ops, so the result must be bit-identical to the
direct calls, and at parity with the oracle like them.  (More ranks need
more GPUs; the multi-rank host logic is covered on CPU gloo ranks.)
"""
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


@pytest.mark.parametrize("route", ["factor", "inverse"])
def test_one_rank_sequence_equals_the_direct_calls(G, route):
    from post_weight_quantization_26_b200 import sharded
    spec = synth.tiny_spec(96, 512, 3000, seed=8).with_(group=128)
    cfg = G.make_config(bits=4, group_size=128)
    x, w = synth.gen_tokens(spec).cuda(), synth.gen_weight(spec).cuda()
    qw, sc, ze, H = sharded.quantize_layer_sharded(
        sharded.cuda_steps(cfg, 0.01, 1, route=route), x, w, 512)
    prep = G.gptq_prepare_factor if route == "factor" else G.gptq_prepare_hinv
    quant = G.gptq_quantize_layer_factor if route == "factor" else G.gptq_quantize_layer
    # the direct calls
    h = torch.zeros((512, 512), dtype=torch.float32, device="cuda")
    g = torch.empty_like(h)
    dead = torch.empty(512, dtype=torch.uint8, device="cuda")
    ws = G.alloc_workspace(96, 512, cfg)
    q2, s2, z2 = G.alloc_outputs(96, 512, cfg)
    G.gptq_hessian_accumulate(h, x)
    prep(h, 0.01, g, dead, ws)
    quant(w, g, dead, cfg, q2, s2, z2, ws)
    torch.cuda.synchronize()
    assert G.gptq_device_status() == 0
    # the Hessian's tiles are summed by TMA reduce-add in a run-dependent
    # order, so H (and what follows from it) may differ in the last bits
    iu = np.triu_indices(512)
    a, b = H.cpu().numpy()[iu].astype(np.float64), h.cpu().numpy()[iu].astype(np.float64)
    assert np.linalg.norm(a - b) <= 1e-6 * np.linalg.norm(b)
    codes = O.unpack_codes(qw.cpu().numpy().view(np.uint32), 4, 512)
    codes2 = O.unpack_codes(q2.cpu().numpy().view(np.uint32), 4, 512)
    assert np.mean(codes != codes2) <= 1e-3
    ref = O.gptq(w.cpu().numpy().astype(np.float64), O.hessian(x.cpu().float().numpy()), bits=4,
                 group=128, sym=False, block=128, damp_rel=0.01)
    diff = np.abs(codes - ref["codes"])
    assert diff.max() <= 1 and np.mean(diff != 0) <= 1e-3


def test_one_rank_empty_token_shard_and_empty_rows(G):
    """A rank with no tokens adds nothing to H; a rank with no rows returns
    empty outputs (both happen when a layer has fewer rows or tokens than
    there are ranks)."""
    from post_weight_quantization_26_b200 import sharded
    cfg = G.make_config(bits=4, group_size=0)
    steps = sharded.cuda_steps(cfg, 0.01, 1)
    H = steps.zeros_h(256)
    steps.accumulate(H, torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"))
    assert float(H.abs().max()) == 0.0
    H += torch.eye(256, device="cuda") * 2.0
    g, dead = steps.prepare(H)
    qw, sc, ze = steps.quantize(torch.empty((0, 256), device="cuda"), g, dead)
    torch.cuda.synchronize()
    assert qw.shape[0] == sc.shape[0] == ze.shape[0] == 0
    assert G.gptq_device_status() == 0
