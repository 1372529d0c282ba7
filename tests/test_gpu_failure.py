"""Failure detection on the GPU, without faulting it, and a reproducible H.

* A bounded wait that runs out: the fault-injection switch makes the
  producer warp of the Hessian kernel (or of the trailing-update kernel)
  issue nothing, so the MMA thread's first wait on its mbarrier can never
  complete.  With a 20 ms limit the wait gives up, the kernel records
  GPTQ_ERR_TIMEOUT, frees its tensor memory and returns.  The tests check
  that status, that the stalled call wrote nothing (the Hessian), that the
  status is cleared once read, and that the next normal call on the same
  context is at parity with the oracle, which shows the abort path left the
  GPU usable.  No test traps, faults or hangs a kernel.
* A NaN or Inf in W is reported as GPTQ_ERR_NONFINITE by the quantize call.
* gptq_hessian_accumulate_ordered gives a bitwise reproducible H.
"""
import numpy as np
import pytest
import torch

from gptq_parity import check_layer
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth

pytestmark = pytest.mark.gpu

TIMEOUT, NONFINITE = 6, 3
LIMIT_NS = 20_000_000  # 20 ms


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_26_b200 import build, gptq
    build.build()
    gptq.load_library()
    yield gptq
    gptq.gptq_fault_inject(gptq.FAULT_NONE, 0)


def _rel_upper(h_gpu, h_ref):
    iu = np.triu_indices(h_ref.shape[0])
    a = h_gpu.cpu().numpy()[iu].astype(np.float64)
    return np.linalg.norm(a - h_ref[iu]) / np.linalg.norm(h_ref[iu])


def _layer(d_row, d_col, n, seed, **kw):
    spec = synth.tiny_spec(d_row, d_col, n, seed=seed).with_(**kw)
    return spec, synth.gen_weight(spec), synth.gen_tokens(spec)


def _quantize(G, spec, w, g, dead, ws):
    cfg = G.make_config(bits=spec.bits, group_size=spec.group, sym=spec.sym, block=spec.block)
    qw, sc, ze = G.alloc_outputs(spec.d_row, spec.d_col, cfg)
    G.gptq_quantize_layer(w, g, dead, cfg, qw, sc, ze, ws)
    return qw, sc, ze


def test_hessian_wait_runs_out_and_the_context_recovers(G):
    spec, _, x = _layer(8, 512, 4096, seed=71)
    xd = x.cuda()
    h = torch.zeros((512, 512), dtype=torch.float32, device="cuda")
    assert G.gptq_device_status() == 0
    G.gptq_fault_inject(G.FAULT_SYRK_STALL, LIMIT_NS)
    try:
        G.gptq_hessian_accumulate(h, xd)
        status = G.gptq_device_status()
    finally:
        G.gptq_fault_inject(G.FAULT_NONE, 0)
    assert status == TIMEOUT
    assert G.gptq_device_status() == 0           # read once, then cleared
    assert float(h.abs().max()) == 0.0           # the aborted kernel added nothing
    G.gptq_hessian_accumulate(h, xd)             # the same context, normal limits
    assert G.gptq_device_status() == 0
    assert _rel_upper(h, O.hessian(x.float().numpy())) <= 1e-5


def test_trailing_update_wait_runs_out_and_the_context_recovers(G):
    spec, w, x = _layer(64, 512, 2048, seed=72, group=128)
    h64 = O.hessian(x.float().numpy())
    hd, dead = O.dampen(h64, 0.01)
    u32 = np.ascontiguousarray(O.hinv_cholesky_upper(hd), dtype=np.float32)
    g = torch.from_numpy(u32).cuda()
    wd = w.cuda()
    cfg = G.make_config(bits=4, group_size=128)
    ws = G.alloc_workspace(64, 512, cfg)
    before = _quantize(G, spec, wd, g, None, ws)
    assert G.gptq_device_status() == 0
    G.gptq_fault_inject(G.FAULT_TRAILING_STALL, LIMIT_NS)
    try:
        _quantize(G, spec, wd, g, None, ws)      # 4 blocks: two trailing launches stall
        status = G.gptq_device_status()
    finally:
        G.gptq_fault_inject(G.FAULT_NONE, 0)
    assert status == TIMEOUT
    assert G.gptq_device_status() == 0
    after = _quantize(G, spec, wd, g, None, ws)
    assert G.gptq_device_status() == 0
    for a, b in zip(before, after):               # the sweep is deterministic
        assert torch.equal(a, b)
    codes = O.unpack_codes(after[0].cpu().numpy().view(np.uint32), 4, 512)
    ref_codes, ref_s, ref_z, _, _ = O.gptq_quantize(
        w.numpy().astype(np.float64), u32.astype(np.float64), 4, 128, False, 128)
    check_layer(codes, after[1].cpu().numpy(), after[2].cpu().numpy(), ref_codes, ref_s,
                ref_z, 128)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_weight_is_reported(G, bad):
    spec, w, x = _layer(40, 256, 1024, seed=73)
    h64 = O.hessian(x.float().numpy())
    hd, _ = O.dampen(h64, 0.01)
    g = torch.from_numpy(np.ascontiguousarray(O.hinv_cholesky_upper(hd), dtype=np.float32)).cuda()
    cfg = G.make_config()
    ws = G.alloc_workspace(40, 256, cfg)
    wd = w.clone()
    wd[7, 100] = bad
    _quantize(G, spec, wd.cuda(), g, None, ws)
    assert G.gptq_device_status() == NONFINITE
    assert G.gptq_device_status() == 0
    # a dead input column is zeroed before quantization: a NaN there is harmless
    dead = torch.zeros(256, dtype=torch.uint8)
    dead[100] = 1
    _quantize(G, spec, wd.cuda(), g, dead.cuda(), ws)
    assert G.gptq_device_status() == 0


@pytest.mark.parametrize("d,n,chunks", [(1024, 20000, 1), (512, 30000, 3), (4096, 8192, 1)])
def test_ordered_hessian_is_bitwise_reproducible(G, d, n, chunks):
    """The same inputs give the same H bit for bit, at parity with the
    oracle and with the fast path (whose split partials may land in any
    order).  At these sizes the fast path splits the tokens."""
    _, _, x = _layer(8, d, n, seed=d + n)
    xd = x.cuda()
    bounds = np.linspace(0, n, chunks + 1).astype(int)
    hs = []
    for fn in (G.gptq_hessian_accumulate_ordered, G.gptq_hessian_accumulate_ordered,
               G.gptq_hessian_accumulate):
        h = torch.zeros((d, d), dtype=torch.float32, device="cuda")
        for a, b in zip(bounds[:-1], bounds[1:]):
            fn(h, xd[a:b])
        hs.append(h)
    assert G.gptq_device_status() == 0
    assert torch.equal(hs[0], hs[1])
    ref = O.hessian(x.float().numpy())
    assert _rel_upper(hs[0], ref) <= 1e-5
    assert _rel_upper(hs[2], ref) <= 1e-5
    assert float(torch.tril(hs[0], -1).abs().max()) == 0.0
