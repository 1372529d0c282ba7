"""The factor checks used by the full-size GPU tests, run on the CPU with the
oracle's own matrices: U^T U H' v = v for G, and Vt Vt^T v = H' v for the
factor route's F (Vt rebuilt block column by block column).  Each must accept
the oracle's matrix rounded to fp32 and reject one with a planted mistake
(one dropped term, one row off by 1e-3, a transposed diagonal block)."""
import numpy as np
import pytest
import torch

import test_gpu_fullsize as T
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth


@pytest.fixture(scope="module", params=[384, 512])
def layer(request):
    d = request.param
    spec = synth.tiny_spec(64, d, 8 * d, seed=11)
    x = synth.gen_tokens(spec)
    h = O.hessian(x.float().numpy())
    hd, _ = O.dampen(h.astype(np.float32).astype(np.float64), spec.damp)
    u = O.hinv_cholesky_upper(hd).astype(np.float32)
    return spec, h, u


def test_accepts_oracle_factor(layer):
    spec, h, u = layer
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    T._check_g_property(hu, torch.from_numpy(u), spec.damp, seed=0)


@pytest.mark.parametrize("plant", ["drop", "scale_row"])
def test_rejects_wrong_factor(layer, plant):
    spec, h, u = layer
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    bad_u = u.copy()
    if plant == "drop":
        bad_u[5, 9] = 0.0            # one dropped term
    else:
        bad_u[20] *= 1.001           # one row off by 1e-3
    with pytest.raises(AssertionError):
        T._check_g_property(hu, torch.from_numpy(bad_u), spec.damp, seed=0)


@pytest.fixture(scope="module", params=[384, 416])
def factor_layer(request):
    d = request.param
    spec = synth.tiny_spec(64, d, 8 * d, seed=12)
    x = synth.gen_tokens(spec)
    h = O.hessian(x.float().numpy())
    hd, _ = O.dampen(h.astype(np.float32).astype(np.float64), spec.damp)
    f = O.factor_blocks(O.hinv_cholesky_upper(hd)).astype(np.float32)
    return spec, h, f


def test_f_check_accepts_oracle_f(factor_layer):
    spec, h, f = factor_layer
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    T._check_f_property(hu, torch.from_numpy(f), spec.damp, seed=0)


@pytest.mark.parametrize("plant", ["drop", "scale_row", "diag_transposed"])
def test_f_check_rejects_wrong_f(factor_layer, plant):
    spec, h, f = factor_layer
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    bad = f.copy()
    if plant == "drop":
        bad[5, 200] = 0.0             # one dropped term right of the diagonal block
    elif plant == "scale_row":
        bad[20] *= 1.001
    else:                             # V_ab G_bb^T in place of V_ab G_bb for one panel
        g = f[128:256, 128:256].astype(np.float64)
        vab = f[:128, 128:256].astype(np.float64) @ np.linalg.inv(g)
        bad[:128, 128:256] = (vab @ g.T).astype(np.float32)
    with pytest.raises(AssertionError):
        T._check_f_property(hu, torch.from_numpy(bad), spec.damp, seed=0)
