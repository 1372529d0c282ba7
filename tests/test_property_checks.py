"""The factor check used by the full-size GPU tests (U^T U H' v = v on random
vectors), run on the CPU with the oracle's own factor: it must accept the
oracle's U and reject a factor with a planted mistake (one dropped term, one
row off by 1e-3)."""
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
