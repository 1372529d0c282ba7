"""The any-size checks used by the full-size GPU tests, run on the CPU with
the oracle's own outputs: they must accept the oracle's GPTQ result and
reject outputs with a planted mistake (no error propagation, i.e. RTN codes;
a propagation with a sign error; a wrong factor)."""
import numpy as np
import pytest
import torch

import test_gpu_fullsize as T
from oracle import gptq_oracle as O
from post_weight_quantization_26_b200 import synth


def _as_out(codes, s, z, bits, group, d):
    cg = np.arange(d) // (group or d)
    return dict(qw=torch.from_numpy(O.pack_codes(codes, bits).astype(np.uint32).view(np.int32)),
                sc=torch.from_numpy(s.astype(np.float32)),
                ze=torch.from_numpy(z.astype(np.uint8)),
                w_hat=torch.from_numpy((s[:, cg] * (codes - z[:, cg])).astype(np.float32)))


@pytest.fixture(scope="module", params=[(0, 4), (128, 3)])
def layer(request):
    group, bits = request.param
    spec = synth.tiny_spec(64, 384, 3072, seed=11).with_(group=group, bits=bits)
    x = synth.gen_tokens(spec)
    w = synth.gen_weight(spec)
    h = O.hessian(x.float().numpy())
    hd, _ = O.dampen(h.astype(np.float32).astype(np.float64), spec.damp)
    u = O.hinv_cholesky_upper(hd).astype(np.float32)
    return spec, x, w, h, u


def _quantize(spec, w, u):
    return O.gptq_quantize(w.double().numpy(), u.astype(np.float64), spec.bits, spec.group,
                           spec.sym, spec.block, dtype=np.float32)


def test_accepts_oracle_output(layer):
    spec, x, w, h, u = layer
    codes, s, z, _, _ = _quantize(spec, w, u)
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    a, b = T._check_g_property(hu, torch.from_numpy(u), spec.damp, seed=0)
    T._check_rows_property(spec, w, _as_out(codes, s, z, spec.bits, spec.group, spec.d_col),
                           b, a, seed=1)
    T._check_h_rows(hu, x, spec, seed=0)


def test_rejects_rtn_output(layer):
    spec, x, w, h, u = layer
    r = O.rtn(w.double().numpy(), spec.bits, spec.group, spec.sym, dtype=np.float32)
    hu = np.triu(h).astype(np.float32)
    with pytest.raises(AssertionError):
        T._check_rows_property(spec, w, _as_out(r["codes"], r["scales"], r["zeros"], spec.bits,
                                                spec.group, spec.d_col), u, hu, seed=1)


def test_rejects_sign_error_in_propagation(layer):
    spec, x, w, h, u = layer
    flipped = u.copy()
    iu = np.triu_indices(u.shape[0], 1)
    flipped[iu] = -flipped[iu]       # updates go the wrong way
    codes, s, z, _, _ = _quantize(spec, w, flipped)
    hu = np.triu(h).astype(np.float32)
    with pytest.raises(AssertionError):
        T._check_rows_property(spec, w, _as_out(codes, s, z, spec.bits, spec.group, spec.d_col),
                               u, hu, seed=1)


def test_rejects_wrong_factor_and_wrong_h(layer):
    spec, x, w, h, u = layer
    hu = torch.from_numpy(np.triu(h).astype(np.float32))
    for plant in ("drop", "scale_row"):
        bad_u = u.copy()
        if plant == "drop":
            bad_u[5, 9] = 0.0            # one dropped term
        else:
            bad_u[20] *= 1.001           # one row off by 1e-3
        with pytest.raises(AssertionError):
            T._check_g_property(hu, torch.from_numpy(bad_u), spec.damp, seed=0)
    bad_h = hu.clone()
    bad_h[0, 10:] *= 1.001       # row 0 is always among the sampled rows
    with pytest.raises(AssertionError):
        T._check_h_rows(bad_h, x, spec, seed=0)
