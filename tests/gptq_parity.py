"""The parity bars of the GPTQ path, shared by the GPU tests.

The quantized layer is compared with the plain fp64 oracle (integer
decisions in fp64) at the stated tolerances:

* codes: at most 0.1% differ, and only by +-1;
* scales within 1e-5 relative and zero points equal, with one reading for
  group-wise layers (the dingiv.github.io "量化" page, section GPTQ, fits
  nothing about it, so it follows from the method): a group's parameters
  are fitted to the error-updated weights when its first column is reached,
  so a permitted +-1 code earlier in the same row changes them.  Such a
  group's scale and zero point count as differing items under the same 0.1%
  budget as the codes (codes, scales and zeros pooled), and zero points stay
  within +-1.  Every group of a row up to and including the group of its
  first differing code is held to 1e-5 and exact zeros, as are per-channel
  parameters (fitted to the original row, before any propagation).
* the layer loss within 0.5% of the oracle's.
"""
from __future__ import annotations

import numpy as np

CODE_FRAC = 1e-3    # at most 0.1% of codes (and of all pooled items) differ
SCALE_RTOL = 1e-5
LOSS_RTOL = 5e-3


def check_codes(c_gpu, c_ref, frac=CODE_FRAC):
    """At most `frac` of the codes differ, and only by +-1; returns the
    fraction that differs."""
    diff = np.abs(np.asarray(c_gpu, np.int64) - np.asarray(c_ref, np.int64))
    assert diff.max(initial=0) <= 1, f"a code is off by {diff.max()}"
    f = float(np.mean(diff != 0)) if diff.size else 0.0
    assert f <= frac, f"{f:.2e} of codes differ"
    return f


def check_layer(codes, scales, zeros, ref_codes, ref_scales, ref_zeros, group):
    """Codes, scales and zero points of a quantized layer (or of a set of its
    rows) against the oracle's, under the bars above.  Returns a summary."""
    codes = np.asarray(codes, np.int64)
    ref_codes = np.asarray(ref_codes, np.int64)
    sc = np.asarray(scales, np.float64)
    rs = np.asarray(ref_scales, np.float64)
    ze = np.asarray(zeros, np.int64)
    rz = np.rint(np.asarray(ref_zeros, np.float64)).astype(np.int64)
    assert codes.shape == ref_codes.shape and sc.shape == rs.shape == ze.shape == rz.shape
    code_frac = check_codes(codes, ref_codes)
    d_col = codes.shape[1]
    diff_cols = codes != ref_codes
    first = np.where(diff_cols.any(1), diff_cols.argmax(1), d_col)
    if group:
        starts = np.arange(sc.shape[1]) * group
        strict = starts[None, :] <= first[:, None]   # groups not after a differing code
    else:
        strict = np.ones(sc.shape, dtype=bool)
    rel = np.abs(sc - rs) / np.abs(rs)
    zd = np.abs(ze - rz)
    bad_s = rel > SCALE_RTOL
    bad_z = zd != 0
    assert not (bad_s & strict).any(), \
        f"scale rel {rel[strict].max():.2e} where no earlier code differs"
    assert not (bad_z & strict).any(), "a zero point differs where no earlier code differs"
    assert zd.max(initial=0) <= 1, f"a zero point is off by {zd.max()}"
    n_items = codes.size + sc.size + ze.size
    n_diff = int(diff_cols.sum() + bad_s.sum() + bad_z.sum())
    assert n_diff <= CODE_FRAC * n_items, \
        f"{n_diff} of {n_items} codes, scales and zeros differ"
    return {"code_frac": code_frac, "items_differing": n_diff, "items": n_items,
            "scale_rel_max_strict": float(rel[strict].max(initial=0.0))}


def check_loss(loss, ref_loss, rtol=LOSS_RTOL):
    assert abs(loss - ref_loss) <= rtol * abs(ref_loss), \
        f"loss {loss:.6g} vs the oracle's {ref_loss:.6g}"
