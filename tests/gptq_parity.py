"""The parity bars of the GPTQ path, shared by the GPU tests.

The quantized layer is compared with the plain fp64 oracle (integer
decisions in fp64) at the stated tolerances, read as follows:

* a decision is a code, or a group's scale and zero point, fitted when the
  group's first column is reached (per channel: once per row, before any
  propagation);
* in every row, the first decision that differs from the oracle's is a +-1
  change: a code one step away, or a zero point one step away (with its
  scale);
* at most 0.1% of all items (codes, scales, zero points pooled) differ;
* everything a row holds before its first differing decision matches:
  codes and zero points exactly, scales within 1e-5 relative;
* the layer loss within 0.5% of the oracle's.

Why the first decision and not every code: GPTQ feeds each rounding error
into the columns to its right (dingiv.github.io "量化" page, section GPTQ).
The kernels work in fp32 and the oracle in fp64, so now and then a value
lands on the other side of a rounding boundary (a near-tie).  That first
flip is a legitimate +-1 difference, and the rest of the row is then
quantized from different inputs: its codes, and the group parameters fitted
to them, are later decisions on other data and may differ by more than one
step.  They count against the 0.1% budget.
"""
from __future__ import annotations

import numpy as np

CODE_FRAC = 1e-3    # at most 0.1% of the items differ
SCALE_RTOL = 1e-5
LOSS_RTOL = 5e-3


def check_codes(c_gpu, c_ref, frac=CODE_FRAC):
    """At most `frac` of the codes differ, and only by +-1 (for layers with
    no error feedback); returns the fraction that differs."""
    diff = np.abs(np.asarray(c_gpu, np.int64) - np.asarray(c_ref, np.int64))
    assert diff.max(initial=0) <= 1, f"a code is off by {diff.max()}"
    f = float(np.mean(diff != 0)) if diff.size else 0.0
    assert f <= frac, f"{f:.2e} of codes differ"
    return f


def check_layer(codes, scales, zeros, ref_codes, ref_scales, ref_zeros, group):
    """Codes, scales and zero points of a quantized layer (or of some of its
    rows) against the oracle's, under the bars above.  Returns a summary."""
    codes = np.asarray(codes, np.int64)
    ref_codes = np.asarray(ref_codes, np.int64)
    sc = np.asarray(scales, np.float64)
    rs = np.asarray(ref_scales, np.float64)
    ze = np.asarray(zeros, np.int64)
    rz = np.rint(np.asarray(ref_zeros, np.float64)).astype(np.int64)
    assert codes.shape == ref_codes.shape and sc.shape == rs.shape == ze.shape == rz.shape
    rows, d_col = codes.shape
    g = group or d_col
    rel = np.abs(sc - rs) / np.abs(rs)
    code_diff = codes != ref_codes
    par_diff = (rel > SCALE_RTOL) | (ze != rz)
    first_code = np.where(code_diff.any(1), code_diff.argmax(1), d_col)
    first_par = np.where(par_diff.any(1), par_diff.argmax(1) * g, d_col)
    for r in np.nonzero((first_code < d_col) | (first_par < d_col))[0]:
        if first_par[r] <= first_code[r]:   # the group's parameters differ first
            gi = first_par[r] // g
            # fitted to the same values up to rounding: the scale agrees and
            # the zero point is one step away (a near-tie of -xmin/s)
            assert rel[r, gi] <= SCALE_RTOL, \
                f"row {r}: group {gi}'s scale differs by {rel[r, gi]:.2e} before any code"
            assert abs(ze[r, gi] - rz[r, gi]) == 1, \
                f"row {r}: the first differing zero point is off by {ze[r, gi] - rz[r, gi]}"
        else:
            c = first_code[r]
            assert abs(codes[r, c] - ref_codes[r, c]) == 1, \
                f"row {r}: the first differing code (column {c}) is off by " \
                f"{codes[r, c] - ref_codes[r, c]}"
    n_items = codes.size + sc.size + ze.size
    n_diff = int(code_diff.sum() + (rel > SCALE_RTOL).sum() + (ze != rz).sum())
    assert n_diff <= CODE_FRAC * n_items, \
        f"{n_diff} of {n_items} codes, scales and zeros differ"
    return {"code_frac": float(code_diff.mean()), "items_differing": n_diff,
            "items": n_items, "rows_differing": int(((first_code < d_col) |
                                                     (first_par < d_col)).sum()),
            "max_code_step": int(np.abs(codes - ref_codes).max(initial=0))}


def check_loss(loss, ref_loss, rtol=LOSS_RTOL):
    assert abs(loss - ref_loss) <= rtol * abs(ref_loss), \
        f"loss {loss:.6g} vs the oracle's {ref_loss:.6g}"
