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


TIE_MARGIN = 1e-4   # in units of s: below the fp32 resolution of a running weight


def decision_margins(w_hat, err, u_diag, scales, group):
    """How far each of the oracle's code decisions lay from a rounding
    boundary, in units of the step s: the running weight a column was coded
    from is w^ + e U_qq, and its code rounds w'/s."""
    d_col = w_hat.shape[1]
    s = np.asarray(scales, np.float64)[:, np.arange(d_col) // (group or d_col)]
    x = (np.asarray(w_hat, np.float64) + np.asarray(err, np.float64) * u_diag[None, :]) / s
    return np.abs(x - np.floor(x) - 0.5)


def check_layer_up_to_ties(codes, scales, zeros, ref_codes, ref_scales, ref_zeros, margins,
                           group, max_tie_rows=2):
    """A row equals the oracle's row (codes and zero points exactly, scales
    within SCALE_RTOL) unless its first differing decision is a code one step
    away whose oracle margin is below TIE_MARGIN: a tie at the kernel's fp32
    resolution, where either code is correct and the rest of the row then
    follows from different values.  For layers of few rows, where one such
    row's later codes alone can pass the pooled 0.1% budget.  Returns the
    rows that met a tie."""
    codes = np.asarray(codes, np.int64)
    ref_codes = np.asarray(ref_codes, np.int64)
    rel = np.abs(np.asarray(scales, np.float64) - ref_scales) / np.abs(ref_scales)
    ze = np.asarray(zeros, np.int64)
    rz = np.rint(np.asarray(ref_zeros, np.float64)).astype(np.int64)
    g = group or codes.shape[1]
    tie_rows = []
    for r in range(codes.shape[0]):
        cd = np.nonzero(codes[r] != ref_codes[r])[0]
        pd = np.nonzero((rel[r] > SCALE_RTOL) | (ze[r] != rz[r]))[0]
        if cd.size == 0 and pd.size == 0:
            continue
        c = int(cd[0]) if cd.size else codes.shape[1]
        assert pd.size == 0 or pd[0] > c // g, f"row {r}: group {pd[0]}'s parameters differ first"
        assert abs(codes[r, c] - ref_codes[r, c]) == 1, f"row {r}: column {c} off by more than 1"
        assert margins[r, c] < TIE_MARGIN, \
            f"row {r}: column {c} differs {margins[r, c]:.2e} s from the tie"
        tie_rows.append((r, c, float(margins[r, c])))
    assert len(tie_rows) <= max_tie_rows, f"{len(tie_rows)} rows met a tie"
    return tie_rows


def check_loss(loss, ref_loss, rtol=LOSS_RTOL):
    assert abs(loss - ref_loss) <= rtol * abs(ref_loss), \
        f"loss {loss:.6g} vs the oracle's {ref_loss:.6g}"
