"""Plain, slow, fp64 CPU oracle for GPTQ layer-wise weight quantization.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` import this module.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers), and
the library never imports it.

What it follows (all on the dingiv.github.io "量化" page unless noted):

* section 量化基础: symmetric ``x_q = round(x/s)`` and asymmetric
  ``x_q = round(x/s + z)`` quantizers, dequantization ``x_q * s``;
* youleyou.com "LLM quantization basics", section 四 (量化形式): linear
  quantization with round() and clip() to ``[qmin, qmax]``, ``s`` the step,
  ``z`` the offset (the formula itself is lost in the page's extraction);
* section GPTQ: the per-layer objective ``argmin_W^ ||W X - W^ X||^2``; the
  Hessian ``H = 2 X X^T``; the OBS compensation
  ``delta_q = -(w_q - quant(w_q)) / [H^-1]_qq * H^-1_{:,q}`` applied to every
  not-yet-quantized weight; the fixed left-to-right column order; the
  Cholesky factor of ``H^-1`` through which all updates go; blocks of
  ``B = 128`` columns with immediate in-block updates and one lazy batched
  update of the columns to the right after each block; per-output-channel
  INT4 output;
* psvmc.cn "common LLM quantization methods", section 按量化粒度划分:
  per-channel and group-wise (128 elements per group) granularity, and the
  "simple rounding" / min-max quantizer that GPTQ improves on (round to
  nearest, the RTN comparator here).

Readings of points the pages leave open (each also listed in the design
notes): the matrix norm is the squared Frobenius norm; ``G`` is the upper
triangular ``U`` with ``U^T U = H^-1``; asymmetric codes live in
``[0, 2^b - 1]`` with ``s = (max(0,xmax) - min(0,xmin)) / (2^b - 1)`` and
``z = rint(-xmin / s)``, the quotient taken with s exact, i.e.
``rint((2^b - 1) (-xmin) / (xmax - xmin))`` with one rounding; symmetric
codes use ``s = max|x| / (2^(b-1) - 1)``, clip to ``[-2^(b-1), 2^(b-1) - 1]``
and are stored offset by ``2^(b-1)``;
rounding is half-to-even; group parameters come from the current (already
error-updated) weights at the group's first column, per-channel parameters
from the original weights; the damping adds ``damp * mean(diag H)`` to the
diagonal; a dead input channel (``H_ii = 0``) gets ``H'_ii = 1`` and its
weight column is zeroed.

Every function here is pinned by ``tests/test_oracle.py`` against closed
forms, invariants, brute force and hand-worked cases, except
``factor_blocks`` and ``factor_rows``: they define F for the sweep that
needs U only on its diagonal blocks, a reading of section GPTQ's
recurrence rather than a step the page prints, so the pages leave their
parity unpinned; ``tests/test_oracle_factor.py`` pins them against this
module's own sweep through U (and planted mistakes), the reversed-route
Cholesky and closed forms.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# Hessian  (section GPTQ: H = 2 X X^T, X is d_col x n)
# ---------------------------------------------------------------------------
def hessian(x_tokens, chunk: int = 16384) -> np.ndarray:
    """``H = 2 * sum_t x_t x_t^T`` in fp64 from token-major ``[n][d]`` input.

    bf16 inputs are exact in fp64, and so is each product; only the sum over
    tokens rounds.  Large inputs are processed ``chunk`` tokens at a time;
    anything with ``.shape`` whose token slices convert with ``np.asarray``
    is accepted.
    """
    x = x_tokens if hasattr(x_tokens, "shape") else np.asarray(x_tokens)
    n, d = x.shape
    h = np.zeros((d, d), dtype=F64)
    for t0 in range(0, n, chunk):
        xc = np.asarray(x[t0:t0 + chunk], dtype=F64)
        h += xc.T @ xc
    return 2.0 * h


def hessian_rows(x_tokens, rows, chunk: int = 4096) -> np.ndarray:
    """Rows ``rows`` of ``H = 2 * sum_t x_t x_t^T`` in fp64, for checking a
    few entries of a Hessian too large to form on the host.

    Same definition as :func:`hessian`, restricted to the requested rows.
    ``x_tokens`` is token-major ``[n][d]``; it only needs ``.shape`` and
    slicing along tokens whose slices convert with ``np.asarray``.
    """
    rows = np.asarray(rows, dtype=np.int64)
    n, d = x_tokens.shape
    out = np.zeros((rows.size, d), dtype=F64)
    for t0 in range(0, n, chunk):
        xc = np.asarray(x_tokens[t0:t0 + chunk], dtype=F64)
        out += xc[:, rows].T @ xc
    return 2.0 * out


# ---------------------------------------------------------------------------
# Damping, dead channels, and the Cholesky factor of H^-1
# ---------------------------------------------------------------------------
def dampen(h: np.ndarray, damp_rel: float):
    """Return ``(H', dead)``: ``H' = H + lambda*I`` with
    ``lambda = damp_rel * mean(diag H)``; a dead channel (``H_ii == 0``) gets
    ``H'_ii = 1`` instead.  The pages give no damping; the relative 1% rule is
    the workload's stated setting."""
    h = np.array(h, dtype=F64, copy=True)
    diag = np.diag(h).copy()
    dead = diag == 0.0
    lam = damp_rel * float(np.mean(diag))
    idx = np.arange(h.shape[0])
    h[idx, idx] += lam
    h[dead, dead] = 1.0
    return h, dead


def hinv_cholesky_upper(hd: np.ndarray) -> np.ndarray:
    """``U`` upper triangular with ``U^T U = H'^-1`` (section GPTQ, the
    Cholesky factor of the inverse Hessian), by the direct route: factor,
    invert, form the inverse, factor again."""
    lo = np.linalg.cholesky(hd)  # H' = L L^T
    lo_inv = np.linalg.inv(lo)
    hinv = lo_inv.T @ lo_inv  # H'^-1 = L^-T L^-1
    hinv = 0.5 * (hinv + hinv.T)
    return np.linalg.cholesky(hinv).T  # (chol lower)^T is upper


def hinv_cholesky_upper_reversed(hd: np.ndarray) -> np.ndarray:
    """The same ``U`` by the reversed route: with ``J`` the order-reversing
    permutation, ``J H' J = L' L'^T`` gives ``H' = V V^T`` for the upper
    triangular ``V = J L' J``, and then ``U = V^-1``.  Exact arithmetic gives
    the direct route's result; the oracle keeps both to pin that reading."""
    d = hd.shape[0]
    rev = np.arange(d)[::-1]
    lp = np.linalg.cholesky(hd[np.ix_(rev, rev)])
    v = lp[np.ix_(rev, rev)]
    return np.linalg.inv(v)


# ---------------------------------------------------------------------------
# Quantizer (section 量化基础; youleyou section 四; psvmc min-max)
# ---------------------------------------------------------------------------
def quant_params(x, bits: int, sym: bool, dtype=F64):
    """Per-row scale and zero point for the values ``x`` (``[rows][k]``).

    ``dtype`` is the precision in which the integer decision is taken
    (float64 here; float32 when matching a float32 implementation)."""
    x = np.asarray(x, dtype=dtype)
    maxq = dtype(2 ** bits - 1)
    if sym:
        amax = np.max(np.abs(x), axis=1)
        amax = np.where(amax == 0, dtype(1), amax)
        s = amax / dtype(2 ** (bits - 1) - 1)
        z = np.full_like(s, dtype(2 ** (bits - 1)))
    else:
        xmin = np.minimum(np.min(x, axis=1), dtype(0))
        xmax = np.maximum(np.max(x, axis=1), dtype(0))
        both0 = (xmin == 0) & (xmax == 0)
        xmin = np.where(both0, dtype(-1), xmin)
        xmax = np.where(both0, dtype(1), xmax)
        s = (xmax - xmin) / maxq
        # z = rint(-xmin / s) with s = (xmax - xmin) / maxq taken exactly, as
        # one fp64 division of (for fp32 data) exact operands.  A tie, such
        # as a symmetric range (7.5 at 4 bits), is then rounded half to even
        # as the formula says, instead of being decided by how s rounded.
        z = np.rint(F64(maxq) * (-xmin.astype(F64)) / (xmax.astype(F64) - xmin.astype(F64)))
    return s.astype(dtype), z.astype(dtype)


def quantize(x, s, z, bits: int, dtype=F64):
    """Codes ``q = clip(rint(x/s) + z, 0, 2^b - 1)`` for a column ``x`` with
    per-row ``s``, ``z`` (the stored form of both quantizers)."""
    x = np.asarray(x, dtype=dtype)
    q = np.rint(x / np.asarray(s, dtype=dtype)) + np.asarray(z, dtype=dtype)
    return np.clip(q, 0, 2 ** bits - 1).astype(np.int64)


def dequantize(q, s, z) -> np.ndarray:
    """``x^ = s * (q - z)`` in fp64."""
    return np.asarray(s, dtype=F64) * (np.asarray(q, dtype=F64) -
                                       np.asarray(z, dtype=F64))


def _group_bounds(d_col: int, group: int):
    g = d_col if group == 0 else group
    return [(c, min(c + g, d_col)) for c in range(0, d_col, g)]


def factor_blocks(u: np.ndarray, block: int = 128) -> np.ndarray:
    """``F`` for the sweep that never forms ``U`` outside its diagonal
    blocks.  Reading of section GPTQ's recurrence: with ``e_q = (w_q -
    w^_q) / U_qq`` and ``e_q U[q, k]`` subtracted from each later column,
    the original weights are ``W = W^ + E U``, so ``E = (W - W^) V`` with
    ``V = U^-1`` (upper, ``H' = V V^T``).  The running weights at the start
    of block ``b`` are then ``W_b + sum_{a<b} (W - W^)_a V_ab U_bb``.
    ``F`` holds ``U_bb`` on the diagonal blocks (``[block*b, block*b +
    block)``, the last one ragged) and ``V_ab U_bb`` right of them, zero
    below.  Parity unpinned by the pages (it is this reading); pinned by the
    tests against ``gptq_quantize`` and the identity ``E = (W - W^) V``."""
    u = np.asarray(u, dtype=F64)
    d = u.shape[0]
    v = np.linalg.inv(u)
    f = np.zeros_like(u)
    for b0 in range(0, d, block):
        b1 = min(b0 + block, d)
        f[b0:b1, b0:b1] = np.triu(u[b0:b1, b0:b1])
        f[:b0, b0:b1] = v[:b0, b0:b1] @ u[b0:b1, b0:b1]
    return f


def factor_rows(u: np.ndarray, rows, block: int = 128) -> np.ndarray:
    """Rows of ``factor_blocks(u, block)`` without inverting all of ``U``:
    row ``i`` of ``V = U^-1`` solves ``U^T x = e_i`` (one triangular solve),
    then ``F[i, b] = V[i, b] U_bb`` for the blocks right of ``i``'s and
    ``U[i, b]`` in its own block."""
    import scipy.linalg
    u = np.asarray(u, dtype=F64)
    d = u.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    rhs = np.zeros((d, rows.size), dtype=F64)
    rhs[rows, np.arange(rows.size)] = 1.0
    v_rows = scipy.linalg.solve_triangular(u, rhs, trans="T", lower=False).T
    out = np.zeros((rows.size, d), dtype=F64)
    for k, i in enumerate(rows):
        b0 = (i // block) * block
        b1 = min(b0 + block, d)
        out[k, i:b1] = u[i, i:b1]
        for c0 in range(b1, d, block):
            c1 = min(c0 + block, d)
            out[k, c0:c1] = v_rows[k, c0:c1] @ u[c0:c1, c0:c1]
    return out


# ---------------------------------------------------------------------------
# GPTQ  (section GPTQ: fixed order, Cholesky of H^-1, blocks + lazy update)
# ---------------------------------------------------------------------------
def gptq_quantize(w, u, bits: int, group: int, sym: bool, block: int,
                  dead=None, dtype=F64):
    """Quantize ``W`` (``[d_row][d_col]``) column by column, left to right,
    given ``U`` (upper, ``U^T U = H'^-1``).

    For column ``q``: code it, ``e = (w_q - w^_q) / U_qq``; subtract
    ``e * U[q, k]`` from every later column ``k`` of the same block at once;
    after the block, subtract ``E @ U[block, right]`` from all columns to the
    right.  ``e * U[q, q:]`` is the page's OBS step
    ``(w_q - quant(w_q)) / [H_F^-1]_qq * H_F^-1[:, q]`` over the remaining set
    ``F``, because ``U[q:, q:]^T U[q:, q:] = (H'_FF)^-1``.

    Returns ``codes [d_row][d_col]``, ``scales``/``zeros [d_row][n_groups]``,
    ``w_hat`` and the error matrix ``E`` (all columns).
    """
    w = np.array(w, dtype=F64, copy=True)
    u = np.asarray(u, dtype=F64)
    d_row, d_col = w.shape
    if dead is not None:
        w[:, np.asarray(dead, dtype=bool)] = 0.0
    groups = _group_bounds(d_col, group)
    n_groups = len(groups)
    scales = np.zeros((d_row, n_groups), dtype=F64)
    zeros = np.zeros((d_row, n_groups), dtype=F64)
    codes = np.zeros((d_row, d_col), dtype=np.int64)
    w_hat = np.zeros((d_row, d_col), dtype=F64)
    err = np.zeros((d_row, d_col), dtype=F64)
    g_of = np.zeros(d_col, dtype=np.int64)
    for gi, (c0, c1) in enumerate(groups):
        g_of[c0:c1] = gi
    if group == 0:  # per output channel: from the original (dead-zeroed) W
        s, z = quant_params(w, bits, sym, dtype)
        scales[:, 0], zeros[:, 0] = s, z
    for j0 in range(0, d_col, block):
        j1 = min(j0 + block, d_col)
        for q in range(j0, j1):
            gi = g_of[q]
            if group != 0 and q == groups[gi][0]:
                c0, c1 = groups[gi]
                s, z = quant_params(w[:, c0:c1], bits, sym, dtype)
                scales[:, gi], zeros[:, gi] = s, z
            s, z = scales[:, gi], zeros[:, gi]
            code = quantize(w[:, q], s, z, bits, dtype)
            wq = dequantize(code, s, z)
            e = (w[:, q] - wq) / u[q, q]
            w[:, q + 1:j1] -= np.outer(e, u[q, q + 1:j1])
            codes[:, q], w_hat[:, q], err[:, q] = code, wq, e
        if j1 < d_col:
            w[:, j1:] -= err[:, j0:j1] @ u[j0:j1, j1:]
    return codes, scales, zeros, w_hat, err


def gptq(w, h, bits: int = 4, group: int = 0, sym: bool = False,
         block: int = 128, damp_rel: float = 0.01, dtype=F64,
         route: str = "direct"):
    """Full layer: damp ``H``, factor, quantize.  Returns a dict."""
    hd, dead = dampen(h, damp_rel)
    u = (hinv_cholesky_upper(hd) if route == "direct"
         else hinv_cholesky_upper_reversed(hd))
    codes, scales, zeros, w_hat, err = gptq_quantize(
        w, u, bits, group, sym, block, dead=dead, dtype=dtype)
    return dict(codes=codes, scales=scales, zeros=zeros, w_hat=w_hat,
                err=err, u=u, h_damped=hd, dead=dead)


def rtn(w, bits: int = 4, group: int = 0, sym: bool = False, dtype=F64):
    """Round-to-nearest with the same quantizer and no error feedback:
    every group's parameters come from the original weights."""
    w = np.asarray(w, dtype=F64)
    d_row, d_col = w.shape
    groups = _group_bounds(d_col, group)
    scales = np.zeros((d_row, len(groups)))
    zeros = np.zeros((d_row, len(groups)))
    codes = np.zeros((d_row, d_col), dtype=np.int64)
    for gi, (c0, c1) in enumerate(groups):
        s, z = quant_params(w[:, c0:c1], bits, sym, dtype)
        scales[:, gi], zeros[:, gi] = s, z
        for q in range(c0, c1):
            codes[:, q] = quantize(w[:, q], s, z, bits, dtype)
    w_hat = np.zeros_like(w)
    for gi, (c0, c1) in enumerate(groups):
        w_hat[:, c0:c1] = dequantize(codes[:, c0:c1], scales[:, gi:gi + 1],
                                     zeros[:, gi:gi + 1])
    return dict(codes=codes, scales=scales, zeros=zeros, w_hat=w_hat)


def obs_unblocked(w, hd, bits: int, group: int = 0, sym: bool = False,
                  dtype=F64):
    """OBS-style reference for tiny layers: for each column ``q`` in order,
    explicitly invert ``H'`` restricted to the not-yet-quantized columns
    ``F = {q, ..., d-1}`` and apply the page's compensation
    ``delta = -(w_q - quant(w_q)) / [H_F^-1]_qq * H_F^-1[:, q]``.
    No Cholesky factor and no blocking."""
    w = np.array(w, dtype=F64, copy=True)
    hd = np.asarray(hd, dtype=F64)
    d_row, d_col = w.shape
    groups = _group_bounds(d_col, group)
    codes = np.zeros((d_row, d_col), dtype=np.int64)
    w_hat = np.zeros((d_row, d_col))
    if group == 0:
        s, z = quant_params(w, bits, sym, dtype)
    for q in range(d_col):
        if group != 0:
            for (c0, c1) in groups:
                if q == c0:
                    s, z = quant_params(w[:, c0:c1], bits, sym, dtype)
        hinv_f = np.linalg.inv(hd[q:, q:])
        code = quantize(w[:, q], s, z, bits, dtype)
        wq = dequantize(code, s, z)
        delta = -np.outer((w[:, q] - wq) / hinv_f[0, 0], hinv_f[:, 0])
        w[:, q:] += delta
        codes[:, q], w_hat[:, q] = code, wq
    return codes, w_hat


# ---------------------------------------------------------------------------
# Layer loss (section GPTQ objective)
# ---------------------------------------------------------------------------
def layer_loss_direct(w, w_hat, x_tokens) -> float:
    """``||W X - W^ X||_F^2`` with X given token-major (``X^T``)."""
    dw = np.asarray(w, dtype=F64) - np.asarray(w_hat, dtype=F64)
    y = dw @ np.asarray(x_tokens, dtype=F64).T
    return float(np.sum(y * y))


def layer_loss_hessian(w, w_hat, h) -> float:
    """The same loss through ``H = 2 X X^T``: ``1/2 * sum_r dW_r H dW_r^T``."""
    dw = np.asarray(w, dtype=F64) - np.asarray(w_hat, dtype=F64)
    return float(0.5 * np.sum((dw @ np.asarray(h, dtype=F64)) * dw))


# ---------------------------------------------------------------------------
# Packing of b-bit codes into 32-bit words
# ---------------------------------------------------------------------------
def pack_codes(codes, bits: int) -> np.ndarray:
    """Pack each row's codes into a little-endian bit stream of uint32 words:
    code ``k`` occupies bits ``[b*k, b*k + b)`` of the row, and word ``w``
    holds bits ``[32w, 32w + 32)``.  The row length times ``b`` must be a
    multiple of 32."""
    codes = np.asarray(codes, dtype=np.int64)
    rows, cols = codes.shape
    assert (cols * bits) % 32 == 0
    nwords = cols * bits // 32
    out = np.zeros((rows, nwords), dtype=np.uint64)
    for k in range(cols):
        bit = bits * k
        wi, off = bit // 32, bit % 32
        v = codes[:, k].astype(np.uint64)
        out[:, wi] |= (v << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            out[:, wi + 1] |= v >> np.uint64(32 - off)
    return out.astype(np.uint32)


def unpack_codes(words, bits: int, cols: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    words = np.asarray(words, dtype=np.uint64)
    rows = words.shape[0]
    mask = np.uint64((1 << bits) - 1)
    out = np.zeros((rows, cols), dtype=np.int64)
    for k in range(cols):
        bit = bits * k
        wi, off = bit // 32, bit % 32
        v = words[:, wi] >> np.uint64(off)
        if off + bits > 32:
            v |= words[:, wi + 1] << np.uint64(32 - off)
        out[:, k] = (v & mask).astype(np.int64)
    return out


# ---------------------------------------------------------------------------
# Using the packed output: Y = X W^T with W dequantized (weight-only
# quantized matmul; dingiv.github.io page, section GPTQ: the INT4 weights
# serve inference, where memory-bound batch-1 decoding speeds up)
# ---------------------------------------------------------------------------
def dequantized_matmul(words, scales, zeros, x, bits: int, group: int) -> np.ndarray:
    """``Y[b][r] = sum_k X[b][k] W^[r][k]`` in fp64, where ``W^`` is the
    dequantized layer: ``W^[r][k] = s[r][g(k)] * (q[r][k] - z[r][g(k)])``
    with ``q`` unpacked from ``words`` and ``g(k) = k // group`` (one group
    per row when ``group`` is 0)."""
    x = np.asarray(x, dtype=F64)
    cols = x.shape[1]
    q = unpack_codes(words, bits, cols).astype(F64)
    s = np.asarray(scales, dtype=F64)
    z = np.asarray(zeros, dtype=F64)
    g = np.arange(cols) // (group if group else cols)
    w_hat = s[:, g] * (q - z[:, g])
    return x @ w_hat.T
