"""Seeded synthetic inputs for GPTQ layer quantization.

This module only draws random numbers: it holds none of the quantization
arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any of the method's code.

The workloads stand in for the calibration set and weights that the GPTQ
description uses (dingiv.github.io "量化" page, section GPTQ: 128 calibration
segments sampled from C4, LLaMA layers).  Neither C4 nor trained LLaMA
weights exist here, so:

* calibration activations X are token-major ``[n_tokens][d_col]`` bf16 with
  N(0,1) entries (or a SiLU-gated product ``silu(a)*b`` of two N(0,1) draws for
  the input of a down projection); a fixed set of "outlier" channels is
  multiplied by a factor in fp32 and the result rounded once to bf16;
* weights W are ``[d_row][d_col]`` with N(0, sigma^2) or Student-t(nu=5)*sigma
  entries, the latter drawn as ``z / sqrt(sum_{i<5} z_i^2 / 5)``; bf16-valued
  for the LLaMA-shaped layers, fp32 for the small layer.

Token chunk ``i`` (``CHUNK`` tokens) of an activation stream with seed ``s`` is
drawn from a CPU ``torch.Generator`` seeded with ``s * 1000003 + i``, so any
token range can be regenerated independently and identically.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, replace

import torch

CHUNK = 8192  # tokens per independently seeded activation chunk


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer's quantization problem: shapes, input recipe, quantizer."""

    name: str
    d_row: int  # output channels (rows of W)
    d_col: int  # input channels (columns of W, dimension of H)
    n_tokens: int  # calibration tokens
    w_dist: str = "normal"  # "normal" | "student_t5"
    w_sigma: float = 0.02
    w_bf16: bool = False  # round W to bf16 (LLaMA-shaped layers)
    x_dist: str = "normal"  # "normal" | "silu_gated"
    outlier_count: int = 0
    outlier_scale: float = 1.0
    bits: int = 4
    group: int = 0  # 0 = one scale per output channel
    sym: bool = False
    block: int = 128
    damp: float = 0.01
    w_seed: int = 0
    x_seed: int = 0

    @property
    def n_groups(self) -> int:
        return 1 if self.group == 0 else -(-self.d_col // self.group)

    def with_(self, **kw) -> "LayerSpec":
        return replace(self, **kw)


def _outliers(d: int, frac: float) -> int:
    return int(d * frac)


# The five workloads.  Seeds: W uses w_seed, X uses x_seed (+k for the k-th
# distinct input of a decoder block).
SMALL_256 = LayerSpec(
    name="small_256x256_t2048", d_row=256, d_col=256, n_tokens=2048,
    w_dist="normal", w_sigma=0.02, w_bf16=False, x_dist="normal",
    outlier_count=4, outlier_scale=20.0, bits=4, group=0, sym=False,
    block=128, damp=0.01, w_seed=0, x_seed=0)

Q_PROJ_7B = LayerSpec(
    name="llama7b_q_proj_4096x4096_t262144", d_row=4096, d_col=4096,
    n_tokens=262144, w_dist="student_t5", w_sigma=0.02, w_bf16=True,
    x_dist="normal", outlier_count=_outliers(4096, 0.01), outlier_scale=20.0,
    bits=4, group=0, sym=False, block=128, damp=0.01, w_seed=0, x_seed=1)

DOWN_PROJ_7B = LayerSpec(
    name="llama7b_down_proj_4096x11008_t262144", d_row=4096, d_col=11008,
    n_tokens=262144, w_dist="student_t5", w_sigma=0.02, w_bf16=True,
    x_dist="silu_gated", outlier_count=_outliers(11008, 0.01),
    outlier_scale=20.0, bits=4, group=128, sym=False, block=128, damp=0.01,
    w_seed=0, x_seed=1)


def decoder_block_7b(bits: int) -> list[tuple[LayerSpec, int]]:
    """The seven sublayers of a LLaMA-7B-shaped decoder block.

    Returns ``(spec, input_id)`` pairs; layers with the same ``input_id``
    share their calibration input and hence their Hessian (q/k/v share the
    attention input, gate/up share the MLP input; o and down have their own).
    """
    base = dict(n_tokens=262144, w_dist="student_t5", w_sigma=0.02,
                w_bf16=True, outlier_scale=20.0, bits=bits, group=128,
                sym=False, block=128, damp=0.01)
    out = []
    for k, (nm, dr, dc, xin, xd) in enumerate([
            ("q_proj", 4096, 4096, 0, "normal"),
            ("k_proj", 4096, 4096, 0, "normal"),
            ("v_proj", 4096, 4096, 0, "normal"),
            ("o_proj", 4096, 4096, 1, "normal"),
            ("gate_proj", 11008, 4096, 2, "normal"),
            ("up_proj", 11008, 4096, 2, "normal"),
            ("down_proj", 4096, 11008, 3, "silu_gated")]):
        spec = LayerSpec(name=f"llama7b_block_{nm}_{bits}bit", d_row=dr,
                         d_col=dc, x_dist=xd,
                         outlier_count=_outliers(dc, 0.01), w_seed=k,
                         x_seed=1 + xin, **base)
        out.append((spec, xin))
    return out


def mlp_65b(bits: int) -> list[tuple[LayerSpec, int]]:
    """65B-scale MLP: gate/up 22016x8192 sharing one input, down 8192x22016."""
    base = dict(n_tokens=131072, w_dist="student_t5", w_sigma=0.015,
                w_bf16=True, x_dist="normal", outlier_scale=30.0, bits=bits,
                group=128, sym=False, block=128, damp=0.01)
    return [
        (LayerSpec(name=f"llama65b_gate_proj_{bits}bit", d_row=22016,
                   d_col=8192, outlier_count=_outliers(8192, 0.005), w_seed=0,
                   x_seed=1, **base), 0),
        (LayerSpec(name=f"llama65b_up_proj_{bits}bit", d_row=22016,
                   d_col=8192, outlier_count=_outliers(8192, 0.005), w_seed=1,
                   x_seed=1, **base), 0),
        (LayerSpec(name=f"llama65b_down_proj_{bits}bit", d_row=8192,
                   d_col=22016, outlier_count=_outliers(22016, 0.005),
                   w_seed=2, x_seed=2, **base), 1),
    ]


def outlier_channels(spec: LayerSpec) -> torch.Tensor:
    """Indices of the channels of X that are scaled by ``outlier_scale``."""
    if spec.outlier_count == 0:
        return torch.zeros(0, dtype=torch.long)
    g = torch.Generator().manual_seed(spec.x_seed * 7919 + 17)
    return torch.randperm(spec.d_col, generator=g)[: spec.outlier_count]


def _student_t5(shape, g) -> torch.Tensor:
    z = torch.randn(shape, generator=g, dtype=torch.float32)
    chi = torch.zeros(shape, dtype=torch.float32)
    for _ in range(5):
        chi += torch.randn(shape, generator=g, dtype=torch.float32) ** 2
    return z / torch.sqrt(chi / 5.0)


def gen_weight(spec: LayerSpec) -> torch.Tensor:
    """W as a CPU fp32 tensor ``[d_row][d_col]`` (bf16-valued when w_bf16)."""
    g = torch.Generator().manual_seed(spec.w_seed * 1000003 + 12345)
    shape = (spec.d_row, spec.d_col)
    if spec.w_dist == "normal":
        w = torch.randn(shape, generator=g, dtype=torch.float32) * spec.w_sigma
    elif spec.w_dist == "student_t5":
        w = _student_t5(shape, g) * spec.w_sigma
    else:
        raise ValueError(spec.w_dist)
    if spec.w_bf16:
        w = w.to(torch.bfloat16).to(torch.float32)
    return w.contiguous()


def _chunk(spec: LayerSpec, i: int, idx: torch.Tensor) -> torch.Tensor:
    g = torch.Generator().manual_seed(spec.x_seed * 1000003 + i)
    shape = (CHUNK, spec.d_col)
    if spec.x_dist == "normal":
        x = torch.randn(shape, generator=g, dtype=torch.float32)
    elif spec.x_dist == "silu_gated":
        a = torch.randn(shape, generator=g, dtype=torch.float32)
        b = torch.randn(shape, generator=g, dtype=torch.float32)
        x = torch.nn.functional.silu(a) * b
    else:
        raise ValueError(spec.x_dist)
    if idx.numel():
        x[:, idx] *= spec.outlier_scale
    return x.to(torch.bfloat16)


def _free_host_bytes() -> float:
    """Available host memory in bytes (48 GB if it cannot be read)."""
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    return float(line.split()[1]) * 1024.0
    except OSError:
        pass
    return 48e9


def gen_tokens(spec: LayerSpec, t0: int = 0, t1: int | None = None,
               out: torch.Tensor | None = None,
               threads: int | None = None) -> torch.Tensor:
    """Calibration tokens ``[t0, t1)`` as a CPU bf16 tensor ``[t1-t0][d_col]``.

    ``out`` (optional, e.g. pinned memory) receives the rows in place.
    Chunks are independent, so they are drawn on a thread pool.
    """
    t1 = spec.n_tokens if t1 is None else t1
    assert 0 <= t0 <= t1 <= spec.n_tokens
    n = t1 - t0
    if out is None:
        out = torch.empty((n, spec.d_col), dtype=torch.bfloat16)
    assert out.shape == (n, spec.d_col) and out.dtype == torch.bfloat16
    if n == 0:
        return out
    idx = outlier_channels(spec)
    c0, c1 = t0 // CHUNK, (t1 - 1) // CHUNK

    def work(i: int) -> None:
        lo, hi = max(t0, i * CHUNK), min(t1, (i + 1) * CHUNK)
        x = _chunk(spec, i, idx)
        out[lo - t0: hi - t0].copy_(x[lo - i * CHUNK: hi - i * CHUNK])

    chunks = list(range(c0, c1 + 1))
    # one chunk's fp32 draws take ~3 x CHUNK x d_col x 4 bytes while in flight;
    # the chunks in flight may use up to a quarter of the free host memory
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    by_mem = max(1, int(_free_host_bytes() // 4 // (3 * CHUNK * spec.d_col * 4)))
    nthreads = threads or min(len(chunks), max(1, cores), by_mem)
    if nthreads <= 1 or len(chunks) == 1:
        for i in chunks:
            work(i)
    else:
        prev = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            with _cf.ThreadPoolExecutor(nthreads) as ex:
                list(ex.map(work, chunks))
        finally:
            torch.set_num_threads(prev)
    return out


def tiny_spec(d_row: int, d_col: int, n_tokens: int, seed: int = 0,
              **kw) -> LayerSpec:
    """A small layer with the same recipe as the 256x256 case, for tests."""
    kw.setdefault("outlier_count", max(0, d_col // 64))
    return SMALL_256.with_(name=f"tiny_{d_row}x{d_col}_t{n_tokens}",
                           d_row=d_row, d_col=d_col, n_tokens=n_tokens,
                           w_seed=seed, x_seed=seed, **kw)


def gen_packed_layer(d_row: int, d_col: int, group: int, seed: int = 0):
    """A random 4-bit packed layer in the quantizer's output format, as CPU
    tensors: ``words`` int32 ``[d_row][d_col/8]`` (uniform random bits, so
    every code 0..15 is equally likely), ``scales`` fp32 ``[d_row][n_groups]``
    drawn as ``0.002 + 0.01 |N(0,1)|``, ``zeros`` uint8 ``[d_row][n_groups]``
    uniform in 0..15.  Stands in for a quantized layer where only the format
    matters (the dequantized matmul), so no GPTQ run is needed at full size."""
    assert d_col % 8 == 0
    ng = 1 if group == 0 else d_col // group
    g = torch.Generator().manual_seed(seed * 1000003 + 4242)
    words = torch.randint(-(1 << 31), 1 << 31, (d_row, d_col // 8),
                          generator=g, dtype=torch.int64).to(torch.int32)
    scales = 0.002 + 0.01 * torch.randn((d_row, ng), generator=g).abs()
    zeros = torch.randint(0, 16, (d_row, ng), generator=g, dtype=torch.uint8)
    return words.contiguous(), scales.contiguous(), zeros.contiguous()


def gen_activations(batch: int, d_col: int, seed: int = 0) -> torch.Tensor:
    """``batch`` activation rows ``[batch][d_col]`` bf16 with N(0,1) entries
    (the decoding-time input of a quantized linear layer)."""
    g = torch.Generator().manual_seed(seed * 1000003 + 777)
    return torch.randn((batch, d_col), generator=g).to(torch.bfloat16)
