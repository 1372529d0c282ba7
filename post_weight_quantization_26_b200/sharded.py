"""One layer quantized on several GPUs (strong scaling).

GPTQ splits two ways (dingiv.github.io "量化" page, section GPTQ):

* H = 2 X X^T is a sum over calibration tokens, so rank r accumulates H over
  its own token shard and one sum all-reduce gives every rank the full H.
  This is the path's only exchange step.
* Given G (or F, the factor route's matrix), every row of W is quantized
  independently of the others, so every rank factors the same H (the
  kernels are deterministic, so the ranks get identical matrices and
  dead-channel masks, and nothing is broadcast) and quantizes its own
  contiguous shard of rows.  The packed outputs are
  row-major, so gathering the shards in rank order gives the layer's
  output.

The sequence is written once, over a ``steps`` object that supplies the
four compute steps and the two collectives.  :func:`cuda_steps` is the
product's implementation: the library's kernels on the rank's GPU and NCCL
over NVLink for the collectives.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Callable


def shard(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous balanced range [lo, hi) of n items for ``rank`` of
    ``world``: the first n % world ranks take one item more."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


@dataclass
class Steps:
    """The compute steps and collectives of one rank.

    ``zeros_h(d)`` returns a zeroed d x d Hessian buffer; ``accumulate(H,
    x)`` adds 2 x^T x for token-major x; ``allreduce_sum(H)`` sums H over
    the ranks in place; ``prepare(H)`` returns (G, dead); ``quantize(w, G,
    dead)`` returns (qweight, scales, zeros) for the rows w;
    ``allgather_rows(t)`` concatenates every rank's rows in rank order."""

    zeros_h: Callable[[int], Any]
    accumulate: Callable[[Any, Any], None]
    allreduce_sum: Callable[[Any], None]
    prepare: Callable[[Any], tuple]
    quantize: Callable[[Any, Any, Any], tuple]
    allgather_rows: Callable[[Any], Any]


def quantize_layer_sharded(steps: Steps, x_local, w_local, d_col: int, *, gather: bool = True):
    """Quantize one layer on all ranks.

    ``x_local``: this rank's calibration tokens (its token shard, token-major,
    possibly empty); ``w_local``: this rank's rows of W (its row shard).
    Returns ``(qweight, scales, zeros, H)``; with ``gather`` the packed
    outputs hold every rank's rows in rank order, else only this rank's."""
    H = steps.zeros_h(d_col)
    steps.accumulate(H, x_local)
    steps.allreduce_sum(H)
    G, dead = steps.prepare(H)
    out = steps.quantize(w_local, G, dead)
    if gather:
        out = tuple(steps.allgather_rows(t) for t in out)
    return (*out, H)


def gather_padded(t, world: int, device):
    """All-gather of row blocks whose sizes differ between ranks (balanced
    shards differ by at most one row): each part is padded to the largest,
    gathered in one call (the collectives want equal sizes), and trimmed."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return t
    n = torch.tensor([t.shape[0]], dtype=torch.int64, device=device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n)
    rows = [int(s.item()) for s in sizes]
    width = max(rows)
    padded = torch.zeros((width, *t.shape[1:]), dtype=t.dtype, device=device)
    padded[: t.shape[0]] = t
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded)
    return torch.cat([p[:r] for p, r in zip(parts, rows)], 0)


def cuda_steps(cfg, damp: float, world: int, device=None, route: str = "factor") -> Steps:
    """The library's kernels on this rank's GPU; NCCL collectives over the
    default process group (none when ``world`` is 1).  ``route`` "factor"
    prepares F and sweeps through it; "inverse" prepares G = chol(H^-1)."""
    import torch
    import torch.distributed as dist

    from . import gptq as G

    G.load_library()  # fails loudly without the library: there is no other path
    dev = torch.device(device or "cuda")
    if route not in ("factor", "inverse"):
        raise ValueError(f"unknown route {route!r}")
    prep = G.gptq_prepare_factor if route == "factor" else G.gptq_prepare_hinv
    quant = G.gptq_quantize_layer_factor if route == "factor" else G.gptq_quantize_layer

    def zeros_h(d):
        return torch.zeros((d, d), dtype=torch.float32, device=dev)

    def accumulate(H, x):
        G.gptq_hessian_accumulate(H, x)

    def allreduce_sum(H):
        if world > 1:
            dist.all_reduce(H, op=dist.ReduceOp.SUM)

    def prepare(H):
        d = H.shape[0]
        g = torch.empty_like(H)
        dead = torch.empty(d, dtype=torch.uint8, device=dev)
        ws = G.alloc_workspace(1, d, cfg, device=dev)
        prep(H, damp, g, dead, ws)
        return g, dead

    def quantize(w, g, dead):
        d_row, d_col = w.shape
        qw, sc, ze = G.alloc_outputs(d_row, d_col, cfg, device=dev)
        if d_row:
            ws = G.alloc_workspace(d_row, d_col, cfg, device=dev)
            quant(w, g, dead, cfg, qw, sc, ze, ws)
        return qw, sc, ze

    def allgather_rows(t):
        return gather_padded(t, world, dev)

    return Steps(zeros_h, accumulate, allreduce_sum, prepare, quantize, allgather_rows)
