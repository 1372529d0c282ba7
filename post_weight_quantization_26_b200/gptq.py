"""Python binding of libgptq.so (the C ABI in include/gptq.h).

Each function has the name of the C entry point it wraps and only marshals
arguments: torch CUDA tensors become device pointers, the current torch
stream becomes the ``stream`` argument, and a non-OK status raises
:class:`GptqError`.  Every step of the path runs in the library's kernels;
there is no CPU or PyTorch fallback, and importing this module fails if the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq.so")

GPTQ_OK = 0
STATUS_NAMES = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID", 2: "GPTQ_ERR_NOT_SPD",
                3: "GPTQ_ERR_NONFINITE", 4: "GPTQ_ERR_WORKSPACE",
                5: "GPTQ_ERR_CUDA", 6: "GPTQ_ERR_TIMEOUT"}

EXPORTED = ("gptq_workspace_size", "gptq_hessian_accumulate",
            "gptq_hessian_accumulate_ordered", "gptq_fault_inject", "gptq_prepare_hinv", "gptq_quantize_layer", "gptq_dequant_check",
            "gptq_prepare_factor", "gptq_quantize_layer_factor",
            "gptq_device_status", "gptq_status_string", "gptq_launch_count",
            "gptq_dequant_check_noalloc", "gptq_w4a16_matmul", "gptq_awq_channel_scale",
            "gptq_awq_workspace_size", "gptq_awq_search")
NOALLOC_MAX_TILES = 65536  # GPTQ_NOALLOC_MAX_TILES in include/gptq.h
FAULT_NONE, FAULT_SYRK_STALL, FAULT_TRAILING_STALL = 0, 1, 2  # GPTQ_FAULT_* in include/gptq.h


class GptqError(RuntimeError):
    def __init__(self, status: int, where: str, extra: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}{extra}")


class GptqConfig(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int),
                ("sym", ctypes.c_int), ("block", ctypes.c_int),
                ("damp_rel", ctypes.c_double)]


def make_config(bits=4, group_size=0, sym=False, block=128, damp_rel=0.01):
    return GptqConfig(int(bits), int(group_size), int(bool(sym)), int(block),
                      float(damp_rel))


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgptq.so; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libgptq.so not found at {path}; build it with "
            "`python -m post_weight_quantization_26_b200.build`")
    lib = ctypes.CDLL(path)
    P, I64, SZ, I, D, F = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t,
                           ctypes.c_int, ctypes.c_double, ctypes.c_float)
    cfgp = ctypes.POINTER(GptqConfig)
    lib.gptq_workspace_size.argtypes = [I64, I64, cfgp]
    lib.gptq_workspace_size.restype = SZ
    lib.gptq_hessian_accumulate.argtypes = [P, P, I64, I64, I64, F, P]
    lib.gptq_hessian_accumulate.restype = I
    lib.gptq_hessian_accumulate_ordered.argtypes = [P, P, I64, I64, I64, F, P]
    lib.gptq_hessian_accumulate_ordered.restype = I
    lib.gptq_fault_inject.argtypes = [I, I64]
    lib.gptq_fault_inject.restype = I
    lib.gptq_prepare_hinv.argtypes = [P, I64, D, P, P, P, SZ,
                                      ctypes.POINTER(I64), P]
    lib.gptq_prepare_hinv.restype = I
    lib.gptq_quantize_layer.argtypes = [P, I64, I64, P, P, cfgp, P, P, P, P,
                                        SZ, P]
    lib.gptq_quantize_layer.restype = I
    lib.gptq_prepare_factor.argtypes = lib.gptq_prepare_hinv.argtypes
    lib.gptq_prepare_factor.restype = I
    lib.gptq_quantize_layer_factor.argtypes = lib.gptq_quantize_layer.argtypes
    lib.gptq_quantize_layer_factor.restype = I
    lib.gptq_dequant_check.argtypes = [P, P, P, P, P, I64, I64, cfgp, P,
                                       ctypes.POINTER(D), P, SZ, P]
    lib.gptq_dequant_check.restype = I
    lib.gptq_dequant_check_noalloc.argtypes = [P, P, P, P, P, I64, I64, cfgp, P,
                                               ctypes.POINTER(D), P]
    lib.gptq_dequant_check_noalloc.restype = I
    lib.gptq_w4a16_matmul.argtypes = [P, P, P, I64, I64, cfgp, P, I64, P, P]
    lib.gptq_w4a16_matmul.restype = I
    lib.gptq_awq_channel_scale.argtypes = [P, I64, I64, I64, P, P]
    lib.gptq_awq_channel_scale.restype = I
    lib.gptq_awq_workspace_size.argtypes = [I64, I64, cfgp]
    lib.gptq_awq_workspace_size.restype = SZ
    lib.gptq_awq_search.argtypes = [P, P, P, I64, I64, cfgp, I, P, P, P, P, P, P, P, SZ, P]
    lib.gptq_awq_search.restype = I
    lib.gptq_device_status.argtypes = [P]
    lib.gptq_device_status.restype = I
    lib.gptq_launch_count.argtypes = []
    lib.gptq_launch_count.restype = ctypes.c_uint64
    lib.gptq_status_string.argtypes = [I]
    lib.gptq_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str, extra: str = ""):
    if st != GPTQ_OK:
        raise GptqError(st, where, extra)


def gptq_workspace_size(d_row: int, d_col: int, cfg: GptqConfig) -> int:
    n = load_library().gptq_workspace_size(d_row, d_col, ctypes.byref(cfg))
    if n == 0:
        raise GptqError(1, "gptq_workspace_size")
    return int(n)


def alloc_workspace(d_row: int, d_col: int, cfg: GptqConfig, device=None):
    """A uint8 CUDA tensor of gptq_workspace_size bytes (256-byte aligned)."""
    n = gptq_workspace_size(d_row, d_col, cfg)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def gptq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor,
                            scale: float = 2.0, stream=None) -> None:
    """H (fp32 d x d) += scale * X^T X for token-major bf16 X (n x d)."""
    _accumulate("gptq_hessian_accumulate", H, X, scale, stream)


def gptq_hessian_accumulate_ordered(H: torch.Tensor, X: torch.Tensor,
                                    scale: float = 2.0, stream=None) -> None:
    """gptq_hessian_accumulate with a fixed summation order (bitwise
    reproducible H)."""
    _accumulate("gptq_hessian_accumulate_ordered", H, X, scale, stream)


def _accumulate(name, H, X, scale, stream):
    assert H.dtype == torch.float32 and X.dtype == torch.bfloat16
    n, d = X.shape
    assert H.shape == (d, d) and H.is_contiguous() and X.stride(1) == 1
    st = getattr(load_library(), name)(
        _ptr(H), _ptr(X), n, d, X.stride(0), float(scale), _stream(stream))
    _check(st, name)


def gptq_fault_inject(where: int, wait_limit_ns: int = 0) -> None:
    """Set the fault injection of the failure-detection tests (FAULT_NONE
    and 0 restore normal operation)."""
    _check(load_library().gptq_fault_inject(int(where), int(wait_limit_ns)),
           "gptq_fault_inject")


def gptq_prepare_hinv(H: torch.Tensor, damp_rel: float, G: torch.Tensor,
                      dead_mask: torch.Tensor, ws: torch.Tensor,
                      stream=None) -> int:
    """G = upper U with U^T U = (H + damp)^-1.  Returns bad_pivot (-1 if SPD)."""
    d = H.shape[0]
    assert H.dtype == torch.float32 and H.shape == (d, d) and H.is_contiguous()
    assert G.dtype == torch.float32 and G.shape == (d, d) and G.is_contiguous()
    assert dead_mask.dtype == torch.uint8 and dead_mask.numel() == d
    piv = ctypes.c_int64(-1)
    st = load_library().gptq_prepare_hinv(
        _ptr(H), d, float(damp_rel), _ptr(G), _ptr(dead_mask), _ptr(ws),
        ws.numel(), ctypes.byref(piv), _stream(stream))
    _check(st, "gptq_prepare_hinv", f" (bad_pivot={piv.value})")
    return int(piv.value)


def gptq_prepare_factor(H: torch.Tensor, damp_rel: float, F: torch.Tensor,
                        dead_mask: torch.Tensor, ws: torch.Tensor,
                        stream=None) -> int:
    """F for gptq_quantize_layer_factor: G's 128x128 diagonal blocks and
    V_ab G_bb right of them (H + damp = V V^T).  Returns bad_pivot."""
    d = H.shape[0]
    assert H.dtype == torch.float32 and H.shape == (d, d) and H.is_contiguous()
    assert F.dtype == torch.float32 and F.shape == (d, d) and F.is_contiguous()
    assert dead_mask.dtype == torch.uint8 and dead_mask.numel() == d
    piv = ctypes.c_int64(-1)
    st = load_library().gptq_prepare_factor(
        _ptr(H), d, float(damp_rel), _ptr(F), _ptr(dead_mask), _ptr(ws),
        ws.numel(), ctypes.byref(piv), _stream(stream))
    _check(st, "gptq_prepare_factor", f" (bad_pivot={piv.value})")
    return int(piv.value)


def _quantize(name, W, G, dead_mask, cfg, qweight, scales, zeros, ws, stream):
    d_row, d_col = W.shape
    assert W.dtype == torch.float32 and W.is_contiguous()
    assert G.dtype == torch.float32 and G.shape == (d_col, d_col) and G.is_contiguous()
    assert qweight.dtype == torch.int32 or qweight.dtype == torch.uint32
    st = getattr(load_library(), name)(
        _ptr(W), d_row, d_col, _ptr(G), _ptr(dead_mask), ctypes.byref(cfg),
        _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(ws), ws.numel(),
        _stream(stream))
    _check(st, name)


def gptq_quantize_layer(W: torch.Tensor, G: torch.Tensor, dead_mask,
                        cfg: GptqConfig, qweight: torch.Tensor,
                        scales: torch.Tensor, zeros: torch.Tensor,
                        ws: torch.Tensor, stream=None) -> None:
    _quantize("gptq_quantize_layer", W, G, dead_mask, cfg, qweight, scales,
              zeros, ws, stream)


def gptq_quantize_layer_factor(W: torch.Tensor, F: torch.Tensor, dead_mask,
                               cfg: GptqConfig, qweight: torch.Tensor,
                               scales: torch.Tensor, zeros: torch.Tensor,
                               ws: torch.Tensor, stream=None) -> None:
    """The same layer from F (gptq_prepare_factor); block 128, group_size 0
    or a divisor of 128."""
    _quantize("gptq_quantize_layer_factor", W, F, dead_mask, cfg, qweight,
              scales, zeros, ws, stream)


def gptq_dequant_check(qweight, scales, zeros, W, H, cfg: GptqConfig,
                       W_hat=None, ws=None, want_loss: bool = True,
                       stream=None):
    """Returns the layer loss 1/2 sum_r dW_r H dW_r^T (or None)."""
    d_row, d_col = W.shape if W is not None else W_hat.shape
    loss = ctypes.c_double(float("nan"))
    st = load_library().gptq_dequant_check(
        _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(W), _ptr(H), d_row,
        d_col, ctypes.byref(cfg), _ptr(W_hat),
        ctypes.byref(loss) if want_loss else None, _ptr(ws),
        0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "gptq_dequant_check")
    return loss.value if want_loss else None


def gptq_dequant_check_noalloc(qweight, scales, zeros, W, H, cfg: GptqConfig,
                               W_hat=None, want_loss: bool = True, stream=None):
    """gptq_dequant_check for callers that cannot allocate device memory:
    no workspace argument; the library's fixed 512 KB device array serves as
    scratch (see include/gptq.h for the size limit and the rules on
    overlapping calls).  Returns the layer loss (or None)."""
    d_row, d_col = W.shape if W is not None else W_hat.shape
    loss = ctypes.c_double(float("nan"))
    st = load_library().gptq_dequant_check_noalloc(
        _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(W), _ptr(H), d_row,
        d_col, ctypes.byref(cfg), _ptr(W_hat),
        ctypes.byref(loss) if want_loss else None, _stream(stream))
    _check(st, "gptq_dequant_check_noalloc")
    return loss.value if want_loss else None


def gptq_w4a16_matmul(qweight, scales, zeros, cfg: GptqConfig, X, Y=None,
                      stream=None):
    """Y = X W^T for bf16 X (batch x d_col, batch 1..8) and the packed 4-bit
    layer (qweight, scales, zeros) as gptq_quantize_layer wrote it.  Y is fp32
    batch x d_row, allocated here when not given.  Returns Y."""
    assert X.dtype == torch.bfloat16 and X.dim() == 2 and X.is_contiguous()
    batch, d_col = X.shape
    d_row = scales.shape[0]
    if Y is None:
        Y = torch.empty(batch, d_row, dtype=torch.float32, device=X.device)
    assert Y.dtype == torch.float32 and Y.shape == (batch, d_row) and Y.is_contiguous()
    st = load_library().gptq_w4a16_matmul(
        _ptr(qweight), _ptr(scales), _ptr(zeros), d_row, d_col,
        ctypes.byref(cfg), _ptr(X), batch, _ptr(Y), _stream(stream))
    _check(st, "gptq_w4a16_matmul")
    return Y


def gptq_awq_channel_scale(X, sx=None, stream=None):
    """sx[k] = mean_t |X[t][k]| (fp64) for token-major bf16 X (n x d)."""
    assert X.dtype == torch.bfloat16 and X.dim() == 2 and X.stride(1) == 1
    n, d = X.shape
    if sx is None:
        sx = torch.empty(d, dtype=torch.float64, device=X.device)
    st = load_library().gptq_awq_channel_scale(_ptr(X), n, d, X.stride(0), _ptr(sx),
                                               _stream(stream))
    _check(st, "gptq_awq_channel_scale")
    return sx


def gptq_awq_workspace_size(d_row: int, d_col: int, cfg: GptqConfig) -> int:
    n = load_library().gptq_awq_workspace_size(d_row, d_col, ctypes.byref(cfg))
    if n == 0:
        raise GptqError(1, "gptq_awq_workspace_size")
    return int(n)


def gptq_awq_search(W, H, sx, cfg: GptqConfig, n_grid: int = 20, ws=None, out=None,
                    stream=None):
    """The AWQ grid search over alpha; returns (losses fp64[n_grid], best
    int32[1], s fp32[d_col], qweight, scales, zeros), all on the device."""
    d_row, d_col = W.shape
    dev = W.device
    if ws is None:
        ws = torch.empty(gptq_awq_workspace_size(d_row, d_col, cfg), dtype=torch.uint8,
                         device=dev)
    if out is None:
        qw, sc, ze = alloc_outputs(d_row, d_col, cfg, device=dev)
        out = (torch.empty(n_grid, dtype=torch.float64, device=dev),
               torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty(d_col, dtype=torch.float32, device=dev), qw, sc, ze)
    losses, best, s, qw, sc, ze = out
    st = load_library().gptq_awq_search(
        _ptr(W), _ptr(H), _ptr(sx), d_row, d_col, ctypes.byref(cfg), int(n_grid), _ptr(losses),
        _ptr(best), _ptr(s), _ptr(qw), _ptr(sc), _ptr(ze), _ptr(ws), ws.numel(),
        _stream(stream))
    _check(st, "gptq_awq_search")
    return out


def gptq_device_status(stream=None) -> int:
    return int(load_library().gptq_device_status(_stream(stream)))


def gptq_launch_count() -> int:
    return int(load_library().gptq_launch_count())


def gptq_status_string(status: int) -> str:
    return load_library().gptq_status_string(int(status)).decode()


def n_groups(d_col: int, group_size: int) -> int:
    return 1 if group_size == 0 else d_col // group_size


def alloc_outputs(d_row: int, d_col: int, cfg: GptqConfig, device="cuda"):
    """qweight (int32 words), scales (fp32), zeros (uint8) for one layer."""
    ng = n_groups(d_col, cfg.group_size)
    qweight = torch.empty((d_row, d_col * cfg.bits // 32), dtype=torch.int32,
                          device=device)
    scales = torch.empty((d_row, ng), dtype=torch.float32, device=device)
    zeros = torch.empty((d_row, ng), dtype=torch.uint8, device=device)
    return qweight, scales, zeros
