"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every function include/gptq.h declares, and its argument
validation rejects bad calls before anything is launched."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_26_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(0x7F0000000000)  # never dereferenced: validation fails first


@pytest.fixture(scope="module")
def lib():
    B.build()
    from post_weight_quantization_26_b200 import gptq as G
    return G.load_library()


def _declared_functions():
    names = []
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[\w]+\*?\s+\*?(gptq_\w+)\s*\(",
                            text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("gptq_hessian_accumulate", "gptq_prepare_hinv",
              "gptq_quantize_layer", "gptq_dequant_check",
              "gptq_workspace_size", "gptq_status_string",
              "gptq_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    from post_weight_quantization_26_b200 import gptq as G
    for n in _declared_functions():
        assert callable(getattr(G, n)), n


def test_status_strings(lib):
    from post_weight_quantization_26_b200 import gptq as G
    for code, name in G.STATUS_NAMES.items():
        assert lib.gptq_status_string(code).decode() == name


def test_workspace_size_rules(lib):
    from post_weight_quantization_26_b200 import gptq as G
    cfg = G.make_config(bits=4, group_size=0, block=128)
    n = lib.gptq_workspace_size(4096, 4096, ctypes.byref(cfg))
    # the fp64 factorization buffer dominates: d*d*8 bytes plus leaf inverses
    assert n >= 4096 * 4096 * 8
    assert n % 256 == 0
    for bad in (G.make_config(bits=9), G.make_config(bits=1),
                G.make_config(block=96), G.make_config(group_size=48),
                G.make_config(group_size=96, block=128),
                G.make_config(damp_rel=-1.0), G.GptqConfig(4, 0, 2, 128, 0.01)):
        assert lib.gptq_workspace_size(256, 256, ctypes.byref(bad)) == 0
    assert lib.gptq_workspace_size(256, 250, ctypes.byref(cfg)) == 0  # d_col % 32
    assert lib.gptq_workspace_size(0, 256, ctypes.byref(cfg)) == 0
    g256 = G.make_config(group_size=256, block=128)
    assert lib.gptq_workspace_size(64, 512, ctypes.byref(g256)) > 0
    assert lib.gptq_workspace_size(64, 384, ctypes.byref(g256)) == 0  # group must divide


@pytest.mark.parametrize("name", ["gptq_hessian_accumulate", "gptq_hessian_accumulate_ordered"])
def test_hessian_accumulate_validation(lib, name):
    f = getattr(lib, name)
    assert f(None, FAKE, 16, 64, 64, 2.0, None) == 1
    assert f(FAKE, None, 16, 64, 64, 2.0, None) == 1
    assert f(FAKE, None, 0, 64, 64, 2.0, None) == 0    # empty chunk, no data
    assert f(FAKE, FAKE, 16, 60, 64, 2.0, None) == 1   # d % 8
    assert f(FAKE, FAKE, 16, 64, 60, 2.0, None) == 1   # ldx < d
    assert f(FAKE, FAKE, 16, 64, 68, 2.0, None) == 1   # ldx % 8
    assert f(FAKE, FAKE, -1, 64, 64, 2.0, None) == 1   # n < 0
    assert f(FAKE, FAKE, 16, 64, 64, float("nan"), None) == 1
    assert f(FAKE, ctypes.c_void_p(0x7F0000000002), 16, 64, 64, 2.0, None) == 1  # alignment
    assert f(FAKE, FAKE, 0, 64, 64, 2.0, None) == 0    # n == 0 is a no-op
    assert f(FAKE, FAKE, (1 << 31) - 64, 64, 64, 2.0, None) == 1  # a chunk past 2^31 tokens


def test_fault_inject_validation(lib):
    """Only the documented switches and limits are accepted; normal
    operation is restored by (NONE, 0)."""
    from post_weight_quantization_26_b200 import gptq as G
    f = lib.gptq_fault_inject
    assert f(3, 0) == 1 and f(-1, 0) == 1                 # unknown switch
    assert f(G.FAULT_SYRK_STALL, 999_999) == 1            # limit below 1 ms
    assert f(G.FAULT_SYRK_STALL, 10_000_000_001) == 1     # limit above 10 s
    assert f(G.FAULT_TRAILING_STALL, 20_000_000) == 0
    assert f(G.FAULT_NONE, 0) == 0


def test_prepare_and_quantize_validation(lib):
    from post_weight_quantization_26_b200 import gptq as G
    piv = ctypes.c_int64(123)
    assert lib.gptq_prepare_hinv(FAKE, 60, 0.01, FAKE, FAKE, FAKE, 1 << 30,
                                 ctypes.byref(piv), None) == 1
    assert piv.value == -1
    assert lib.gptq_prepare_hinv(FAKE, 64, 0.01, FAKE, FAKE, None, 1 << 30,
                                 None, None) == 4
    assert lib.gptq_prepare_hinv(FAKE, 64, 0.01, FAKE, FAKE, FAKE, 16,
                                 None, None) == 4
    assert lib.gptq_prepare_hinv(FAKE, 64, -0.5, FAKE, FAKE, FAKE, 1 << 30,
                                 None, None) == 1
    cfg = G.make_config()
    q = lib.gptq_quantize_layer
    assert q(FAKE, 64, 100, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
             FAKE, 1 << 30, None) == 1
    bad = G.make_config(bits=9)
    assert q(FAKE, 64, 128, FAKE, None, ctypes.byref(bad), FAKE, FAKE, FAKE,
             FAKE, 1 << 30, None) == 1
    assert q(FAKE, 64, 128, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
             FAKE, 8, None) == 4
    assert q(FAKE, 64, 128, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
             ctypes.c_void_p(0x7F0000000010), 1 << 30, None) == 4  # ws alignment
    assert lib.gptq_dequant_check(FAKE, FAKE, FAKE, None, None, 64, 128,
                                  ctypes.byref(cfg), None,
                                  ctypes.byref(ctypes.c_double()), FAKE,
                                  1 << 20, None) == 1


def test_factor_route_validation(lib):
    """The factor route's calls take the same arguments and checks as the
    inverse route's, and the sweep also rejects what F cannot serve: a block
    other than 128 and a group size that does not divide 128."""
    from post_weight_quantization_26_b200 import gptq as G
    piv = ctypes.c_int64(123)
    p = lib.gptq_prepare_factor
    assert p(FAKE, 60, 0.01, FAKE, FAKE, FAKE, 1 << 30, ctypes.byref(piv), None) == 1
    assert piv.value == -1
    assert p(FAKE, 64, 0.01, FAKE, FAKE, None, 1 << 30, None, None) == 4
    assert p(FAKE, 64, float("nan"), FAKE, FAKE, FAKE, 1 << 30, None, None) == 1
    q = lib.gptq_quantize_layer_factor
    for block, group in ((64, 0), (32, 32), (128, 256)):
        cfg = G.make_config(group_size=group, block=block)
        assert q(FAKE, 64, 512, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
                 FAKE, 1 << 30, None) == 1, (block, group)
    cfg = G.make_config(group_size=32)
    assert q(FAKE, 64, 100, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
             FAKE, 1 << 30, None) == 1
    assert q(FAKE, 64, 512, FAKE, None, ctypes.byref(cfg), FAKE, FAKE, FAKE,
             FAKE, 8, None) == 4


def test_w4a16_matmul_validation(lib):
    """Rejected before any launch: other widths, batches, shapes, alignment."""
    from post_weight_quantization_26_b200 import gptq as G
    f = lib.gptq_w4a16_matmul
    cfg4, cfg3 = G.make_config(bits=4), G.make_config(bits=3)
    ok = (FAKE, FAKE, FAKE, 64, 256)
    assert f(*ok, ctypes.byref(cfg3), FAKE, 1, FAKE, None) == 1   # width 3
    assert f(*ok, ctypes.byref(cfg4), FAKE, 0, FAKE, None) == 1   # batch 0
    assert f(*ok, ctypes.byref(cfg4), FAKE, 9, FAKE, None) == 1   # batch 9
    assert f(FAKE, FAKE, FAKE, 64, 48, ctypes.byref(cfg4), FAKE, 1, FAKE,
             None) == 1                                            # d_col % 32
    assert f(FAKE, FAKE, FAKE, 0, 256, ctypes.byref(cfg4), FAKE, 1, FAKE,
             None) == 1                                            # no rows
    assert f(*ok, ctypes.byref(cfg4), ctypes.c_void_p(0x7F0000000008), 1,
             FAKE, None) == 1                                      # X alignment
    assert f(ctypes.c_void_p(0x7F0000000004), FAKE, FAKE, 64, 256,
             ctypes.byref(cfg4), FAKE, 1, FAKE, None) == 1         # words alignment
    assert f(*ok, ctypes.byref(cfg4), None, 1, FAKE, None) == 1   # null X
    g100 = G.make_config(bits=4, group_size=100)
    assert f(*ok, ctypes.byref(g100), FAKE, 1, FAKE, None) == 1   # group % 32


def test_awq_validation(lib):
    """The AWQ entry points reject bad sizes, configurations and pointers
    before anything is launched."""
    from post_weight_quantization_26_b200 import gptq as G
    g128, bad3, sym = G.make_config(bits=4, group_size=128), G.make_config(bits=3), \
        G.make_config(bits=4, sym=True)
    wsz = lib.gptq_awq_workspace_size
    assert wsz(64, 256, ctypes.byref(g128)) >= 2 * 256 * 256 * 4 + 3 * 64 * 256 * 4
    assert wsz(64, 256, ctypes.byref(bad3)) == 0          # AWQ is 4-bit only
    assert wsz(64, 256, ctypes.byref(sym)) == 0           # asymmetric quantizer
    assert wsz(64, 48, ctypes.byref(G.make_config(bits=4))) == 0  # d_col % 32
    assert wsz(1 << 16, 1 << 15, ctypes.byref(g128)) == 0            # 2^31 weights
    cs = lib.gptq_awq_channel_scale
    assert cs(FAKE, 0, 64, 64, FAKE, None) == 1            # no tokens
    assert cs(FAKE, 16, 12, 16, FAKE, None) == 1           # d % 8
    assert cs(FAKE, 16, 64, 60, FAKE, None) == 1           # ldx < d
    assert cs(ctypes.c_void_p(0x7F0000000008), 16, 64, 64, FAKE, None) == 1  # alignment
    sr = lib.gptq_awq_search
    args = [FAKE, FAKE, FAKE, 64, 256, ctypes.byref(g128)]
    out = [FAKE] * 6
    assert sr(*args, 1, *out, FAKE, 1 << 30, None) == 1    # n_grid < 2
    assert sr(*args, 65, *out, FAKE, 1 << 30, None) == 1   # n_grid > 64
    assert sr(*args, 20, *out, FAKE, 16, None) == 4        # short workspace
    assert sr(*args, 20, *out, ctypes.c_void_p(0x7F0000000010), 1 << 30, None) == 4
    assert sr(FAKE, FAKE, FAKE, 64, 256, ctypes.byref(bad3), 20, *out, FAKE, 1 << 30,
              None) == 1


def test_product_path_has_no_fallback():
    """The binding refuses to run without its library (no CPU path)."""
    from post_weight_quantization_26_b200 import gptq as G
    saved = G._lib
    G._lib = None
    try:
        with pytest.raises(RuntimeError, match="not found"):
            G.load_library("/nonexistent/libgptq.so")
    finally:
        G._lib = saved


def test_package_does_not_import_oracle():
    """The product package never imports the CPU oracle."""
    pkg = os.path.join(ROOT, "post_weight_quantization_26_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
