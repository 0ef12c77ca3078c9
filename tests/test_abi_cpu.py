"""CPU checks of the C ABI boundary: the library loads without a GPU and
exports every entry point include/moesq.h declares; host-only helpers
answer without touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moesq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moesq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from grouped_gemm_moesq_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for need in ("moesq_pack_weights", "moesq_quantize_act", "moesq_route_permute",
                 "moesq_grouped_sparse_gemm", "moesq_moe_layer"):
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_declares_every_symbol():
    import grouped_gemm_moesq_b200 as m
    L = m.load()
    for n in declared_functions():
        assert getattr(L, n).restype is not None or n == "moesq_set_wait_timeout_ns"


def test_host_only_helpers(lib):
    import grouped_gemm_moesq_b200 as m
    m.load()
    # Eq. 7 storage: values K/4 + mask K/16 + scales K/32 per row, plus kernel form
    per = (ctypes.c_size_t * 5)()
    m.load().moesq_weights_bytes(384, 4096, 7168, per)
    assert per[0] == 384 * 4096 * 7168 // 4 and per[1] == per[0] // 4 and per[2] == per[0] // 8
    assert per[0] + per[1] + per[2] == 11 * 384 * 4096 * 7168 // 32
    assert per[4] == per[0] + per[1] + per[2]          # kernel form: the same bytes, tiled
    assert m.moesq_rows_capacity(1, 8, 384) == 1024
    assert m.moesq_rows_capacity(8192, 8, 384) % 128 == 0
    assert m.moesq_rows_capacity(8192, 8, 384) >= 8192 * 8 + 127 * 384
    assert m.load().moesq_status_str(2) == b"unsupported shape"
    assert m.moesq_version().startswith("moesq")
    assert m.moesq_layer_workspace_bytes(16, 8, 384, 7168, 2048) > 0


def test_no_cpu_fallback_in_product_path():
    """The package never imports the oracle and never computes on the host."""
    pkg = os.path.join(ROOT, "grouped_gemm_moesq_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn
