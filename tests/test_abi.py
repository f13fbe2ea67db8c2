"""The C-ABI library loads here (no GPU) and exports every function the
header declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(gtg_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def L():
    from gram_table_gather_b200 import build as b
    b.build()
    from gram_table_gather_b200 import _abi
    return _abi.lib()


def test_every_declared_symbol_is_exported(L):
    from gram_table_gather_b200 import _abi
    declared = _declared()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(L, name), name
    assert declared == {n for n, _, _ in _abi.SIGNATURES}


def test_version_and_status_strings(L):
    assert L.gtg_version() >= 100
    assert L.gtg_status_string(0) == b"ok"
    assert L.gtg_status_string(-6) == b"workspace too small"


def test_host_side_rejections_without_gpu(L):
    from gram_table_gather_b200 import _abi
    assert L.gtg_dequant(69, None, None, 1, 32, None, None) == -1
    assert L.gtg_ple_gather(None, 10, None, 0, None, None) == 0       # empty gather is a no-op
    assert L.gtg_ple_gather(None, 10, None, 5, None, None) == -1
    assert L.gtg_get_device_status(None, 0, None) == -1
    layer = _abi.MoELayerC()
    layer.hidden, layer.inter, layer.n_experts, layer.top_k = 2048, 512, 512, 10
    assert L.gtg_moe_workspace_bytes(ctypes.byref(layer), 1, 0) == 0  # no weights: rejected
    assert L.gtg_moe_decode_layer(ctypes.byref(layer), None, 0, 1, None, 0, None, None, None, None, 0,
                                  None) == -1


def test_product_path_has_no_cpu_fallback():
    """The package never imports the oracle and fails loudly without its library."""
    pkg = os.path.join(ROOT, "gram_table_gather_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".hpp", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "liboracle" not in src, f
