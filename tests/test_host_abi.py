"""Host-side checks of the C-ABI library (CPU only: no compute call needs a
device here). The library loads without a GPU and exports every function
include/csa2.h declares; host logic (plan, argument validation, workspace
layout, status strings) behaves as documented."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT, golden

HEADER = os.path.join(ROOT, "include", "csa2.h")


@pytest.fixture(scope="module")
def lib():
    from compressed_sparse_attention_quant_b200 import _build
    _build.build()
    from compressed_sparse_attention_quant_b200 import lib as L
    return L


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("csa2_quant_kv_fp4", "csa2_indexer_topk", "csa2_sparse_attn_decode", "csa2_plan"):
        assert required in names
    src = open(HEADER).read()
    assert "CSA2_FULL = 0" in src and "CSA2_REINDEX = 1" in src and "CSA2_REUSE = 2" in src


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    so = ctypes.CDLL(lib.library_path())
    for n in names:
        assert hasattr(so, n), f"{n} not exported"
    assert set(names) == set(lib.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", lib.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (csa2_\w+)", out))
    assert set(names) <= exported


def test_library_does_not_link_the_oracle(lib):
    out = subprocess.run(["nm", "-D", lib.library_path()], capture_output=True, text=True).stdout
    assert "orc_" not in out
    deps = subprocess.run(["ldd", lib.library_path()], capture_output=True, text=True).stdout
    assert "liboracle" not in deps and "libtorch" not in deps


def test_plan_through_abi_matches_golden(lib):
    with open(golden("mode_plans.txt")) as f:
        rows = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for row in rows:
        parts = [p.strip() for p in row.split("|")]
        modes = parts[0].split()
        if parts[1] == "error":
            with pytest.raises(lib.Csa2Error) as e:
                lib.plan(modes)
            assert e.value.status == 4                   # CSA2_ERR_BAD_PLAN
            continue
        own, src = lib.plan(modes)
        assert own == [int(x) for x in parts[1].split()]
        assert src == [int(x) for x in parts[2].split()]


def test_status_strings(lib):
    for code, name in lib.STATUS.items():
        assert lib.status_string(code) == name


def test_unsupported_shapes_rejected_on_host(lib):
    L = lib._L
    cache = lib._Cache(1, 1, 1, 1, 4)
    # wrong channel count, wrong indexer shape, wrong head count / window
    assert L.csa2_quant_kv_fp4(16, 4, 512, 16, None, None, ctypes.byref(cache), None) == 2
    assert L.csa2_indexer_topk(16, 16, 1, 1, 8, 64, ctypes.byref(cache), 16, 1, 16, 4, 16, 256, 1 << 20,
                               None) == 2
    assert L.csa2_sparse_attn_decode(16, 1, 1, 8, 576, ctypes.byref(cache), 16, 1, 16, 16, 4, 16, 128, 0.1,
                                     16, 16, 256, 1 << 20, None) == 2
    assert L.csa2_sparse_attn_decode(16, 1, 1, 16, 576, ctypes.byref(cache), 16, 1, 16, 16, 4, 16, 64, 0.1,
                                     16, 16, 256, 1 << 20, None) == 2
    # null pointers / negative sizes
    assert L.csa2_quant_kv_fp4(None, 4, 576, 16, None, None, ctypes.byref(cache), None) == 1
    assert L.csa2_quant_kv_fp4(16, -1, 576, 16, None, None, ctypes.byref(cache), None) == 1
    assert L.csa2_quant_kv_fp4(16, 4, 576, 16, None, None, None, None) == 1
    assert L.csa2_plan(None, 3, None, None) == 1
    # indexer FP8 quantiser: 64 channels only; null / negative; 16-byte alignment; empty is a no-op
    assert L.csa2_quant_indexer_fp8(16, 4, 128, 16, 16, None) == 2
    assert L.csa2_quant_indexer_fp8(None, 4, 64, 16, 16, None) == 1
    assert L.csa2_quant_indexer_fp8(16, -1, 64, 16, 16, None) == 1
    assert L.csa2_quant_indexer_fp8(24, 4, 64, 16, 16, None) == 8
    assert L.csa2_quant_indexer_fp8(16, 4, 64, 24, 16, None) == 8
    assert L.csa2_quant_indexer_fp8(16, 0, 64, None, None, None) == 0
    # candidate-pool top-k: indexer shape, pool size limit, bad sizes, null pointers
    assert L.csa2_indexer_pool_topk(16, 16, 1, 1, 8, 64, ctypes.byref(cache), 16, 1, 16, 16, 64, 8, 16, None) == 2
    assert L.csa2_indexer_pool_topk(16, 16, 1, 1, 4, 64, ctypes.byref(cache), 16, 1, 16, 16, 40000, 8, 16,
                                    None) == 2
    assert L.csa2_indexer_pool_topk(16, 16, 1, 1, 4, 64, ctypes.byref(cache), 16, 1, 16, 16, 64, 0, 16, None) == 1
    assert L.csa2_indexer_pool_topk(16, 16, 1, 1, 4, 64, ctypes.byref(cache), 16, 1, 16, 16, 0, 8, 16, None) == 1
    assert L.csa2_indexer_pool_topk(16, 16, 1, 1, 4, 64, ctypes.byref(cache), 16, 1, 16, None, 64, 8, 16,
                                    None) == 1
    assert lib.launch_count() == 0


def test_indexer_workspace_layout(lib):
    a = lib.indexer_topk_workspace_bytes(64, 1, 2048, 2048)
    # scores alone: 64 rows x 131072 positions x 4 B
    assert a >= 64 * 131072 * 4 and a % 256 == 0
    assert lib.indexer_topk_workspace_bytes(64, 2, 2048, 2048) > a
    assert lib.indexer_topk_workspace_bytes(0, 1, 1, 1) == 0
