"""The C-ABI library builds for sm_100a, loads without a GPU, and exports
every symbol include/dsa.h declares; host-only calls work (no compute)."""
import os
import re

import pytest

import dynamic_sparse_attention_03_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(\w+)\s*\(", text, flags=re.M)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(dsa.SYMBOLS)


def test_library_exports_every_declared_symbol():
    from dynamic_sparse_attention_03_b200 import build
    build.build()
    lib = dsa.load_library()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.dsa_version().startswith(b"dsa")


@pytest.mark.parametrize("n,kf,rho,want", [(1024, 4, 0.0, 4), (32768, 0, 0.10, 54), (131072, 0, 0.10, 207),
                                            (1048576, 0, 0.02, 330)])
def test_capacity_query_matches_oracle(n, kf, rho, want):
    import oracle
    assert oracle.max_blocks_per_row(n // 64, kf, rho) == want
    assert dsa.block_index_capacity(n, kf, rho) == want


def test_capacity_query_rejects_bad_args():
    with pytest.raises(dsa.DSAError):
        dsa.block_index_capacity(1000, 0, 0.1)
    with pytest.raises(dsa.DSAError):
        dsa.block_index_capacity(1024, 4, 0.1)


def test_workspace_size_queries_launch_nothing():
    """ws == NULL returns the size without touching the GPU (works on a CPU machine)."""
    import ctypes
    lib = dsa.load_library()
    size = ctypes.c_size_t(0)
    q = ctypes.c_void_p(0x1000)   # never dereferenced in a size query
    rc = lib.sparse_index_estimate(q, q, 32, 8, 32768, 128, 64, 0, ctypes.c_float(0.1), q, q, 54, None, None,
                                   ctypes.byref(size), None)
    assert rc == 0 and size.value > 32 * 512 * 128 * 4
    rc = lib.block_sparse_attn_fwd(q, q, q, q, 32, 8, 32768, 128, ctypes.c_float(0.088), q, q, 54, None, None, 0,
                                   None, None, ctypes.byref(size), None)
    assert rc == 0 and size.value == 256
    rc = lib.sparse_decode_attn(q, q, q, q, 16, 32, 8, 131072, 128, 512, 1, ctypes.c_float(0.088), q, None, None, 0,
                                None, ctypes.byref(size), None)
    assert rc == 0 and size.value > 0
    # bad shapes are rejected before any launch
    rc = lib.block_sparse_attn_fwd(q, q, q, q, 32, 8, 1000, 128, ctypes.c_float(0.088), q, q, 54, None, None, 0,
                                   None, None, ctypes.byref(size), None)
    assert rc == -2
