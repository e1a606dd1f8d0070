"""The C ABI without a GPU: libcsa.so loads, exports every function include/csa.h
declares, and rejects invalid arguments on the host before anything reaches
the device (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(?:int|size_t|const char\*)\s+(\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import long_context_compressed_gated_b200 as csa
    from long_context_compressed_gated_b200 import build
    build.build()
    return csa.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["csa_compress", "csa_indexer_topk", "csa_sparse_attn", "hca_attn", "csa_decode", "hca_decode",
              "csa_status_string", "csa_check_status"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(0, -8, -1):
        s = lib.csa_status_string(code)
        assert s and s != b"unknown status"
    assert lib.csa_status_string(-99) == b"unknown status"


def test_host_side_validation_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)        # 16-byte aligned, never dereferenced: validation fails first
    odd = P(0x1001)
    # unsupported head dim
    assert lib.csa_compress(fake, fake, fake, fake, 64, 96, 4, fake, fake, None) == -3
    # negative T
    assert lib.csa_compress(fake, fake, fake, fake, -1, 128, 4, fake, fake, None) == -1
    # misaligned pointer
    assert lib.csa_compress(odd, fake, fake, fake, 64, 128, 4, fake, fake, None) == -2
    # null pointer
    assert lib.csa_compress(None, fake, fake, fake, 64, 128, 4, fake, fake, None) == -1
    # indexer: k out of range, bad head count, missing workspace
    ws = P(0x2000)
    assert lib.csa_indexer_topk(fake, fake, fake, fake, fake, 8, 0, 8, 16, 128, 4, 0, fake, None, ws, 256,
                                None) == -1
    assert lib.csa_indexer_topk(fake, fake, fake, fake, fake, 8, 0, 8, 12, 128, 4, 8, fake, None, ws, 256,
                                None) == -3
    assert lib.csa_indexer_topk(fake, fake, fake, fake, fake, 8, 0, 8, 16, 128, 4, 8, fake, None, None, 0,
                                None) == -5
    # attention: window too large, bad H
    assert lib.csa_sparse_attn(fake, fake, fake, fake, fake, fake, 8, 0, 8, 64, 128, 16, 5000,
                               ctypes.c_float(0.1), fake, None, ws, 256, None) == -1
    assert lib.csa_sparse_attn(fake, fake, fake, fake, fake, fake, 8, 0, 8, 48, 128, 16, 64,
                               ctypes.c_float(0.1), fake, None, ws, 256, None) == -3
    assert lib.hca_attn(fake, fake, fake, fake, fake, 8, 0, 8, 64, 128, 0, 64, ctypes.c_float(0.1), fake, None,
                        ws, 256, None) == -1
    # decode: workspace smaller than required
    need = lib.csa_decode_workspace_bytes(4, 1024, 64, 128, 16, 128, 64, 32)
    assert need > 256
    pos = (ctypes.c_int64 * 4)(10, 20, 30, 40)
    assert lib.csa_decode(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, pos, 4, 1024, 64, 128, 16, 128,
                          4, 64, 32, ctypes.c_float(0.1), fake, None, None, None, ws, 256, None) == -5


def test_zero_sized_calls_are_no_ops(lib):
    fake = ctypes.c_void_p(0x1000)
    assert lib.csa_compress(fake, fake, fake, fake, 0, 128, 4, fake, fake, None) == 0
    assert lib.csa_indexer_topk(fake, fake, fake, fake, fake, 0, 0, 0, 16, 128, 4, 8, fake, None, fake, 256,
                                None) == 0
