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
                               ctypes.c_float(0.1), fake, 0, None, ws, 256, None) == -1
    assert lib.csa_sparse_attn(fake, fake, fake, fake, fake, fake, 8, 0, 8, 48, 128, 16, 64,
                               ctypes.c_float(0.1), fake, 0, None, ws, 256, None) == -3
    assert lib.hca_attn(fake, fake, fake, fake, fake, 8, 0, 8, 64, 128, 0, 64, ctypes.c_float(0.1), fake, 0, None,
                        ws, 256, None) == -1
    # output element type other than CSA_BF16 (0) / CSA_F32 (1)
    assert lib.csa_sparse_attn(fake, fake, fake, fake, fake, fake, 8, 0, 8, 64, 128, 16, 64,
                               ctypes.c_float(0.1), fake, 2, None, ws, 256, None) == -1
    assert lib.hca_attn(fake, fake, fake, fake, fake, 8, 0, 8, 64, 128, 4, 64, ctypes.c_float(0.1), fake, -1, None,
                        ws, 256, None) == -1
    # selected-entry tiles of one block beyond the list: H = 4 gives 32 tokens x 16 tiles at k = 2048
    assert lib.csa_sparse_attn(fake, fake, fake, fake, fake, fake, 8, 0, 8, 4, 128, 2048, 64,
                               ctypes.c_float(0.1), fake, 0, None, ws, 256, None) == -3
    # decode: workspace smaller than required
    need = lib.csa_decode_workspace_bytes(4, 1024, 64, 128, 16, 128, 64, 32)
    assert need > 256
    pos = (ctypes.c_int64 * 4)(10, 20, 30, 40)
    assert lib.csa_decode(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, pos, 4, 1024, 64, 128, 16, 128,
                          4, 64, 32, ctypes.c_float(0.1), fake, 0, None, None, None, ws, 256, None) == -5


def test_zero_sized_calls_are_no_ops(lib):
    fake = ctypes.c_void_p(0x1000)
    assert lib.csa_compress(fake, fake, fake, fake, 0, 128, 4, fake, fake, None) == 0
    assert lib.csa_indexer_topk(fake, fake, fake, fake, fake, 0, 0, 0, 16, 128, 4, 8, fake, None, fake, 256,
                                None) == 0


def _align256(x):
    return (x + 255) // 256 * 256


def _decode_workspace(B, Ncap, H, d, k, W):
    """The decode workspace layout: a 256-byte status header, positions [B] i64,
    the merged selection [B,k] i32, each key range's candidate keys [B,ns,k] u64
    and counts [B,ns] i32, and split-attention partials [B,nsa,H,d] f32 + [B,nsa,H]
    f32 when a sequence's attention is split.  ns: key ranges per sequence (one
    wave of one-CTA-per-SM blocks, at most one per 128-key tile, at most what one
    finalize block merges, at most 63); nsa: attention splits (one wave, at most
    16, at most one per key tile)."""
    ns = max(1, min(148 // B, -(-Ncap // 128), 256 * 40 // k, 63))
    tiles = -(-k // 128) + (-(-W // 128) if W > 0 else 0)
    nsa = max(1, min(148 // B, 16, tiles))
    part = _align256(B * nsa * H * d * 4) + _align256(B * nsa * H * 4) if nsa > 1 else 0
    return 256 + _align256(B * 8) + _align256(B * k * 4) + _align256(B * ns * k * 8) + _align256(B * ns * 4) + part


@pytest.mark.parametrize("B,Ncap,k,W", [
    (16, 262144, 1024, 128),   # the 1M-context decode: 9 key ranges per sequence
    (1, 65536, 1024, 128),     # one sequence: the merge limit (10 ranges at k = 1024)
    (1, 32768, 64, 128),       # one sequence, small k: the 63-range limit
    (4, 1024, 64, 32),         # short cache: one range per 128-key tile
    (64, 262144, 512, 0),      # many sequences, no window
])
def test_decode_workspace_follows_the_split_rule(lib, B, Ncap, k, W):
    H, d = 64, 128
    got = lib.csa_decode_workspace_bytes(B, Ncap, H, d, 16, 128, k, W)
    assert got == _decode_workspace(B, Ncap, H, d, k, W)


def test_debug_inject_rejects_unknown_codes(lib):
    assert lib.csa_debug_inject(99) == -1
    assert lib.csa_debug_inject(0) == 0
