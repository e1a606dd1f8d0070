"""csa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (serving loops that forbid allocator calls once running,
embedders that own every buffer).  It keeps its scratch in a static device
array inside the library.  Checked through the C ABI against csa_decode with a
caller workspace, on two calls in a row (the shared scratch keeps the previous
call's contents), and checked to leave torch's allocator untouched.  This file
sorts last so that a run stopping at the first failure has already run every
other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

from long_context_compressed_gated_b200 import inputs
from tests.parity import assert_attention_close

pytestmark = pytest.mark.gpu


def _lib():
    import long_context_compressed_gated_b200 as csa
    L = csa.lib()
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    L.csa_decode_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I64, I, I, I, I, I, I, I, F, P, P, P, P, P,
                                     P]
    L.csa_decode_noalloc.restype = I
    return csa, L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_decode_twice():
    csa, L = _lib()
    wl = inputs.Workload("noalloc", H=64, d=128, m=4, k=1024, W=128, HI=16, dI=128, batch=4, context=1 << 18,
                         seed=31)
    g = {k: v.cuda() for k, v in inputs.decode_batch(wl).items()}
    scale = 1.0 / math.sqrt(wl.d)
    pos = [wl.context - 1, 100000, 5000, 3]
    O_ref, lse_ref, idx_ref, sc_ref, ws = csa.csa_decode(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"],
                                                         g["Kc"], g["Vc"], g["kI_codes"], g["kI_scales"], g["Kwin"],
                                                         g["Vwin"], pos, wl.m, wl.k, scale)
    assert csa.csa_check_status(ws) == 0
    B, H, d = g["q"].shape
    posa = (ctypes.c_int64 * B)(*pos)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        sc = torch.full_like(sc_ref, float("nan"))
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        allocated = torch.cuda.memory_allocated()
        rc = L.csa_decode_noalloc(_p(g["q"]), _p(g["qI_codes"]), _p(g["qI_scales"]), _p(g["w_codes"]), _p(g["Kc"]),
                                  _p(g["Vc"]), _p(g["kI_codes"]), _p(g["kI_scales"]), _p(g["Kwin"]), _p(g["Vwin"]),
                                  posa, B, g["Kc"].shape[1], H, d, wl.HI, wl.dI, wl.m, wl.k, wl.W, scale, _p(O),
                                  _p(lse), _p(idx), _p(sc), _p(status), stream)
        assert rc == 0, csa.csa_status_string(rc)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == allocated  # nothing went through torch's allocator
        assert int(status.item()) == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref.cpu().numpy())
        np.testing.assert_array_equal(sc.cpu().numpy(), sc_ref.cpu().numpy())
        assert_attention_close(O, O_ref.float().cpu().double().numpy(), "noalloc decode call %d" % call)
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), atol=2e-3)


@pytest.mark.parametrize("B,H,k", [
    (1024, 64, 2048),  # many sequences with a large k
    (16, 128, 1024),   # 128 heads: the split attention partials alone exceed the scratch
])
def test_noalloc_rejects_problems_beyond_its_scratch(B, H, k):
    csa, L = _lib()
    need = csa.lib().csa_decode_workspace_bytes(B, 1 << 18, H, 128, 16, 128, k, 128)
    assert need > (8 << 20)
    fake = ctypes.c_void_p(0x1000)
    posa = (ctypes.c_int64 * B)(*([(1 << 20) - 1] * B))
    rc = L.csa_decode_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, posa, B, 1 << 18, H,
                              128, 16, 128, 4, k, 128, 0.088, fake, None, None, None, None, None)
    assert rc == -5  # CSA_ERR_WORKSPACE
