"""The MXFP8 compressed cache (E4M3 codes + an E8M0 scale per 32 channels; the
raw window stays bf16): the GPU quantiser against the oracle bit for bit, and
decode over the FP8 cache.  Dequantised entries are exact bf16 values, so
csa_decode_fp8 must equal csa_decode over the dequantised cache bit for bit,
and the oracle over that cache within the attention tolerance.  KV cache in
mixed BF16/FP8 storage: ferris-liu.github.io ... deepseek-v4, engineering layer."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import assert_attention_close, assert_topk_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import long_context_compressed_gated_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("rows,n,seed", [(2000, 128, 1), (777, 64, 2)])
def test_mxfp8_quantize_bit_exact(csa, rows, n, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, n, generator=g) * torch.pow(2.0, torch.randint(-130, 120, (rows, n // 32),
                                                                         generator=g).float()).repeat_interleave(32, 1)
    x[0, :32] = 0.0
    x[1, 3] = float("inf")
    x[2, :32] = torch.tensor([448.0, 464.0, 480.0, 500.0, -1000.0, 0.001953125, 2.0 ** -12, -0.0] * 4)
    x = x.to(torch.bfloat16)
    codes, scales = csa.csa_mxfp8_quantize(x.cuda())
    torch.cuda.synchronize()
    c_want, s_want = oracle.mxfp8_quantize(x)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_want, err_msg="scales")
    np.testing.assert_array_equal(codes.cpu().numpy(), c_want, err_msg="codes")


def _dequant_bf16(codes, scales):
    v = oracle.mxfp8_dequantize(codes, scales)
    t = torch.from_numpy(v).to(torch.bfloat16)
    assert np.array_equal(t.double().numpy(), v)  # exact in bf16
    return t


@pytest.mark.parametrize("B,context,k,W", [(4, 1 << 18, 1024, 128), (3, 5000, 64, 32)])
def test_decode_over_the_fp8_cache(csa, B, context, k, W):
    wl = inputs.Workload("dec_fp8", H=64, d=128, m=4, k=k, W=W, HI=16, dI=128, batch=B, context=context, seed=71)
    g = {key: v.cuda() for key, v in inputs.decode_batch(wl).items()}
    scale = 1.0 / math.sqrt(wl.d)
    pos = [context - 1] + [max(0, context - 1 - 997 * b) for b in range(1, B)]
    Kq, Ks = csa.csa_mxfp8_quantize(g["Kc"])
    Vq, Vs = csa.csa_mxfp8_quantize(g["Vc"])
    O8, lse8, idx8, sc8, ws = csa.csa_decode_fp8(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"], Kq, Ks, Vq, Vs,
                                                  g["kI_codes"], g["kI_scales"], g["Kwin"], g["Vwin"], pos, wl.m, k,
                                                  scale, out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    Kd = _dequant_bf16(Kq.cpu(), Ks.cpu()).cuda()
    Vd = _dequant_bf16(Vq.cpu(), Vs.cpu()).cuda()
    O, lse, idx, sc, ws = csa.csa_decode(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"], Kd, Vd, g["kI_codes"],
                                         g["kI_scales"], g["Kwin"], g["Vwin"], pos, wl.m, k, scale,
                                         out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    assert torch.equal(idx8, idx) and torch.equal(sc8, sc)
    assert torch.equal(O8, O), "FP8 cache path differs from the bf16 path over the dequantised cache"
    for b in (0, B - 1):
        t = pos[b]
        I = oracle.indexer(g["qI_codes"][b:b + 1].cpu(), g["qI_scales"][b:b + 1].cpu(), g["w_codes"][b:b + 1].cpu(),
                           g["kI_codes"][b].cpu(), g["kI_scales"][b].cpu(), t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), k)
        assert_topk_exact(idx8[b:b + 1], sc8[b:b + 1], want_idx, want_top, "fp8 decode seq %d" % b)
        o, _ = oracle.attention(g["q"][b:b + 1].cpu(), Kd[b].cpu(), Vd[b].cpu(), g["Kwin"][b].cpu(),
                                g["Vwin"][b].cpu(), t, wl.m, wl.W, scale, sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
        assert_attention_close(O8[b:b + 1], o, "fp8 decode attention seq %d" % b)
