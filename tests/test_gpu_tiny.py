"""GPU parity on the tiny CSA+HCA workload (T=1024, 4 heads x 64, CSA m=4 k=16
W=64, HCA m'=64, indexer 4 x 64 MXFP4): every output element against the oracle.

Method: blog.nickys.cn/?p=150 sections "1. CSA" and "2. HCA"; indexer on FP4:
ifanr repost, attention section.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import (assert_attention_close, assert_topk_exact, assert_within_bf16_ulp, fp32_pool_slack,
                          from_words, words)

pytestmark = pytest.mark.gpu

WL = inputs.TINY


@pytest.fixture(scope="module")
def lib():
    import long_context_compressed_gated_b200 as csa
    csa.lib()
    return csa


@pytest.fixture(scope="module")
def data():
    return inputs.prefill_layer(WL)


def _cuda(d):
    return {k: v.cuda() for k, v in d.items()}


def test_compress_csa_and_hca(lib, data):
    g = _cuda(data)
    for m, B in ((WL.m, "B"), (WL.m_hca, "B_hca")):
        Kc, Vc = lib.csa_compress(g["K"], g["V"], g["Z"], g[B], m)
        torch.cuda.synchronize()
        Kx, Vx = oracle.compress(data["K"], data["V"], data["Z"], data[B], m)
        assert_within_bf16_ulp(Kc, Kx, "Kc m=%d" % m, fp32_pool_slack(data["K"], m, data["Z"], data[B]))
        assert_within_bf16_ulp(Vc, Vx, "Vc m=%d" % m, fp32_pool_slack(data["V"], m, data["Z"], data[B]))


def test_indexer_topk_exact(lib, data):
    g = _cuda(data)
    idx, scores, ws = lib.csa_indexer_topk(g["qI_codes"], g["qI_scales"], g["w_codes"], g["kI_codes"],
                                           g["kI_scales"], WL.m, WL.k)
    assert lib.csa_check_status(ws) == 0
    I = oracle.indexer(data["qI_codes"], data["qI_scales"], data["w_codes"], data["kI_codes"], data["kI_scales"], 0,
                       WL.m)
    want_idx, want_top = oracle.topk(I, oracle.n_vis(np.arange(WL.T), WL.m), WL.k)
    assert_topk_exact(idx, scores, want_idx, want_top, "tiny indexer")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_sparse_attention_against_oracle(lib, data, out_dtype):
    scale = 1.0 / math.sqrt(WL.d)
    Kc64, Vc64 = oracle.compress(data["K"], data["V"], data["Z"], data["B"], WL.m)
    Kcw, Vcw = oracle.to_bf16_words(Kc64), oracle.to_bf16_words(Vc64)
    I = oracle.indexer(data["qI_codes"], data["qI_scales"], data["w_codes"], data["kI_codes"], data["kI_scales"], 0,
                       WL.m)
    sel, _ = oracle.topk(I, oracle.n_vis(np.arange(WL.T), WL.m), WL.k)
    O_want, lse_want = oracle.attention(data["Q"], Kcw, Vcw, data["K"], data["V"], 0, WL.m, WL.W, scale, sel=sel)
    g = _cuda(data)
    O, lse, ws = lib.csa_sparse_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"),
                                     torch.from_numpy(sel).cuda(), g["K"], g["V"], WL.W, scale, out_dtype=out_dtype)
    assert lib.csa_check_status(ws) == 0
    assert O.dtype == out_dtype
    assert_attention_close(O, O_want, "tiny CSA attention")
    np.testing.assert_allclose(lse.cpu().numpy(), lse_want, atol=2e-3)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_hca_attention_against_oracle(lib, data, out_dtype):
    scale = 1.0 / math.sqrt(WL.d)
    Kc64, Vc64 = oracle.compress(data["K"], data["V"], data["Z"], data["B_hca"], WL.m_hca)
    Kcw, Vcw = oracle.to_bf16_words(Kc64), oracle.to_bf16_words(Vc64)
    O_want, lse_want = oracle.attention(data["Q"], Kcw, Vcw, data["K"], data["V"], 0, WL.m_hca, WL.W_hca, scale)
    g = _cuda(data)
    O, lse, ws = lib.hca_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"), g["K"], g["V"], WL.m_hca,
                              WL.W_hca, scale, out_dtype=out_dtype)
    assert lib.csa_check_status(ws) == 0
    assert O.dtype == out_dtype
    assert_attention_close(O, O_want, "tiny HCA attention")
    np.testing.assert_allclose(lse.cpu().numpy(), lse_want, atol=2e-3)


def test_end_to_end_gpu_pipeline(lib, data):
    """GPU compress -> GPU indexer -> GPU attention against the oracle's own chain."""
    scale = 1.0 / math.sqrt(WL.d)
    g = _cuda(data)
    Kc, Vc = lib.csa_compress(g["K"], g["V"], g["Z"], g["B"], WL.m)
    idx, _, _ = lib.csa_indexer_topk(g["qI_codes"], g["qI_scales"], g["w_codes"], g["kI_codes"], g["kI_scales"],
                                     WL.m, WL.k)
    O, _, _ = lib.csa_sparse_attn(g["Q"], Kc, Vc, idx, g["K"], g["V"], WL.W, scale)
    ref = oracle.csa_layer(data, WL.m, WL.k, WL.W, scale)
    assert_attention_close(O, ref["O"], "tiny CSA end to end")
