"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times, checked on sampled rows the oracle computes one by one.

CSA prefill T=32768 (64 x 128, m=4, k=512, W=128, indexer 64 x 128 MXFP4),
HCA prefill T=131072 (m'=128, W=128), CSA decode B=16 over a 1M-token context
(262144 entries, k=1024).  Method: blog.nickys.cn/?p=150 "1. CSA"/"2. HCA";
ifanr repost attention section (FP4 indexer, window branch).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import (assert_attention_close, assert_topk_exact, assert_within_bf16_ulp, fp32_pool_slack,
                          from_words, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import long_context_compressed_gated_b200 as m
    m.lib()
    return m


def _host(d, keys):
    return {k: d[k].cpu() for k in keys}


def test_csa_prefill_full_size_sampled(csa):
    wl = inputs.CSA_PREFILL
    g = inputs.prefill_layer(wl, device="cuda")
    scale = 1.0 / math.sqrt(wl.d)
    Kc, Vc = csa.csa_compress(g["K"], g["V"], g["Z"], g["B"], wl.m)
    idx, scores, ws = csa.csa_indexer_topk(g["qI_codes"], g["qI_scales"], g["w_codes"], g["kI_codes"],
                                           g["kI_scales"], wl.m, wl.k)
    assert csa.csa_check_status(ws) == 0
    h = _host(g, ["K", "V", "Z", "B", "qI_codes", "qI_scales", "w_codes", "kI_codes", "kI_scales"])
    special = [0, 1, 3, 4, 5, 127, 128, 2046, 2047, 2048, 2051, 4095, 8191, 16383, 16384, wl.T - 2, wl.T - 1]
    rows = sample_rows(wl.T, 24, special, seed=11)
    # compression of every block
    Kx, Vx = oracle.compress(h["K"], h["V"], h["Z"], h["B"], wl.m)
    assert_within_bf16_ulp(Kc, Kx, "Kc", fp32_pool_slack(h["K"], wl.m, h["Z"], h["B"]))
    assert_within_bf16_ulp(Vc, Vx, "Vc", fp32_pool_slack(h["V"], wl.m, h["Z"], h["B"]))
    # indexer + top-k on sampled rows
    I = oracle.indexer(h["qI_codes"], h["qI_scales"], h["w_codes"], h["kI_codes"], h["kI_scales"], 0, wl.m, rows)
    want_idx, want_top = oracle.topk(I, oracle.n_vis(rows, wl.m), wl.k)
    assert_topk_exact(idx[torch.from_numpy(rows).cuda()], scores[torch.from_numpy(rows).cuda()], want_idx, want_top,
                      "CSA prefill indexer (sampled rows)")
    # attention: oracle-produced compressed entries and selection fed to both sides
    Kcw, Vcw = oracle.to_bf16_words(Kx), oracle.to_bf16_words(Vx)
    sel_all = idx.clone()
    sel_all[torch.from_numpy(rows).cuda()] = torch.from_numpy(want_idx).cuda()
    O, lse, ws = csa.csa_sparse_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"), sel_all, g["K"],
                                     g["V"], wl.W, scale)
    assert csa.csa_check_status(ws) == 0
    Qs = g["Q"][torch.from_numpy(rows).cuda()].cpu()
    # one oracle call per sampled row, at its absolute position
    O_want = np.zeros((len(rows), wl.H, wl.d))
    lse_want = np.zeros((len(rows), wl.H))
    for i, r in enumerate(rows):
        o, l = oracle.attention(Qs[i:i + 1], Kcw, Vcw, h["K"], h["V"], int(r), wl.m, wl.W, scale,
                                sel=want_idx[i:i + 1], rows=[0])
        O_want[i], lse_want[i] = o[0], l[0]
    assert_attention_close(O[torch.from_numpy(rows).cuda()], O_want, "CSA prefill attention (sampled rows)")
    np.testing.assert_allclose(lse[torch.from_numpy(rows).cuda()].cpu().numpy(), lse_want, atol=2e-3)
    # the same call with an fp32 output: no bf16 rounding of the result
    O32, _, ws = csa.csa_sparse_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"), sel_all, g["K"],
                                     g["V"], wl.W, scale, out_dtype=torch.float32, want_lse=False)
    assert csa.csa_check_status(ws) == 0
    assert_attention_close(O32[torch.from_numpy(rows).cuda()], O_want, "CSA prefill attention (sampled rows)")


def test_hca_prefill_full_size_sampled(csa):
    wl = inputs.HCA_PREFILL
    g = inputs.prefill_layer(wl, device="cuda", with_indexer=False)
    scale = 1.0 / math.sqrt(wl.d)
    h = _host(g, ["K", "V", "Z", "B_hca"])
    Kx, Vx = oracle.compress(h["K"], h["V"], h["Z"], h["B_hca"], wl.m_hca)
    Kc, Vc = csa.csa_compress(g["K"], g["V"], g["Z"], g["B_hca"], wl.m_hca)
    assert_within_bf16_ulp(Kc, Kx, "HCA Kc", fp32_pool_slack(h["K"], wl.m_hca, h["Z"], h["B_hca"]))
    assert_within_bf16_ulp(Vc, Vx, "HCA Vc", fp32_pool_slack(h["V"], wl.m_hca, h["Z"], h["B_hca"]))
    Kcw, Vcw = oracle.to_bf16_words(Kx), oracle.to_bf16_words(Vx)
    O, lse, ws = csa.hca_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"), g["K"], g["V"], wl.m_hca,
                              wl.W_hca, scale)
    assert csa.csa_check_status(ws) == 0
    special = [0, 1, 126, 127, 128, 129, 255, 256, 65535, 65536, wl.T - 1]
    rows = sample_rows(wl.T, 16, special, seed=12)
    Qs = g["Q"][torch.from_numpy(rows).cuda()].cpu()
    O_want = np.zeros((len(rows), wl.H, wl.d))
    lse_want = np.zeros((len(rows), wl.H))
    for i, r in enumerate(rows):
        o, l = oracle.attention(Qs[i:i + 1], Kcw, Vcw, h["K"], h["V"], int(r), wl.m_hca, wl.W_hca, scale, rows=[0])
        O_want[i], lse_want[i] = o[0], l[0]
    assert_attention_close(O[torch.from_numpy(rows).cuda()], O_want, "HCA prefill attention (sampled rows)")
    np.testing.assert_allclose(lse[torch.from_numpy(rows).cuda()].cpu().numpy(), lse_want, atol=2e-3)
    O32, _, ws = csa.hca_attn(g["Q"], from_words(Kcw, "cuda"), from_words(Vcw, "cuda"), g["K"], g["V"], wl.m_hca,
                              wl.W_hca, scale, out_dtype=torch.float32, want_lse=False)
    assert csa.csa_check_status(ws) == 0
    assert_attention_close(O32[torch.from_numpy(rows).cuda()], O_want, "HCA prefill attention (sampled rows)")


def test_csa_decode_1m_context_sampled_sequences(csa):
    wl = inputs.CSA_DECODE
    g = inputs.decode_batch(wl, device="cuda")
    scale = 1.0 / math.sqrt(wl.d)
    pos = [wl.context - 1] * wl.batch
    O, lse, idx, scores, ws = csa.csa_decode(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"], g["Kc"], g["Vc"],
                                             g["kI_codes"], g["kI_scales"], g["Kwin"], g["Vwin"], pos, wl.m, wl.k,
                                             scale)
    assert csa.csa_check_status(ws) == 0
    O32, _, idx32, _, ws = csa.csa_decode(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"], g["Kc"], g["Vc"],
                                          g["kI_codes"], g["kI_scales"], g["Kwin"], g["Vwin"], pos, wl.m, wl.k,
                                          scale, out_dtype=torch.float32, want_lse=False)
    assert csa.csa_check_status(ws) == 0
    assert torch.equal(idx32, idx)
    for b in (0, 9):
        t = pos[b]
        I = oracle.indexer(g["qI_codes"][b:b + 1].cpu(), g["qI_scales"][b:b + 1].cpu(), g["w_codes"][b:b + 1].cpu(),
                           g["kI_codes"][b].cpu(), g["kI_scales"][b].cpu(), t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
        assert_topk_exact(idx[b:b + 1], scores[b:b + 1], want_idx, want_top, "decode indexer seq %d" % b)
        o, l = oracle.attention(g["q"][b:b + 1].cpu(), g["Kc"][b].cpu(), g["Vc"][b].cpu(), g["Kwin"][b].cpu(),
                                g["Vwin"][b].cpu(), t, wl.m, wl.W, scale, sel=want_idx, rows=[0],
                                raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "decode attention seq %d" % b)
        assert_attention_close(O32[b:b + 1], o, "decode attention seq %d" % b)
        np.testing.assert_allclose(lse[b:b + 1].cpu().numpy(), l, atol=2e-3)
