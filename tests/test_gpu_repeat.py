"""Repeated launches give the same bits.  The attention kernel's warps run ahead
of one another (tiles whose keys are all masked for some rows, narrow window
tiles, items of several tiles per CTA); a barrier waited out of turn shows up as
outputs that differ from launch to launch, even where each stays near the
oracle.  Every call below is made twice on the same inputs and compared bit for
bit."""
import math

import pytest
import torch

from long_context_compressed_gated_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import long_context_compressed_gated_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("W", [0, 1, 127, 128])
def test_hca_attention_repeats_bit_for_bit(csa, W):
    wl = inputs.HCA_PREFILL
    T = 8192
    d = inputs.prefill_layer(wl, T=T, device="cuda", with_indexer=False)
    Kc = torch.empty(T // wl.m_hca, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    csa.csa_compress(d["K"], d["V"], d["Z"], d["B_hca"], wl.m_hca, Kc=Kc, Vc=Vc)
    sc = 1.0 / math.sqrt(wl.d)
    outs = []
    for _ in range(3):
        O, lse, _ = csa.hca_attn(d["Q"], Kc, Vc, d["K"], d["V"], wl.m_hca, W, sc)
        outs.append((O.clone(), lse.clone()))
    for O, lse in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(lse, outs[0][1])


def test_csa_attention_repeats_bit_for_bit(csa):
    wl = inputs.CSA_PREFILL
    T = 4096
    d = inputs.prefill_layer(wl, T=T, device="cuda")
    Kc = torch.empty(T // wl.m, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    csa.csa_compress(d["K"], d["V"], d["Z"], d["B"], wl.m, Kc=Kc, Vc=Vc)
    idx, _, _ = csa.csa_indexer_topk(d["qI_codes"], d["qI_scales"], d["w_codes"], d["kI_codes"], d["kI_scales"], wl.m,
                                     wl.k, want_scores=False)
    sc = 1.0 / math.sqrt(wl.d)
    outs = []
    for _ in range(3):
        O, lse, _ = csa.csa_sparse_attn(d["Q"], Kc, Vc, idx, d["K"], d["V"], wl.W, sc)
        outs.append((O.clone(), lse.clone()))
    for O, lse in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(lse, outs[0][1])


def test_attention_items_without_tiles_do_not_stall(csa):
    """Many work items per CTA whose key sets are empty (no visible compressed
    entry, W = 0): their epilogues wait for nothing, so the softmax warps run
    items ahead of the MMA warp; the kernel must still finish with status 0 and
    write O = 0, lse = -inf (the empty-key-set reading)."""
    wl = inputs.HCA_PREFILL
    T = 296 * 16
    d = inputs.prefill_layer(wl, T=T, device="cuda", with_indexer=False)
    Kc = torch.zeros(1, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    O, lse, ws = csa.hca_attn(d["Q"], Kc, Vc, d["K"], d["V"], 1 << 20, 0, 1.0 / math.sqrt(wl.d))
    assert csa.csa_check_status(ws) == 0
    assert torch.count_nonzero(O) == 0
    assert bool(torch.all(torch.isneginf(lse)))


def test_hca_attention_mixed_empty_and_full_items(csa):
    """Items without tiles between items with tiles in the same CTA (W = 0, the
    first m' - 1 tokens see no entry): same bits on every launch, status 0."""
    wl = inputs.HCA_PREFILL
    T = 296 * 8
    d = inputs.prefill_layer(wl, T=T, device="cuda", with_indexer=False)
    m = 512  # tokens < 511 see no entry: 255 empty items, then items with one entry tile
    Kc = torch.empty(T // m, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    csa.csa_compress(d["K"], d["V"], d["Z"], d["B_hca"][:1].expand(m, -1).contiguous(), m, Kc=Kc, Vc=Vc)
    outs = []
    for _ in range(3):
        O, lse, ws = csa.hca_attn(d["Q"], Kc, Vc, d["K"], d["V"], m, 0, 1.0 / math.sqrt(wl.d))
        assert csa.csa_check_status(ws) == 0
        outs.append(O.clone())
    assert torch.count_nonzero(outs[0][:510]) == 0
    for O in outs[1:]:
        assert torch.equal(O, outs[0])


def test_csa_attention_window_only_items(csa):
    """Selected lists all empty (-1): every item is its two window tiles, the
    second one narrow, so a warp can reach the epilogue with the last PV already
    complete; no barrier phase may be waited for twice.  Status 0 and the same
    bits on every launch."""
    wl = inputs.CSA_PREFILL
    T = 4096
    d = inputs.prefill_layer(wl, T=T, device="cuda", with_indexer=False)
    Kc = torch.empty(T // wl.m, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    csa.csa_compress(d["K"], d["V"], d["Z"], d["B"], wl.m, Kc=Kc, Vc=Vc)
    idx = torch.full((T, 16), -1, dtype=torch.int32, device="cuda")
    sc = 1.0 / math.sqrt(wl.d)
    outs = []
    for _ in range(3):
        O, lse, ws = csa.csa_sparse_attn(d["Q"], Kc, Vc, idx, d["K"], d["V"], wl.W, sc)
        assert csa.csa_check_status(ws) == 0
        outs.append(O.clone())
    for O in outs[1:]:
        assert torch.equal(O, outs[0])
