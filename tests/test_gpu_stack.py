"""GPU parity of the chunked two-layer stack (CSA layer -> bf16 projection -> HCA
layer, chunked causal prefill against the accumulated compressed caches).

Hybrid CSA/HCA interleaving: blog.nickys.cn/?p=150 ("CSA and HCA alternate
across layers"); chunked prefill against an accumulated cache is the stack
workload of the specification.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from long_context_compressed_gated_b200.stack import stack_inputs, stack_prefill_chunked
from tests.parity import assert_attention_close, assert_topk_exact, from_words, sample_rows

pytestmark = pytest.mark.gpu

SMALL = inputs.Workload("stack_small", T=2048, H=4, d=64, m=4, k=16, W=64, HI=4, dI=64, m_hca=64, W_hca=64,
                        chunk=512, seed=41)


def _run(wl, l1, l2, P, chunk):
    g1 = {k: v.cuda() for k, v in l1.items()}
    g2 = {k: v.cuda() for k, v in l2.items()}
    return stack_prefill_chunked(g1, g2, P.cuda(), chunk, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca, return_o1=True)


def _oracle_rows(wl, l1, l2, P, rows):
    """Oracle chain for the given rows: layer 1 in fp64, O1 rounded to bf16,
    Q2 = bf16(O1 @ P) in fp64, layer 2 in fp64."""
    scale = 1.0 / math.sqrt(wl.d)
    Kc1, Vc1 = oracle.compress(l1["K"], l1["V"], l1["Z"], l1["B"], wl.m)
    K1w, V1w = oracle.to_bf16_words(Kc1), oracle.to_bf16_words(Vc1)
    I = oracle.indexer(l1["qI_codes"], l1["qI_scales"], l1["w_codes"], l1["kI_codes"], l1["kI_scales"], 0, wl.m,
                       rows)
    sel, _ = oracle.topk(I, oracle.n_vis(rows, wl.m), wl.k)
    Kc2, Vc2 = oracle.compress(l2["K"], l2["V"], l2["Z"], l2["B"], wl.m_hca)
    K2w, V2w = oracle.to_bf16_words(Kc2), oracle.to_bf16_words(Vc2)
    Pf = oracle.bf16_words_to_f64(oracle._u16(P)).reshape(wl.d, wl.d)
    O1 = np.zeros((len(rows), wl.H, wl.d))
    O2 = np.zeros((len(rows), wl.H, wl.d))
    Q2w = np.zeros((len(rows), wl.H, wl.d), np.uint16)
    for i, r in enumerate(rows):
        o1, _ = oracle.attention(l1["Q"][r:r + 1], K1w, V1w, l1["K"], l1["V"], int(r), wl.m, wl.W, scale,
                                 sel=sel[i:i + 1], rows=[0])
        O1[i] = o1[0]
        q2 = oracle.to_bf16_words(oracle.bf16_words_to_f64(oracle.to_bf16_words(o1[0])) @ Pf)
        Q2w[i] = q2
        o2, _ = oracle.attention(q2.reshape(1, wl.H, wl.d), K2w, V2w, l2["K"], l2["V"], int(r), wl.m_hca, wl.W_hca,
                                 scale, rows=[0])
        O2[i] = o2[0]
    return O1, O2, Q2w, K2w, V2w


def test_chunked_equals_unchunked_small():
    wl = SMALL
    l1, l2, P = stack_inputs(wl)
    O2c, O1c = _run(wl, l1, l2, P, wl.chunk)
    O2u, O1u = _run(wl, l1, l2, P, wl.T)
    # layer 1 is row-local and deterministic: chunking changes nothing
    assert torch.equal(O1c, O1u)
    assert_attention_close(O2c, O2u.float().cpu().double().numpy(), "stack chunked vs unchunked (layer 2)")


def test_small_stack_against_oracle():
    wl = SMALL
    l1, l2, P = stack_inputs(wl)
    O2, O1 = _run(wl, l1, l2, P, wl.chunk)
    rows = sample_rows(wl.T, 40, [0, 63, 64, 511, 512, 513, 1023, 1024, 2047], seed=5)
    O1x, O2x, Q2w, K2w, V2w = _oracle_rows(wl, l1, l2, P, rows)
    sel_rows = torch.from_numpy(rows).cuda()
    assert_attention_close(O1[sel_rows], O1x, "stack layer 1 (sampled rows)")
    assert_attention_close(O2[sel_rows], O2x, "stack layer 2 end to end (sampled rows)")
    # layer 2 alone with the oracle's Q2 and compressed cache on both sides
    import long_context_compressed_gated_b200 as csa
    scale = 1.0 / math.sqrt(wl.d)
    K2g, V2g = from_words(K2w, "cuda"), from_words(V2w, "cuda")
    got = []
    for i, r in enumerate(rows):
        Oi, _, _ = csa.hca_attn(from_words(Q2w[i:i + 1], "cuda"), K2g, V2g, l2["K"][: r + 1].cuda(),
                                l2["V"][: r + 1].cuda(), wl.m_hca, wl.W_hca, scale, t0=int(r))
        got.append(Oi)
    assert_attention_close(torch.cat(got), O2x, "stack layer 2 per layer (sampled rows)")


def _stack_indexer_rows(wl):
    """Rows of the full stack whose layer-1 selection is checked bit for bit: in
    every chunk its first row, the rows either side of the chunk start, its last
    row and two seeded rows; the rows where the visible count crosses k; T-1."""
    rows = {wl.k * wl.m - 2, wl.k * wl.m - 1, wl.k * wl.m, wl.k * wl.m + wl.m, wl.T - 1}
    rng = np.random.default_rng(404)
    for c in range(wl.T // wl.chunk):
        s0 = c * wl.chunk
        rows.update({s0, s0 + 1, s0 - 1, s0 + wl.chunk - 1})
        rows.update(int(x) for x in rng.integers(s0, s0 + wl.chunk, size=2))
    return np.array(sorted(r for r in rows if 0 <= r < wl.T), dtype=np.int64)


def test_full_size_stack_sampled():
    """The T=262144 stack in 16384-token chunks (64 x 128, CSA m=4 k=1024, HCA
    m'=128, indexer 16 x 128).  The layer-1 indexer scores and top-k indices of
    the chunked calls are compared bit for bit with the oracle on rows of every
    chunk (up to 65536 visible entries); the attention outputs on sampled rows."""
    wl = inputs.STACK
    l1, l2, P = stack_inputs(wl, device="cuda")
    idx_all = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    sc_all = torch.empty(wl.T, wl.k, dtype=torch.float32, device="cuda")
    O2, O1 = stack_prefill_chunked(l1, l2, P, wl.chunk, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca, return_o1=True,
                                   idx_out=idx_all, scores_out=sc_all)
    torch.cuda.synchronize()
    irows = _stack_indexer_rows(wl)
    hI = {k: l1[k].cpu() for k in ("qI_codes", "qI_scales", "w_codes", "kI_codes", "kI_scales")}
    I = oracle.indexer(hI["qI_codes"], hI["qI_scales"], hI["w_codes"], hI["kI_codes"], hI["kI_scales"], 0, wl.m,
                       irows)
    want_idx, want_top = oracle.topk(I, oracle.n_vis(irows, wl.m), wl.k)
    del I
    sel = torch.from_numpy(irows).cuda()
    assert_topk_exact(idx_all[sel], sc_all[sel], want_idx, want_top,
                      "stack layer-1 indexer, %d rows of all %d chunks" % (len(irows), wl.T // wl.chunk))
    del idx_all, sc_all
    rows = np.array([0, 4095, 16383, 16384, 16385, 70000, 131071, 200000, wl.T - 1], dtype=np.int64)
    h1 = {k: v.cpu() for k, v in l1.items() if k != "Q"}
    h1["Q"] = l1["Q"][torch.from_numpy(rows).cuda()].cpu()
    h2 = {k: v.cpu() for k, v in l2.items()}
    # the oracle reads Q rows by index: build a Q with the sampled rows at their positions' index i
    O1x = np.zeros((len(rows), wl.H, wl.d))
    O2x = np.zeros((len(rows), wl.H, wl.d))
    scale = 1.0 / math.sqrt(wl.d)
    Kc1, Vc1 = oracle.compress(h1["K"], h1["V"], h1["Z"], h1["B"], wl.m)
    K1w, V1w = oracle.to_bf16_words(Kc1), oracle.to_bf16_words(Vc1)
    Kc2, Vc2 = oracle.compress(h2["K"], h2["V"], h2["Z"], h2["B"], wl.m_hca)
    K2w, V2w = oracle.to_bf16_words(Kc2), oracle.to_bf16_words(Vc2)
    Pf = oracle.bf16_words_to_f64(oracle._u16(P)).reshape(wl.d, wl.d)
    for i, r in enumerate(rows):
        I = oracle.indexer(h1["qI_codes"][r:r + 1], h1["qI_scales"][r:r + 1], h1["w_codes"][r:r + 1],
                           h1["kI_codes"], h1["kI_scales"], int(r), wl.m)
        sel, _ = oracle.topk(I, oracle.n_vis([r], wl.m), wl.k)
        o1, _ = oracle.attention(h1["Q"][i:i + 1], K1w, V1w, h1["K"], h1["V"], int(r), wl.m, wl.W, scale, sel=sel,
                                 rows=[0])
        O1x[i] = o1[0]
        q2 = oracle.to_bf16_words(oracle.bf16_words_to_f64(oracle.to_bf16_words(o1[0])) @ Pf)
        o2, _ = oracle.attention(q2.reshape(1, wl.H, wl.d), K2w, V2w, h2["K"], h2["V"], int(r), wl.m_hca, wl.W_hca,
                                 scale, rows=[0])
        O2x[i] = o2[0]
    sel_rows = torch.from_numpy(rows).cuda()
    assert_attention_close(O1[sel_rows], O1x, "full stack layer 1 (sampled rows)")
    assert_attention_close(O2[sel_rows], O2x, "full stack layer 2 end to end (sampled rows)")
