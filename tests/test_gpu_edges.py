"""GPU parity on edge cases: ragged sizes, chunk offsets (t0 > 0, a cache that
holds only the entries visible so far), an empty cache, no window, fewer
visible entries than k, decode at short contexts, the MXFP4 exact-range check,
and the indexer shapes of the decode/stack workloads (16 heads x 128).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import assert_attention_close, assert_topk_exact, from_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import long_context_compressed_gated_b200 as m
    m.lib()
    return m


def _indexer_case(csa, T, Nc, HI, dI, m, k, t0, seed):
    wl = inputs.Workload("edge", T=T, HI=HI, dI=dI, m=m, k=k, seed=seed)
    qc, qs = inputs.mxfp4((T, HI), dI, seed, "qI")
    w = inputs.uniform_u8((T, HI), seed, "w", 0, 15)
    kc, ks = inputs.mxfp4((Nc,), dI, seed, "kI")
    idx, sc, ws = csa.csa_indexer_topk(qc.cuda(), qs.cuda(), w.cuda(), kc.cuda(), ks.cuda(), m, k, t0=t0)
    assert csa.csa_check_status(ws) == 0
    I = oracle.indexer(qc, qs, w, kc, ks, t0, m)
    rows = np.arange(T)
    want_idx, want_top = oracle.topk(I, np.minimum(oracle.n_vis(t0 + rows, m), Nc), k)
    assert_topk_exact(idx, sc, want_idx, want_top, "indexer T=%d Nc=%d HI=%d dI=%d k=%d t0=%d" % (T, Nc, HI, dI, k, t0))


@pytest.mark.parametrize("T,Nc,HI,dI,m,k,t0", [
    (1000, 250, 4, 64, 4, 16, 0),        # ragged T (not a multiple of the token group)
    (777, 194, 16, 128, 4, 64, 0),       # decode/stack indexer shape, ragged
    (300, 900, 64, 128, 4, 512, 3300),   # chunk at t0 > 0 against an accumulated cache
    (256, 1000, 16, 128, 4, 1024, 2000), # k > visible entries for every row
    (129, 40, 8, 64, 3, 7, 0),           # odd m and k
    (64, 0, 16, 128, 4, 32, 0),          # empty cache: every idx is -1
    (200, 3000, 32, 128, 4, 2048, 9000), # k = 2048 (largest), 32 heads
])
def test_indexer_edges(csa, T, Nc, HI, dI, m, k, t0):
    _indexer_case(csa, T, Nc, HI, dI, m, k, t0, seed=T + Nc)


def test_indexer_many_ties(csa):
    """Exact integer scores make ties common (w = 0 and ReLU zeros): ties must go
    to the smaller block index."""
    T, Nc, HI, dI, m, k = 96, 400, 16, 128, 4, 64
    qc, qs = inputs.mxfp4((T, HI), dI, 5, "qI")
    w = inputs.uniform_u8((T, HI), 5, "w", 0, 15)
    w[:, 4:] = 0                               # only 4 heads count
    qs[:] = 127
    kc, ks = inputs.mxfp4((Nc,), dI, 5, "kI")
    kc[::3] = 0                                # every third key scores exactly 0
    ks[:] = 127
    kc[1::7] = kc[0]                           # duplicated keys -> equal scores
    idx, sc, ws = csa.csa_indexer_topk(qc.cuda(), qs.cuda(), w.cuda(), kc.cuda(), ks.cuda(), m, k)
    assert csa.csa_check_status(ws) == 0
    I = oracle.indexer(qc, qs, w, kc, ks, 0, m)
    want_idx, want_top = oracle.topk(I, np.minimum(oracle.n_vis(np.arange(T), m), Nc), k)
    assert_topk_exact(idx, sc, want_idx, want_top, "indexer ties")


def test_indexer_extreme_magnitudes(csa):
    """All |codes| = 6 with scale 2^1 against mixed 2^-2 / 2^1 blocks: the largest
    head sums the exact range allows."""
    T, Nc, HI, dI, m, k = 32, 64, 64, 128, 1, 16
    qc = torch.full((T, HI, dI // 2), 0x77, dtype=torch.uint8)
    qc[::2] = 0xFF                                 # -6 on every other token
    qs = torch.full((T, HI, dI // 32), 128, dtype=torch.uint8)
    w = torch.full((T, HI), 7, dtype=torch.uint8)  # w = 6
    kc = torch.full((Nc, dI // 2), 0x77, dtype=torch.uint8)
    ks = inputs.uniform_u8((Nc, dI // 32), 9, "ks", 125, 128)
    kc[5::4] = 0x7F                                # mixed signs inside a row
    idx, sc, ws = csa.csa_indexer_topk(qc.cuda(), qs.cuda(), w.cuda(), kc.cuda(), ks.cuda(), m, k)
    assert csa.csa_check_status(ws) == 0
    I = oracle.indexer(qc, qs, w, kc, ks, 0, m)
    want_idx, want_top = oracle.topk(I, np.minimum(oracle.n_vis(np.arange(T), m), Nc), k)
    assert_topk_exact(idx, sc, want_idx, want_top, "indexer extreme magnitudes")


@pytest.mark.parametrize("T,bad", [(8, 3), (64, 60), (200, 7)])
def test_indexer_reports_scale_out_of_range(csa, T, bad):
    """A key scale byte outside [125, 128] is reported (several CTAs: the entry is
    read by the last rows only, or by every row)."""
    Nc, HI, dI = 64, 16, 128
    qc, qs = inputs.mxfp4((T, HI), dI, 1, "qI")
    w = inputs.uniform_u8((T, HI), 1, "w", 0, 15)
    kc, ks = inputs.mxfp4((Nc,), dI, 1, "kI")
    ks[bad, 1] = 124                                # 2^-3: outside the exact range
    _, _, ws = csa.csa_indexer_topk(qc.cuda(), qs.cuda(), w.cuda(), kc.cuda(), ks.cuda(), 1, 8)
    assert csa.csa_check_status(ws) == -7           # CSA_ERR_RANGE
    assert csa.csa_check_status(ws) == 0            # cleared by the read


def _attn_inputs(T, H, d, Nc, seed):
    g = torch.Generator().manual_seed(seed)
    f = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    return f(T, H, d), f(Nc, d), f(Nc, d)


def _raw_kv(n, d, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, d, generator=g).to(torch.bfloat16), torch.randn(n, d, generator=g).to(torch.bfloat16))


@pytest.mark.parametrize("T,t0,H,d,m,k,W", [
    (300, 0, 64, 128, 4, 512, 128),     # ragged T, early rows see < k entries
    (200, 5000, 16, 64, 4, 64, 100),    # chunk offset, odd window
    (130, 40, 128, 128, 4, 16, 0),      # no window, one token per CTA (H=128)
    (97, 0, 8, 64, 5, 9, 33),
])
def test_sparse_attention_edges(csa, T, t0, H, d, m, k, W):
    Nc = (t0 + T) // m
    Q, Kc, Vc = _attn_inputs(T, H, d, Nc, seed=T + t0)
    Kraw, Vraw = _raw_kv(t0 + T, d, seed=7 + T)
    rng = np.random.default_rng(T)
    sel = np.full((T, k), -1, np.int32)
    for r in range(T):
        nv = min((t0 + r + 1) // m, Nc)
        c = rng.choice(nv, size=min(k, nv), replace=False) if nv else []
        sel[r, : len(c)] = c
    scale = 1.0 / math.sqrt(d)
    O, lse, ws = csa.csa_sparse_attn(Q.cuda(), Kc.cuda(), Vc.cuda(), torch.from_numpy(sel).cuda(), Kraw.cuda(),
                                     Vraw.cuda(), W, scale, t0=t0)
    assert csa.csa_check_status(ws) == 0
    O_want, lse_want = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale, sel=sel)
    assert_attention_close(O, O_want, "sparse attention edge %s" % ((T, t0, H, d, m, k, W),))
    got = lse.cpu().numpy()
    empty = np.isneginf(lse_want)
    assert np.all(np.isneginf(got[empty])), "rows with no keys must give lse = -inf"
    np.testing.assert_allclose(got[~empty], lse_want[~empty], atol=2e-3)


@pytest.mark.parametrize("T,t0,H,d,m,W", [
    (500, 0, 64, 128, 16, 128),
    (260, 3000, 32, 64, 128, 64),
    (64, 10, 64, 128, 8, 0),            # no window: the first rows see nothing
])
def test_hca_attention_edges(csa, T, t0, H, d, m, W):
    Nc = (t0 + T) // m
    Q, Kc, Vc = _attn_inputs(T, H, d, max(Nc, 1), seed=3 * T + t0)
    Kc, Vc = Kc[:Nc], Vc[:Nc]
    Kraw, Vraw = _raw_kv(t0 + T, d, seed=11 + T)
    scale = 1.0 / math.sqrt(d)
    if Nc == 0:
        pytest.skip("empty cache")
    O, lse, ws = csa.hca_attn(Q.cuda(), Kc.cuda(), Vc.cuda(), Kraw.cuda(), Vraw.cuda(), m, W, scale, t0=t0)
    assert csa.csa_check_status(ws) == 0
    O_want, lse_want = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale)
    assert_attention_close(O, O_want, "HCA edge %s" % ((T, t0, H, d, m, W),))
    got = lse.cpu().numpy()
    empty = np.isneginf(lse_want)
    assert np.all(np.isneginf(got[empty]))
    np.testing.assert_allclose(got[~empty], lse_want[~empty], atol=2e-3)


def test_decode_short_contexts_all_sequences(csa):
    """Decode with different positions per sequence, including one whose window
    reaches before position 0 and one with fewer visible entries than k."""
    wl = inputs.Workload("dec_small", H=64, d=128, m=4, k=64, W=32, HI=16, dI=128, batch=5, context=4096, seed=21)
    g = inputs.decode_batch(wl)
    pos = [4095, 20, 1000, 255, 3]
    scale = 1.0 / math.sqrt(wl.d)
    gc = {k: v.cuda() for k, v in g.items()}
    O, lse, idx, scores, ws = csa.csa_decode(gc["q"], gc["qI_codes"], gc["qI_scales"], gc["w_codes"], gc["Kc"],
                                             gc["Vc"], gc["kI_codes"], gc["kI_scales"], gc["Kwin"], gc["Vwin"], pos,
                                             wl.m, wl.k, scale)
    assert csa.csa_check_status(ws) == 0
    for b, t in enumerate(pos):
        I = oracle.indexer(g["qI_codes"][b:b + 1], g["qI_scales"][b:b + 1], g["w_codes"][b:b + 1], g["kI_codes"][b],
                           g["kI_scales"][b], t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
        assert_topk_exact(idx[b:b + 1], scores[b:b + 1], want_idx, want_top, "decode seq %d" % b)
        o, l = oracle.attention(g["q"][b:b + 1], g["Kc"][b], g["Vc"][b], g["Kwin"][b], g["Vwin"][b], t, wl.m, wl.W,
                                scale, sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "decode attention seq %d" % b)


def test_decode_positions_beyond_the_inline_limit(csa):
    """More sequences (70) than the kernel arguments carry positions for: the
    positions go to the workspace through the copy kernel first, and the search,
    the merge and the attention read them from there.  Sequences on both sides of
    the limit (63, 64) are checked, with mixed positions."""
    B = 70
    wl = inputs.Workload("dec_b70", H=64, d=128, m=4, k=64, W=32, HI=16, dI=128, batch=B, context=2048, seed=27)
    g = inputs.decode_batch(wl)
    pos = [(97 * b + 13) % wl.context for b in range(B)]
    pos[69] = wl.context - 1
    scale = 1.0 / math.sqrt(wl.d)
    gc = {k: v.cuda() for k, v in g.items()}
    O, lse, idx, scores, ws = csa.csa_decode(gc["q"], gc["qI_codes"], gc["qI_scales"], gc["w_codes"], gc["Kc"],
                                             gc["Vc"], gc["kI_codes"], gc["kI_scales"], gc["Kwin"], gc["Vwin"], pos,
                                             wl.m, wl.k, scale)
    assert csa.csa_check_status(ws) == 0
    for b in (0, 5, 63, 64, 69):
        t = pos[b]
        I = oracle.indexer(g["qI_codes"][b:b + 1], g["qI_scales"][b:b + 1], g["w_codes"][b:b + 1], g["kI_codes"][b],
                           g["kI_scales"][b], t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
        assert_topk_exact(idx[b:b + 1], scores[b:b + 1], want_idx, want_top, "decode B=70 seq %d" % b)
        o, l = oracle.attention(g["q"][b:b + 1], g["Kc"][b], g["Vc"][b], g["Kwin"][b], g["Vwin"][b], t, wl.m, wl.W,
                                scale, sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "decode B=70 attention seq %d" % b)


def test_decode_search_long_key_ranges(csa):
    """Long key ranges (38 sequences of 131072 entries: three ranges of 342 tiles
    each), so that the search's candidate buffers are cut back several times and
    meet often.  The k best keys of two sequences are checked against the oracle,
    bit for bit."""
    B, N, HI, dI, m, k = 38, 1 << 17, 16, 128, 4, 512
    qc, qs = inputs.mxfp4((B, HI), dI, 31, "qI")
    w = inputs.uniform_u8((B, HI), 31, "w", 0, 15)
    kc, ks = inputs.mxfp4((B, N), dI, 31, "kI")
    pos = [N * m - 1 - 977 * b for b in range(B)]
    keys, ws = csa.csa_decode_search(qc.cuda(), qs.cuda(), w.cuda(), kc.cuda(), ks.cuda(), pos, m, k)
    assert csa.csa_check_status(ws) == 0
    kk = keys.cpu().numpy().view(np.uint64)
    units = ((kk >> np.uint64(32)).astype(np.uint32) ^ np.uint32(0x80000000)).view(np.int32)
    j = (np.uint64(0xFFFFFFFF) - (kk & np.uint64(0xFFFFFFFF))).astype(np.int64)
    for b in (0, B - 1):
        t = pos[b]
        I = oracle.indexer(qc[b:b + 1], qs[b:b + 1], w[b:b + 1], kc[b], ks[b], t, m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], m), k)
        assert_topk_exact(torch.from_numpy(j[b:b + 1]), torch.from_numpy(units[b:b + 1].astype(np.float32) / 128.0),
                          want_idx, want_top, "decode search seq %d" % b)


def test_decode_k2048_split_search(csa):
    """Decode with k=2048 over a 64K-token context: the key range is split over
    several CTAs and the merged selection is larger than the block finalize's
    register sort, so its shared-memory bitonic path runs."""
    wl = inputs.Workload("dec_k2048", H=64, d=128, m=4, k=2048, W=128, HI=16, dI=128, batch=2, context=1 << 16,
                         seed=23)
    g = inputs.decode_batch(wl)
    pos = [wl.context - 1, 30000]
    scale = 1.0 / math.sqrt(wl.d)
    gc = {k: v.cuda() for k, v in g.items()}
    O, lse, idx, scores, ws = csa.csa_decode(gc["q"], gc["qI_codes"], gc["qI_scales"], gc["w_codes"], gc["Kc"],
                                             gc["Vc"], gc["kI_codes"], gc["kI_scales"], gc["Kwin"], gc["Vwin"], pos,
                                             wl.m, wl.k, scale)
    assert csa.csa_check_status(ws) == 0
    for b, t in enumerate(pos):
        I = oracle.indexer(g["qI_codes"][b:b + 1], g["qI_scales"][b:b + 1], g["w_codes"][b:b + 1], g["kI_codes"][b],
                           g["kI_scales"][b], t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
        assert_topk_exact(idx[b:b + 1], scores[b:b + 1], want_idx, want_top, "decode k=2048 seq %d" % b)
        o, l = oracle.attention(g["q"][b:b + 1], g["Kc"][b], g["Vc"][b], g["Kwin"][b], g["Vwin"][b], t, wl.m, wl.W,
                                scale, sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "decode k=2048 attention seq %d" % b)


@pytest.mark.parametrize("k,context", [(1024, 1 << 18), (64, 1 << 17)])
def test_decode_single_sequence_widest_split(csa, k, context):
    """One sequence over a long context: its key range is split over the most
    CTAs the merge allows (10 ranges at k = 1024; at k = 64 the SM count would give
    148 and the range limit of the block finalize, 63, applies)."""
    wl = inputs.Workload("dec_b1", H=64, d=128, m=4, k=k, W=128, HI=16, dI=128, batch=1, context=context,
                         seed=24 + k)
    g = inputs.decode_batch(wl)
    pos = [wl.context - 1]
    scale = 1.0 / math.sqrt(wl.d)
    gc = {key: v.cuda() for key, v in g.items()}
    O, lse, idx, scores, ws = csa.csa_decode(gc["q"], gc["qI_codes"], gc["qI_scales"], gc["w_codes"], gc["Kc"],
                                             gc["Vc"], gc["kI_codes"], gc["kI_scales"], gc["Kwin"], gc["Vwin"], pos,
                                             wl.m, wl.k, scale)
    assert csa.csa_check_status(ws) == 0
    t = pos[0]
    I = oracle.indexer(g["qI_codes"], g["qI_scales"], g["w_codes"], g["kI_codes"][0], g["kI_scales"][0], t, wl.m)
    want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
    assert_topk_exact(idx, scores, want_idx, want_top, "decode B=1 k=%d" % k)
    o, l = oracle.attention(g["q"], g["Kc"][0], g["Vc"][0], g["Kwin"][0], g["Vwin"][0], t, wl.m, wl.W, scale,
                            sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
    assert_attention_close(O, o, "decode B=1 k=%d attention" % k)
    np.testing.assert_allclose(lse.cpu().numpy(), l, atol=2e-3)


def test_hca_decode(csa):
    wl = inputs.Workload("hdec", H=64, d=128, m=128, W=128, batch=3, context=1 << 20, seed=22)
    n = wl.context // wl.m
    gen = torch.Generator().manual_seed(22)
    f = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    q, Kc, Vc = f(wl.batch, wl.H, wl.d), f(wl.batch, n, wl.d), f(wl.batch, n, wl.d)
    Kw, Vw = f(wl.batch, wl.W, wl.d), f(wl.batch, wl.W, wl.d)
    pos = [wl.context - 1, 5000, 127]
    scale = 1.0 / math.sqrt(wl.d)
    O, lse, ws = csa.hca_decode(q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), pos, wl.m, scale)
    assert csa.csa_check_status(ws) == 0
    for b, t in enumerate(pos):
        o, l = oracle.attention(q[b:b + 1], Kc[b], Vc[b], Kw[b], Vw[b], t, wl.m, wl.W, scale, rows=[0],
                                raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "HCA decode seq %d" % b)
        np.testing.assert_allclose(lse[b:b + 1].cpu().numpy(), l, atol=2e-3)


@pytest.mark.parametrize("T,d,m", [(1000, 128, 4), (1000, 64, 64), (4096, 128, 128), (333, 128, 8), (640, 64, 1),
                                   (1001, 64, 3), (997, 128, 6), (3000, 128, 24), (4000, 64, 40), (2200, 128, 136),
                                   (5120, 128, 512), (5000, 64, 512), (70000, 128, 4), (300000, 128, 128)])
def test_compress_edges(csa, T, d, m):
    from tests.parity import assert_within_bf16_ulp, fp32_pool_slack
    g = torch.Generator().manual_seed(T + m)
    K, V, Z = (torch.randn(T, d, generator=g).to(torch.bfloat16) for _ in range(3))
    B = torch.randn(m, d, generator=g) * 0.5
    Kc, Vc = csa.csa_compress(K.cuda(), V.cuda(), Z.cuda(), B.cuda(), m)
    Kx, Vx = oracle.compress(K, V, Z, B, m)
    assert Kc.shape[0] == T // m
    assert_within_bf16_ulp(Kc, Kx, "Kc", fp32_pool_slack(K, m, Z, B))
    assert_within_bf16_ulp(Vc, Vx, "Vc", fp32_pool_slack(V, m, Z, B))


def test_hca_attention_many_visible_entries(csa):
    """A dense block over ~12.5K visible entries (98 key tiles of 128): dense
    tiles are generated from their index, so no tile list bounds the count."""
    T, t0, H, d, m, W = 64, 200000, 64, 128, 16, 128
    Nc = (t0 + T) // m
    Q, Kc, Vc = _attn_inputs(T, H, d, Nc, seed=77)
    Kraw, Vraw = _raw_kv(t0 + T, d, seed=78)
    scale = 1.0 / math.sqrt(d)
    O, lse, ws = csa.hca_attn(Q.cuda(), Kc.cuda(), Vc.cuda(), Kraw.cuda(), Vraw.cuda(), m, W, scale, t0=t0,
                              out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    O_want, lse_want = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale)
    assert_attention_close(O, O_want, "HCA over %d entries" % Nc)
    np.testing.assert_allclose(lse.cpu().numpy(), lse_want, atol=2e-3)


def test_large_outputs_need_the_fp32_output(csa):
    """A peaked softmax (queries scaled by 10) over V ~ N(0, 1.25^2) gives |O| of 4
    and more: there one bf16 half-ulp (2^-6) alone is above the 1e-2 bound, so
    the fp32 output is the one held to the tolerance; the bf16 output must be
    the round-to-nearest-even of that same fp32 result.  (V much wider than the
    workloads' N(0,1) would not do: the bf16 rounding of the softmax weights
    before the PV product, 2^-9 relative, then exceeds the bound by itself.)"""
    T, t0, H, d, m, k, W = 256, 0, 64, 128, 4, 64, 128
    Nc = (t0 + T) // m
    Q, Kc, Vc = _attn_inputs(T, H, d, Nc, seed=91)
    Kraw, Vraw = _raw_kv(t0 + T, d, seed=92)
    Q = (Q.float() * 10).to(torch.bfloat16)
    Vc = (Vc.float() * 1.25).to(torch.bfloat16)
    Vraw = (Vraw.float() * 1.25).to(torch.bfloat16)
    rng = np.random.default_rng(93)
    sel = np.full((T, k), -1, np.int32)
    for r in range(T):
        nv = (t0 + r + 1) // m
        c = rng.choice(nv, size=min(k, nv), replace=False) if nv else []
        sel[r, : len(c)] = c
    scale = 1.0 / math.sqrt(d)
    O_want, _ = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale, sel=sel)
    assert np.abs(O_want).max() >= 4.0
    O32, _, ws = csa.csa_sparse_attn(Q.cuda(), Kc.cuda(), Vc.cuda(), torch.from_numpy(sel).cuda(), Kraw.cuda(),
                                     Vraw.cuda(), W, scale, t0=t0, out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    assert_attention_close(O32, O_want, "sparse attention, peaked softmax, |O| >= 4")
    O16, _, ws = csa.csa_sparse_attn(Q.cuda(), Kc.cuda(), Vc.cuda(), torch.from_numpy(sel).cuda(), Kraw.cuda(),
                                     Vraw.cuda(), W, scale, t0=t0, out_dtype=torch.bfloat16)
    assert torch.equal(O16, O32.to(torch.bfloat16))


def test_hca_decode_fp32_output(csa):
    wl = inputs.Workload("hdec32", H=64, d=128, m=128, W=128, batch=2, context=1 << 18, seed=29)
    n = wl.context // wl.m
    gen = torch.Generator().manual_seed(29)
    f = lambda *s: torch.randn(*s, generator=gen).to(torch.bfloat16)
    q, Kc, Vc = f(wl.batch, wl.H, wl.d), f(wl.batch, n, wl.d), f(wl.batch, n, wl.d)
    Kw, Vw = f(wl.batch, wl.W, wl.d), f(wl.batch, wl.W, wl.d)
    pos = [wl.context - 1, 70000]
    scale = 1.0 / math.sqrt(wl.d)
    O, lse, ws = csa.hca_decode(q.cuda(), Kc.cuda(), Vc.cuda(), Kw.cuda(), Vw.cuda(), pos, wl.m, scale,
                                out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    assert O.dtype == torch.float32
    for b, t in enumerate(pos):
        o, l = oracle.attention(q[b:b + 1], Kc[b], Vc[b], Kw[b], Vw[b], t, wl.m, wl.W, scale, rows=[0],
                                raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "HCA decode fp32 seq %d" % b)


@pytest.mark.parametrize("HI,dI", [(4, 64), (32, 128), (64, 128)])
def test_decode_indexer_head_counts(csa, HI, dI):
    """Decode with 4, 32 and 64 indexer heads: the 16-warp epilogue (four groups
    taking turns on the key tiles) and, at 64 heads, the 8-warp one."""
    wl = inputs.Workload("dec_hi", H=64, d=128, m=4, k=256, W=64, HI=HI, dI=dI, batch=3, context=1 << 16,
                         seed=90 + HI)
    g = inputs.decode_batch(wl)
    pos = [wl.context - 1, 40000, 777]
    scale = 1.0 / math.sqrt(wl.d)
    gc = {key: v.cuda() for key, v in g.items()}
    O, lse, idx, scores, ws = csa.csa_decode(gc["q"], gc["qI_codes"], gc["qI_scales"], gc["w_codes"], gc["Kc"],
                                             gc["Vc"], gc["kI_codes"], gc["kI_scales"], gc["Kwin"], gc["Vwin"], pos,
                                             wl.m, wl.k, scale, out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    for b, t in enumerate(pos):
        I = oracle.indexer(g["qI_codes"][b:b + 1], g["qI_scales"][b:b + 1], g["w_codes"][b:b + 1], g["kI_codes"][b],
                           g["kI_scales"][b], t, wl.m)
        want_idx, want_top = oracle.topk(I, oracle.n_vis([t], wl.m), wl.k)
        assert_topk_exact(idx[b:b + 1], scores[b:b + 1], want_idx, want_top, "decode HI=%d seq %d" % (HI, b))
        o, _ = oracle.attention(g["q"][b:b + 1], g["Kc"][b], g["Vc"][b], g["Kwin"][b], g["Vwin"][b], t, wl.m, wl.W,
                                scale, sel=want_idx, rows=[0], raw_pos0=t - wl.W + 1)
        assert_attention_close(O[b:b + 1], o, "decode HI=%d attention seq %d" % (HI, b))
