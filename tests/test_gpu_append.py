"""Decode with cache maintenance: a prefill builds the compressed cache, window
and block staging of each sequence; then every decode step appends its token
(csa_decode_append / hca_decode_append) and decodes at that position.  At every
step the selection must equal the oracle's bit for bit and the output must be
within the attention tolerance; at the end the appended entries must be
bit-identical to csa_compress over the same tokens and the window must hold the
latest W raw tokens.  Compressed cache of a 1M-token context: ferris-liu.github.io
... deepseek-v4 section 3; blocks of m (m') tokens: blog.nickys.cn/?p=150
"1. CSA" / "2. HCA"."""
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


def _prefill_state(csa, K, V, Z, Bias, P0, m, W, Ncap, d):
    """Cache, window and staging of one sequence after its first P0 tokens (GPU)."""
    n0 = P0 // m
    Kc = torch.zeros(Ncap, d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    if n0:
        csa.csa_compress(K[: n0 * m], V[: n0 * m], Z[: n0 * m], Bias, m, Kc=Kc[:n0], Vc=Vc[:n0])
    Kw = torch.zeros(W, d, dtype=torch.bfloat16, device="cuda")
    Vw = torch.zeros_like(Kw)
    lo = max(0, P0 - W)
    Kw[W - (P0 - lo):] = K[lo:P0]
    Vw[W - (P0 - lo):] = V[lo:P0]
    Kb = torch.zeros(m, d, dtype=torch.bfloat16, device="cuda")
    Vb, Zb = torch.zeros_like(Kb), torch.zeros_like(Kb)
    r = P0 - n0 * m
    Kb[:r], Vb[:r], Zb[:r] = K[n0 * m:P0], V[n0 * m:P0], Z[n0 * m:P0]
    return Kc, Vc, Kw, Vw, Kb, Vb, Zb


def test_csa_decode_with_appends(csa):
    H, d, m, k, W, HI, dI = 64, 128, 4, 64, 32, 16, 128
    P0 = [1001, 514]            # one token and two tokens into a block
    steps = 23                  # crosses several block boundaries in both sequences
    Bs = len(P0)
    Ltot = max(P0) + steps
    Ncap = Ltot // m + 1
    scale = 1.0 / math.sqrt(d)
    seqs = []
    for b in range(Bs):
        s = 500 + b
        seqs.append(dict(K=inputs.normal_bf16((Ltot, d), s, "K"), V=inputs.normal_bf16((Ltot, d), s, "V"),
                         Z=inputs.normal_bf16((Ltot, d), s, "Z"), q=inputs.normal_bf16((Ltot, H, d), s, "q"),
                         w=inputs.uniform_u8((Ltot, HI), s, "w", 0, 15)))
        seqs[b]["qIc"], seqs[b]["qIs"] = inputs.mxfp4((Ltot, HI), dI, s, "qI")
        seqs[b]["kIc"], seqs[b]["kIs"] = inputs.mxfp4((Ncap,), dI, s, "kI")
    Bias = inputs.normal_f32((m, d), 77, "B", std=0.5)
    Bg = Bias.cuda()
    st = [_prefill_state(csa, sq["K"].cuda(), sq["V"].cuda(), sq["Z"].cuda(), Bg, P0[b], m, W, Ncap, d)
          for b, sq in enumerate(seqs)]
    Kc = torch.stack([x[0] for x in st]); Vc = torch.stack([x[1] for x in st])
    Kw = torch.stack([x[2] for x in st]); Vw = torch.stack([x[3] for x in st])
    Kb = torch.stack([x[4] for x in st]); Vb = torch.stack([x[5] for x in st]); Zb = torch.stack([x[6] for x in st])
    kIc = torch.zeros(Bs, Ncap, dI // 2, dtype=torch.uint8, device="cuda")
    kIs = torch.full((Bs, Ncap, dI // 32), 127, dtype=torch.uint8, device="cuda")
    for b in range(Bs):
        n0 = P0[b] // m
        kIc[b, :n0] = seqs[b]["kIc"][:n0].cuda()
        kIs[b, :n0] = seqs[b]["kIs"][:n0].cuda()
    for step in range(steps):
        pos = [p + step for p in P0]
        g = lambda key, sl=None: torch.stack([seqs[b][key][pos[b]] for b in range(Bs)]).cuda()
        jn = [min((p + 1) // m - 1, Ncap - 1) for p in pos]
        kic_new = torch.stack([seqs[b]["kIc"][max(jn[b], 0)] for b in range(Bs)]).cuda()
        kis_new = torch.stack([seqs[b]["kIs"][max(jn[b], 0)] for b in range(Bs)]).cuda()
        csa.csa_decode_append(g("K"), g("V"), g("Z"), Bg, pos, Kw, Vw, Kb, Vb, Zb, Kc, Vc, kI_codes_new=kic_new,
                              kI_scales_new=kis_new, kI_codes=kIc, kI_scales=kIs)
        O, lse, idx, sc, ws = csa.csa_decode(g("q"), g("qIc"), g("qIs"), g("w"), Kc, Vc, kIc, kIs, Kw, Vw, pos, m,
                                             k, scale, out_dtype=torch.float32)
        assert csa.csa_check_status(ws) == 0
        for b in range(Bs):
            p = pos[b]
            sq = seqs[b]
            nv = (p + 1) // m
            I = oracle.indexer(sq["qIc"][p:p + 1], sq["qIs"][p:p + 1], sq["w"][p:p + 1], sq["kIc"][:nv],
                               sq["kIs"][:nv], p, m)
            want_idx, want_top = oracle.topk(I, [nv], k)
            assert_topk_exact(idx[b:b + 1], sc[b:b + 1], want_idx, want_top, "step %d seq %d" % (step, b))
            Kx, Vx = oracle.compress(sq["K"][: nv * m], sq["V"][: nv * m], sq["Z"][: nv * m], Bias, m)
            o, _ = oracle.attention(sq["q"][p:p + 1], oracle.to_bf16_words(Kx), oracle.to_bf16_words(Vx),
                                    sq["K"], sq["V"], p, m, W, scale, sel=want_idx, rows=[0])
            assert_attention_close(O[b:b + 1], o, "decode after append, step %d seq %d" % (step, b))
    torch.cuda.synchronize()
    for b in range(Bs):
        pend = P0[b] + steps
        n = pend // m
        Kr, Vr = csa.csa_compress(seqs[b]["K"][: n * m].cuda(), seqs[b]["V"][: n * m].cuda(),
                                  seqs[b]["Z"][: n * m].cuda(), Bg, m)
        assert torch.equal(Kc[b, :n], Kr) and torch.equal(Vc[b, :n], Vr), "appended entries differ from prefill"
        assert torch.equal(Kw[b], seqs[b]["K"][pend - W:pend].cuda())
        assert torch.equal(Vw[b], seqs[b]["V"][pend - W:pend].cuda())
        assert torch.equal(kIc[b, :n], seqs[b]["kIc"][:n].cuda())


def test_hca_decode_with_appends(csa):
    """HCA cache (m' = 128): appends across two block boundaries; the window
    (W = 128) and the pooled entries of 128 tokens (two slices merged per channel)."""
    H, d, m, W = 64, 128, 128, 128
    P0, steps = 1000, 290
    Ltot = P0 + steps
    Ncap = Ltot // m + 1
    scale = 1.0 / math.sqrt(d)
    s = 620
    K, V, Z = (inputs.normal_bf16((Ltot, d), s, n) for n in ("K", "V", "Z"))
    q = inputs.normal_bf16((Ltot, H, d), s, "q")
    Bias = inputs.normal_f32((m, d), s, "B", std=0.5)
    Bg = Bias.cuda()
    Kc, Vc, Kw, Vw, Kb, Vb, Zb = (x.unsqueeze(0) for x in
                                  _prefill_state(csa, K.cuda(), V.cuda(), Z.cuda(), Bg, P0, m, W, Ncap, d))
    check_steps = {0, 22, 23, 24, 150, 151, 152, steps - 1}
    for step in range(steps):
        p = P0 + step
        csa.hca_decode_append(K[p:p + 1].cuda(), V[p:p + 1].cuda(), Z[p:p + 1].cuda(), Bg, [p], Kw, Vw, Kb, Vb, Zb,
                              Kc, Vc)
        if step not in check_steps:
            continue
        O, _, ws = csa.hca_decode(q[p:p + 1].cuda(), Kc, Vc, Kw, Vw, [p], m, scale, out_dtype=torch.float32)
        assert csa.csa_check_status(ws) == 0
        nv = (p + 1) // m
        Kx, Vx = oracle.compress(K[: nv * m], V[: nv * m], Z[: nv * m], Bias, m)
        o, _ = oracle.attention(q[p:p + 1], oracle.to_bf16_words(Kx), oracle.to_bf16_words(Vx), K, V, p, m, W, scale,
                                rows=[0])
        assert_attention_close(O, o, "HCA decode after append, step %d" % step)
    torch.cuda.synchronize()
    pend = P0 + steps
    n = pend // m
    Kr, Vr = csa.csa_compress(K[: n * m].cuda(), V[: n * m].cuda(), Z[: n * m].cuda(), Bg, m)
    assert torch.equal(Kc[0, :n], Kr) and torch.equal(Vc[0, :n], Vr)
    assert torch.equal(Kw[0], K[pend - W:pend].cuda())


@pytest.mark.parametrize("d,m", [(64, 3), (128, 6), (64, 64), (128, 40), (128, 512), (64, 512)])
def test_append_pooling_layouts(csa, d, m):
    """Append 2m + 1 tokens from an empty state: the two completed entries are
    bit-identical to csa_compress of the same tokens for pooling layouts with
    sub-warp groups, in-warp levels and cross-warp merges, and within tolerance
    of the oracle."""
    from tests.parity import assert_within_bf16_ulp, fp32_pool_slack
    W, n = 4, 2 * m + 1
    s = 700 + m + d
    K, V, Z = (inputs.normal_bf16((n, d), s, x) for x in ("K", "V", "Z"))
    Bias = inputs.normal_f32((m, d), s, "B", std=0.5)
    Bg = Bias.cuda()
    z = lambda *shape: torch.zeros(*shape, dtype=torch.bfloat16, device="cuda")
    Kw, Vw, Kb, Vb, Zb, Kc, Vc = z(1, W, d), z(1, W, d), z(1, m, d), z(1, m, d), z(1, m, d), z(1, 3, d), z(1, 3, d)
    Kg, Vg, Zg = K.cuda(), V.cuda(), Z.cuda()
    for p in range(n):
        csa.hca_decode_append(Kg[p:p + 1], Vg[p:p + 1], Zg[p:p + 1], Bg, [p], Kw, Vw, Kb, Vb, Zb, Kc, Vc)
    Kr, Vr = csa.csa_compress(Kg[: 2 * m], Vg[: 2 * m], Zg[: 2 * m], Bg, m)
    torch.cuda.synchronize()
    assert torch.equal(Kc[0, :2], Kr) and torch.equal(Vc[0, :2], Vr)
    assert not Kc[0, 2].any()
    Kx, Vx = oracle.compress(K[: 2 * m], V[: 2 * m], Z[: 2 * m], Bias, m)
    assert_within_bf16_ulp(Kr, Kx, "Kc", fp32_pool_slack(K[: 2 * m], m, Z[: 2 * m], Bias))
    assert_within_bf16_ulp(Vr, Vx, "Vc", fp32_pool_slack(V[: 2 * m], m, Z[: 2 * m], Bias))
    assert torch.equal(Kw[0], Kg[n - W:n])
