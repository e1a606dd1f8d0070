"""Pins for the oracle's lightning indexer on MXFP4 and its causal top-k.

Indexer: sz-guanghua.com.cn ifanr repost, attention section (FP4 relevance
score of every query token against every compressed block, then top-k);
m.youleyou.com/wenzhang/2906406.html section 1 (MXFP4 on the indexer QK path).
Score rule I[t,j] = sum_h w[t,h]*ReLU(qI[t,h].kI[j]); visibility j*m+m-1 <= t.
"""
import json
import os

import numpy as np
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_e2m1_table_matches_the_mx_format():
    table = json.load(open(os.path.join(GOLD, "e2m1_table.json")))["values"]
    got = [oracle.e2m1_value(c) for c in range(16)]
    assert got == table
    assert np.signbit(oracle.e2m1_value(8))  # code 8 is -0


def test_e2m1_embeds_losslessly_in_e4m3():
    # ifanr repost: FP4 (E2M1) -> FP8 (E4M3) dequantisation is lossless.
    vals = torch.tensor([oracle.e2m1_value(c) for c in range(16)], dtype=torch.float64)
    assert torch.equal(vals.to(torch.float8_e4m3fn).to(torch.float64), vals)


def test_e8m0_against_torch():
    b = torch.tensor([1, 100, 125, 126, 127, 128, 200, 254], dtype=torch.uint8)
    ref = b.view(torch.float8_e8m0fnu).to(torch.float64).tolist()
    assert [oracle.e8m0_value(int(x)) for x in b] == ref
    assert np.isnan(oracle.e8m0_value(255))


def _one_row_inputs(HI, dI, qcodes, qscale, kcodes, kscale, wcodes):
    """Build packed tensors from per-element codes (element 2i in the low nibble)."""
    def pack(codes):
        codes = np.asarray(codes, np.uint8)
        return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    qc = pack(np.asarray(qcodes, np.uint8).reshape(1, HI, dI))
    qs = np.asarray(qscale, np.uint8).reshape(1, HI, dI // 32)
    kc = pack(np.asarray(kcodes, np.uint8).reshape(-1, dI))
    ks = np.asarray(kscale, np.uint8).reshape(-1, dI // 32)
    w = np.asarray(wcodes, np.uint8).reshape(1, HI)
    return qc, qs, w, kc, ks


def test_hand_example_two_heads():
    g = json.load(open(os.path.join(GOLD, "hand_indexer.json")))["case_two_heads"]
    HI, dI = g["HI"], g["dI"]
    q = np.stack([np.full(dI, g["q_head0_code"]), np.full(dI, g["q_head1_code"])])
    qs = [[g["q_head0_scale_byte"]], [g["q_head1_scale_byte"]]]
    qc, qsc, w, kc, ks = _one_row_inputs(HI, dI, q, qs, np.full(dI, g["k_code"]), [g["k_scale_byte"]],
                                         g["w_codes"])
    I = oracle.indexer(qc, qsc, w, kc, ks, t0=0, m=1)
    assert I[0, 0] == g["I"]


def test_nibble_order():
    g = json.load(open(os.path.join(GOLD, "hand_indexer.json")))["nibble_order"]
    # query: element 0 = 1.0 only; key byte 0x71 -> its element 0 is 0.5
    q = np.zeros(32, np.uint8)
    q[0] = 2
    kc = np.zeros((1, 16), np.uint8)
    kc[0, 0] = g["byte"]
    qc, qs, w, _, ks = _one_row_inputs(1, 32, q, [127], np.zeros(32), [127], [2])
    assert oracle.indexer(qc, qs, w, kc, ks, 0, 1)[0, 0] == g["element0"]
    q[0], q[1] = 0, 2  # now pick element 1 -> 6.0
    qc, qs, w, _, ks = _one_row_inputs(1, 32, q, [127], np.zeros(32), [127], [2])
    assert oracle.indexer(qc, qs, w, kc, ks, 0, 1)[0, 0] == g["element1"]


def test_all_code_pairs_brute_force():
    """Every (q code, k code) product at every position of a 32-block, against the
    MX table (not the oracle's bit-field decoder)."""
    table = json.load(open(os.path.join(GOLD, "e2m1_table.json")))["values"]
    dI = 32
    for pos in (0, 1, 17, 31):
        for cq in range(16):
            q = np.zeros(dI, np.uint8)
            q[pos] = cq
            kcodes = np.zeros((16, dI), np.uint8)
            kcodes[:, pos] = np.arange(16)
            qc, qs, w, kc, ks = _one_row_inputs(1, dI, q, [127], kcodes, [127] * 16, [2])  # w = 1
            I = oracle.indexer(qc, qs, w, kc, ks, 0, m=1, rows=[0])
            # row t=0 with m=1 sees only j=0; widen visibility by placing the query at t0=15
            I = oracle.indexer(qc, qs, w, kc, ks, 15, m=1, rows=[0])[0]
            want = [max(table[cq] * table[ck], 0.0) for ck in range(16)]
            assert list(I) == want, (pos, cq)


def test_scales_apply_per_32_block_with_bias_127():
    dI = 64
    q = np.full(dI, 2, np.uint8)      # all 1.0
    k = np.full(dI, 2, np.uint8)
    for sb0, sb1 in [(127, 127), (128, 125), (125, 128), (126, 126)]:
        qc, qs, w, kc, ks = _one_row_inputs(1, dI, q, [sb0, sb1], k, [127, 127], [2])
        I = oracle.indexer(qc, qs, w, kc, ks, 0, 1)[0, 0]
        assert I == 32 * 2.0 ** (sb0 - 127) + 32 * 2.0 ** (sb1 - 127)


def test_relu_and_signed_weights():
    dI = 32
    q = np.stack([np.full(dI, 2), np.full(dI, 10), np.full(dI, 2)])  # +1, -1, +1
    k = np.full(dI, 2)
    for wc, want in [([2, 2, 2], 64.0), ([10, 7, 2], 0.0), ([15, 15, 15], -12 * 32.0), ([8, 0, 3], 48.0)]:
        qc, qs, w, kc, ks = _one_row_inputs(3, dI, q, [[127]] * 3, k, [127], wc)
        assert oracle.indexer(qc, qs, w, kc, ks, 0, 1)[0, 0] == want, wc


def test_causal_visibility():
    rng = np.random.default_rng(0)
    T, HI, dI, m = 40, 2, 32, 4
    qc = rng.integers(0, 256, (T, HI, dI // 2), dtype=np.uint8)
    qs = rng.integers(125, 129, (T, HI, 1), dtype=np.uint8)
    w = rng.integers(0, 16, (T, HI), dtype=np.uint8)
    kc = rng.integers(0, 256, (T // m, dI // 2), dtype=np.uint8)
    ks = rng.integers(125, 129, (T // m, 1), dtype=np.uint8)
    I = oracle.indexer(qc, qs, w, kc, ks, 0, m)
    for t in range(T):
        nv = (t + 1) // m
        assert np.all(np.isneginf(I[t, nv:])) and np.all(np.isfinite(I[t, :nv]))
    # t0 shifts visibility: rows are absolute positions t0 + r
    I2 = oracle.indexer(qc, qs, w, kc, ks, 8, m)
    assert np.isfinite(I2[0, 1]) and np.isneginf(I2[0, 2])


def test_topk_tie_example():
    g = json.load(open(os.path.join(GOLD, "topk_ties.json")))
    idx, top = oracle.topk(np.array([g["scores"]], np.float64), [5], g["k"])
    assert idx[0].tolist() == g["idx"]
    assert top[0].tolist() == [g["scores"][j] for j in g["idx"]]


def test_topk_against_sorted_brute_force():
    rng = np.random.default_rng(7)
    n, N, k = 50, 200, 24
    S = rng.integers(-3, 4, (n, N)).astype(np.float64)  # many ties
    nvis = rng.integers(0, N + 1, n)
    idx, top = oracle.topk(S, nvis, k)
    for i in range(n):
        order = sorted(range(nvis[i]), key=lambda j: (-S[i, j], j))[:k]
        want = order + [-1] * (k - len(order))
        assert idx[i].tolist() == want
        assert np.all(np.isneginf(top[i, len(order):]))
