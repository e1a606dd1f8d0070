"""Pins for the oracle's attention: joint softmax over compressed entries and the
raw sliding window.

CSA: blog.nickys.cn/?p=150 section "1. CSA" (attend only to the k selected
compressed entries plus a few sliding-window entries).  HCA: same page section
"2. HCA" (dense over every compressed entry).  Sliding window in both:
sz-guanghua.com.cn ifanr repost, attention section.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def words(x):
    return oracle.to_bf16_words(np.asarray(x, np.float64))


def f64(w):
    return torch.from_numpy(oracle.bf16_words_to_f64(w))


def _rand(shape, rng, scale=1.0):
    return words(rng.standard_normal(shape) * scale)


def test_hand_examples():
    g = json.load(open(os.path.join(GOLD, "hand_compress_attention.json")))
    K = words(np.array(g["K"]).reshape(4, 1))
    V = words(np.array(g["V"]).reshape(4, 1))
    Kc = words(np.array(g["Z_zero"]["Kc"]).reshape(2, 1))
    Vc = words(np.array(g["Z_zero"]["Vc"]).reshape(2, 1))
    a = g["attention"]
    Q = words(np.full((4, 1, 1), a["q"]))
    sel = np.array([[0, 1]], np.int32)
    for case in ("all_blocks_no_window", "all_blocks_window2"):
        c = a[case]
        O, _ = oracle.attention(Q, Kc, Vc, K, V, 0, 2, c["W"], a["scale"], sel=sel, rows=[a["t"]])
        assert O[0, 0, 0] == pytest.approx(c["O"], abs=1e-6)
    e = math.e
    O, _ = oracle.attention(Q, Kc, Vc, K, V, 0, 2, 0, 1.0, sel=sel, rows=[3])
    assert O[0, 0, 0] == pytest.approx((15 * e + 35) / (e + 1), rel=1e-15)


def _sdpa(q, k, v, mask, scale):
    """torch library attention in fp64: q [H,T,d], k/v [S,d] shared (MQA), mask [T,S] bool."""
    H = q.shape[0]
    kk = k.unsqueeze(0).expand(H, -1, -1)
    vv = v.unsqueeze(0).expand(H, -1, -1)
    return F.scaled_dot_product_attention(q, kk, vv, attn_mask=mask, scale=scale)


def test_m1_full_topk_no_window_is_causal_attention():
    rng = np.random.default_rng(0)
    T, H, d = 48, 3, 16
    Q, K, V = _rand((T, H, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    Z = _rand((T, d), rng)
    Kc, Vc = oracle.compress(K, V, Z, np.zeros((1, d), np.float32), 1)
    sel = np.tile(np.arange(T, dtype=np.int32), (T, 1))
    sel = np.where(sel <= np.arange(T)[:, None], sel, -1)
    scale = 1 / math.sqrt(d)
    O, lse = oracle.attention(Q, words(Kc), words(Vc), None, None, 0, 1, 0, scale, sel=sel)
    q = f64(Q).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, f64(K).expand(H, T, d), f64(V).expand(H, T, d), is_causal=True,
                                         scale=scale)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), atol=1e-12)
    logits = torch.einsum("thd,sd->ths", f64(Q), f64(K)) * scale
    logits = logits.masked_fill(torch.arange(T)[None, None, :] > torch.arange(T)[:, None, None], -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).numpy(), atol=1e-12)


def test_all_visible_blocks_no_window_is_causal_attention_over_compressed():
    rng = np.random.default_rng(1)
    T, H, d, m = 64, 2, 8, 4
    Q = _rand((T, H, d), rng)
    Kc, Vc = _rand((T // m, d), rng), _rand((T // m, d), rng)
    scale = 0.3
    t = np.arange(T)
    nv = (t + 1) // m
    rows = np.nonzero(nv > 0)[0]
    O, _ = oracle.attention(Q, Kc, Vc, None, None, 0, m, 0, scale, rows=rows)  # HCA form (sel=None)
    mask = torch.from_numpy(np.arange(T // m)[None, :] < nv[rows][:, None])
    ref = _sdpa(f64(Q)[rows].permute(1, 0, 2), f64(Kc), f64(Vc), mask, scale)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), atol=1e-12)
    # CSA with k >= n_vis selects every visible block: same result
    sel = np.where(np.arange(T // m)[None, :] < nv[rows][:, None], np.arange(T // m)[None, :], -1).astype(np.int32)
    O2, _ = oracle.attention(Q, Kc, Vc, None, None, 0, m, 0, scale, sel=sel, rows=rows)
    np.testing.assert_allclose(O2, O, atol=1e-14)


def test_k0_is_sliding_window_attention():
    rng = np.random.default_rng(2)
    T, H, d, W = 50, 2, 8, 7
    Q, K, V = _rand((T, H, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    scale = 1 / math.sqrt(d)
    sel = np.full((T, 1), -1, np.int32)
    O, _ = oracle.attention(Q, None, None, K, V, 0, 4, W, scale, sel=sel)
    i, s = np.arange(T)[:, None], np.arange(T)[None, :]
    mask = torch.from_numpy((s <= i) & (s > i - W))
    ref = _sdpa(f64(Q).permute(1, 0, 2), f64(K), f64(V), mask, scale)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), atol=1e-12)


def test_joint_softmax_with_window_against_explicit_key_set():
    """Selected compressed entries and window tokens in ONE softmax: equal to
    library attention over the concatenated key list."""
    rng = np.random.default_rng(3)
    T, H, d, m, W, k = 40, 2, 8, 4, 6, 3
    Q, K, V = _rand((T, H, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    Kc, Vc = _rand((T // m, d), rng), _rand((T // m, d), rng)
    scale = 0.5
    sel = np.full((T, k), -1, np.int32)
    for t in range(T):
        nv = (t + 1) // m
        if nv:
            c = rng.choice(nv, size=min(k, nv), replace=False)
            sel[t, : len(c)] = c
    O, lse = oracle.attention(Q, Kc, Vc, K, V, 0, m, W, scale, sel=sel)
    for t in range(T):
        keys = [f64(Kc)[j] for j in sel[t] if j >= 0] + [f64(K)[s] for s in range(max(0, t - W + 1), t + 1)]
        vals = [f64(Vc)[j] for j in sel[t] if j >= 0] + [f64(V)[s] for s in range(max(0, t - W + 1), t + 1)]
        kk, vv = torch.stack(keys), torch.stack(vals)
        ref = _sdpa(f64(Q)[t].unsqueeze(1), kk, vv, None, scale)[:, 0]
        np.testing.assert_allclose(O[t], ref.numpy(), atol=1e-12)
        lg = (f64(Q)[t] @ kk.T) * scale
        np.testing.assert_allclose(lse[t], torch.logsumexp(lg, -1).numpy(), atol=1e-12)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(4)
    T, H, d, m, W = 32, 2, 8, 4, 5
    Q, K = _rand((T, H, d), rng), _rand((T, d), rng)
    ones = words(np.ones((T, d)))
    Kc = _rand((T // m, d), rng)
    Vc1 = words(np.ones((T // m, d)))
    O, _ = oracle.attention(Q, Kc, Vc1, K, ones, 0, m, W, 0.4)
    np.testing.assert_allclose(O, 1.0, atol=1e-14)


def test_future_inputs_do_not_leak():
    rng = np.random.default_rng(5)
    T, H, d, m, W = 40, 2, 8, 4, 6
    Q, K, V = _rand((T, H, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    Kc, Vc = _rand((T // m, d), rng), _rand((T // m, d), rng)
    t = 21
    O, _ = oracle.attention(Q, Kc, Vc, K, V, 0, m, W, 0.4, rows=[t])
    K2, V2, Kc2, Vc2 = K.copy(), V.copy(), Kc.copy(), Vc.copy()
    K2[t + 1:] = words(rng.standard_normal((T - t - 1, d)))
    V2[t + 1:] = words(rng.standard_normal((T - t - 1, d)))
    nv = (t + 1) // m
    Kc2[nv:] = words(rng.standard_normal((T // m - nv, d)))
    Vc2[nv:] = words(rng.standard_normal((T // m - nv, d)))
    O2, _ = oracle.attention(Q, Kc2, Vc2, K2, V2, 0, m, W, 0.4, rows=[t])
    np.testing.assert_array_equal(O, O2)


def test_empty_key_set():
    Q = words(np.ones((2, 1, 4)))
    O, lse = oracle.attention(Q, None, None, None, None, 0, 4, 0, 1.0, sel=np.full((2, 1), -1, np.int32))
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_raw_pos0_offsets_window_rows():
    rng = np.random.default_rng(6)
    T, H, d, W = 30, 1, 4, 5
    Q, K, V = _rand((T, H, d), rng), _rand((T, d), rng), _rand((T, d), rng)
    sel = np.full((1, 1), -1, np.int32)
    t = 20
    O, _ = oracle.attention(Q, None, None, K, V, 0, 4, W, 0.5, sel=sel, rows=[t])
    # same window from a buffer that starts at absolute position t-W+1
    O2, _ = oracle.attention(Q, None, None, K[t - W + 1: t + 1], V[t - W + 1: t + 1], 0, 4, W, 0.5, sel=sel,
                             rows=[t], raw_pos0=t - W + 1)
    np.testing.assert_array_equal(O, O2)
