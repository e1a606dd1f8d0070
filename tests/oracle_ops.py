"""The library's call signatures backed by the CPU oracle (test infrastructure):
lets host-side orchestration (the sharded prefill's exchange) run on CPU ranks
without a GPU.  Outputs are torch tensors of the library's dtypes: compressed
entries as round-to-nearest bf16 of the oracle's fp64 pooling, selections as
int32, attention outputs as bf16."""
import numpy as np
import torch

import oracle


def _bf16(a):
    return torch.from_numpy(oracle.to_bf16_words(a).view(np.int16)).view(torch.bfloat16)


def csa_compress(K, V, Z, B, m, Kc=None, Vc=None):
    Kx, Vx = oracle.compress(K, V, Z, B, m, nthreads=1)
    return _bf16(Kx), _bf16(Vx)


def csa_indexer_topk(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, m, k, t0=0, want_scores=True, **_):
    T = qI_codes.shape[0]
    Nc = kI_codes.shape[0]
    I = oracle.indexer(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, t0, m, nthreads=1)
    nv = np.minimum(oracle.n_vis(t0 + np.arange(T), m), Nc)
    idx, top = oracle.topk(I, nv, k, nthreads=1)
    return torch.from_numpy(idx), (torch.from_numpy(top.astype(np.float32)) if want_scores else None), None


def csa_sparse_attn(Q, Kc, Vc, idx, Kraw, Vraw, W, scale, t0=0, want_lse=True, **_):
    O, lse = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, 1, W, scale, sel=idx.numpy(), nthreads=1)
    return _bf16(O), (torch.from_numpy(lse) if want_lse else None), None


def hca_attn(Q, Kc, Vc, Kraw, Vraw, m, W, scale, t0=0, want_lse=True, **_):
    O, lse = oracle.attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale, nthreads=1)
    return _bf16(O), (torch.from_numpy(lse) if want_lse else None), None


# ------------------------------------------------------------------ split-cache decode pieces
# (candidates travel as float64 [B, k, 2] = (score, global entry), -inf / -1 padding)

def csa_decode_search(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, pos, m, k, j_base=0, **_):
    B = qI_codes.shape[0]
    out = np.zeros((B, k, 2))
    for b in range(B):
        n = kI_codes.shape[1]
        # scores of the slice's entries as positions j_base + local
        I = oracle.indexer(qI_codes[b:b + 1], qI_scales[b:b + 1], w_codes[b:b + 1], kI_codes[b], kI_scales[b],
                           pos[b] - j_base * m, m, nthreads=1)
        nv = min(max(0, (pos[b] + 1) // m - j_base), n)
        idx, top = oracle.topk(I, [nv], k, nthreads=1)
        out[b, :, 0] = top[0]
        out[b, :, 1] = np.where(idx[0] >= 0, idx[0] + j_base, -1)
    return torch.from_numpy(out), None


def csa_topk_merge(lists, k):
    L = lists.numpy()  # [B, L, k, 2]
    B = L.shape[0]
    flat = L.reshape(B, -1, 2)
    idx = np.full((B, k), -1, np.int32)
    sc = np.full((B, k), -np.inf, np.float32)
    for b in range(B):
        c = [(s, int(j)) for s, j in flat[b] if j >= 0]
        c.sort(key=lambda p: (-p[0], p[1]))
        for q, (s, j) in enumerate(c[:k]):
            idx[b, q], sc[b, q] = j, s
    return torch.from_numpy(idx), torch.from_numpy(sc)


def csa_decode_attend(q, Kc, Vc, idx, Kwin, Vwin, pos, m, W, scale, j_base=0, **_):
    B, H, d = q.shape
    O = np.zeros((B, H, d), np.float32)
    lse = np.zeros((B, H), np.float32)
    n = Kc.shape[1]
    for b in range(B):
        sel = idx[b].numpy().astype(np.int64) - j_base
        sel = np.where((idx[b].numpy() >= 0) & (sel >= 0) & (sel < n), sel, -1).astype(np.int32)
        o, l = oracle.attention(q[b:b + 1], Kc[b], Vc[b], Kwin[b] if W else None, Vwin[b] if W else None, pos[b], m,
                                W, scale, sel=sel[None], rows=[0], raw_pos0=pos[b] - (W - 1), nthreads=1)
        O[b], lse[b] = o[0], l[0]
    return torch.from_numpy(O), torch.from_numpy(lse)


def csa_attn_combine(O_parts, lse_parts, out_dtype=None):
    O = O_parts.double().numpy()
    L = lse_parts.double().numpy()
    mx = L.max(axis=0)
    w = np.where(np.isneginf(L), 0.0, np.exp(L - np.where(np.isneginf(mx), 0.0, mx)[None]))
    s = w.sum(axis=0)
    out = (w[..., None] * O).sum(axis=0) / np.where(s > 0, s, 1.0)[..., None]
    lse = np.where(s > 0, mx + np.log(np.where(s > 0, s, 1.0)), -np.inf)
    return torch.from_numpy(out), torch.from_numpy(lse)
