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
