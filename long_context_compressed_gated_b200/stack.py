"""Chunked causal prefill of an alternating two-layer stack: a CSA layer, then an
HCA layer (blog.nickys.cn/?p=150 "1. CSA"/"2. HCA" and the hybrid interleaving
of CSA and HCA layers described there; ferris-liu.github.io ... deepseek-v4
section 3, architecture).

Per chunk of C tokens (positions c*C .. c*C+C-1, C a multiple of both ratios):
  layer 1  csa_compress appends the chunk's C/m entries to the CSA cache,
           csa_indexer_topk scores the chunk's queries against every entry so
           far, csa_sparse_attn attends to the selection plus the window;
  glue     Q2[t,h] = bf16(O1[t,h] @ P)  (one d x d projection shared by all
           heads; outside the method, a torch matmul);
  layer 2  csa_compress appends C/m' entries to the HCA cache, hca_attn attends
           densely to every visible entry plus the window.
Only argument plumbing happens here: every step of the method runs in libcsa.
"""
import math

import torch

from . import csa_compress, csa_indexer_topk, csa_sparse_attn, hca_attn, lib


def stack_prefill_chunked(l1, l2, P, chunk, m, k, W, m2, W2, scale=None, out=None, phase_events=None,
                          return_o1=False, idx_out=None, scores_out=None):
    """Run the two-layer stack over all T tokens in chunks of `chunk`.

    l1: dict with Q [T,H,d], K, V, Z [T,d], B [m,d], qI_codes [T,HI,dI/2],
        qI_scales [T,HI,dI/32], w_codes [T,HI], kI_codes [T/m,dI/2], kI_scales.
    l2: dict with K, V, Z [T,d], B [m2,d].   P: [d,d] bf16.
    Returns O2 [T,H,d] (and O1 when return_o1).  phase_events: optional list that
    receives (name, start_event, end_event) per phase for timing.  idx_out [T,k]
    int32 / scores_out [T,k] f32 (optional): keep every chunk's layer-1 selection
    (the indexer writes its rows there instead of a per-chunk buffer).
    """
    Q1 = l1["Q"]
    T, H, d = Q1.shape
    assert T % chunk == 0 and chunk % m == 0 and chunk % m2 == 0
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dev = Q1.device
    Kc1 = torch.empty(T // m, d, dtype=torch.bfloat16, device=dev)
    Vc1 = torch.empty_like(Kc1)
    Kc2 = torch.empty(T // m2, d, dtype=torch.bfloat16, device=dev)
    Vc2 = torch.empty_like(Kc2)
    idx_chunk = torch.empty(chunk, k, dtype=torch.int32, device=dev) if idx_out is None else None
    O1 = torch.empty_like(Q1)
    Q2 = torch.empty_like(Q1)
    O2 = torch.empty_like(Q1) if out is None else out
    L = lib()
    HI, dI = l1["qI_scales"].shape[1], l1["qI_scales"].shape[2] * 32
    ws_bytes = max(L.csa_indexer_topk_workspace_bytes(chunk, T // m, HI, dI, k),
                   L.csa_sparse_attn_workspace_bytes(chunk, H, d, k, W), L.hca_attn_workspace_bytes(chunk, H, d, W2))
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)

    def timed(name, fn):
        if phase_events is None:
            return fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        r = fn()
        e1.record()
        phase_events.append((name, e0, e1))
        return r

    for c in range(T // chunk):
        t0 = c * chunk
        sl = slice(t0, t0 + chunk)
        b1, e1 = t0 // m, (t0 + chunk) // m
        b2, e2 = t0 // m2, (t0 + chunk) // m2
        idx = idx_chunk if idx_out is None else idx_out[sl]
        sc = None if scores_out is None else scores_out[sl]
        # layer 1 (CSA)
        timed("compress", lambda: csa_compress(l1["K"][sl], l1["V"][sl], l1["Z"][sl], l1["B"], m, Kc=Kc1[b1:e1],
                                               Vc=Vc1[b1:e1]))
        timed("indexer_topk", lambda: csa_indexer_topk(l1["qI_codes"][sl], l1["qI_scales"][sl], l1["w_codes"][sl],
                                                       l1["kI_codes"][:e1], l1["kI_scales"][:e1], m, k, t0=t0,
                                                       idx=idx, scores=sc, want_scores=sc is not None,
                                                       workspace=ws))
        timed("sparse_attn", lambda: csa_sparse_attn(Q1[sl], Kc1[:e1], Vc1[:e1], idx, l1["K"][: t0 + chunk],
                                                     l1["V"][: t0 + chunk], W, scale, t0=t0, O=O1[sl],
                                                     want_lse=False, workspace=ws))
        # glue: per-head projection of the layer-1 output into the layer-2 queries
        timed("projection", lambda: torch.matmul(O1[sl].view(-1, d), P, out=Q2[sl].view(-1, d)))
        # layer 2 (HCA)
        timed("compress", lambda: csa_compress(l2["K"][sl], l2["V"][sl], l2["Z"][sl], l2["B"], m2, Kc=Kc2[b2:e2],
                                               Vc=Vc2[b2:e2]))
        timed("hca_attn", lambda: hca_attn(Q2[sl], Kc2[:e2], Vc2[:e2], l2["K"][: t0 + chunk],
                                           l2["V"][: t0 + chunk], m2, W2, scale, t0=t0, O=O2[sl], want_lse=False,
                                           workspace=ws))
    return (O2, O1) if return_o1 else O2


def stack_inputs(wl, device="cpu"):
    """Seeded inputs of the two-layer stack (layer-2 K/V/Z/B independent of layer 1)."""
    from . import inputs
    l1 = inputs.prefill_layer(wl, device=device, prefix="l1.")
    l2full = inputs.prefill_layer(wl, device=device, prefix="l2.", with_indexer=False, with_q=False)
    l2 = {"K": l2full["K"], "V": l2full["V"], "Z": l2full["Z"], "B": l2full["B_hca"]}
    del l2full
    P = inputs.projection(wl, device=device)
    return l1, l2, P
