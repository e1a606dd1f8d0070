"""CPU oracle for the CSA / HCA hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 reference written from the DeepSeek-V4 pages (CSA: compress
m tokens into one entry, lightning indexer on MXFP4, causal top-k, attention over
the selection plus a sliding window; HCA: ratio m' >> m, dense over every visible
compressed entry plus the window).  Only the tests, ``__graft_entry__.smoke()``
and the benchmark's ``cpu_baseline`` / ``--impl reference`` leg may use it; the
library never does.  It shares no code with the CUDA path.

The arithmetic lives in ``csa_oracle.c`` (fp64, libm exp); this module only
marshals numpy arrays through ctypes and composes the steps:

  compress        -- per-channel softmax-gated pooling, weights exp(Z + B[i mod m])
  indexer         -- I[t,j] = sum_h w[t,h] * ReLU(qI[t,h] . kI[j]) on MXFP4, exact
  topk            -- k largest visible I[t,j], ties -> smaller j, pad -1 / -inf
  attention       -- one joint softmax over selected (or all visible) compressed
                     entries and the raw window [max(0,t-W+1), t]
  mxfp4_quantize  -- bf16 -> MXFP4 by the OCP MX scale rule (E8M0 per 32, E2M1
                     nearest with ties to even, saturating)
  mxfp8_quantize  -- bf16 -> MXFP8 (E4M3 + E8M0 per 32) for the FP8 compressed
                     cache; mxfp8_dequantize decodes it
  csa_layer       -- compress, indexer, top-k and attention composed for rows
Decode is the same steps for one query row at the sequence's position; the
tests compose it from these functions.

Parity status of each function is stated in its docstring; every function here
is pinned by tests/test_oracle_*.py against hand-worked values, closed forms,
torch library attention, or invariants.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_compress.argtypes = [P, P, P, P, ctypes.c_long, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int]
        L.oracle_indexer.argtypes = [P, P, P, P, P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, P, ctypes.c_long, P, ctypes.c_int]
        L.oracle_topk.argtypes = [P, ctypes.c_long, ctypes.c_long, P, ctypes.c_int, P, P, ctypes.c_int]
        L.oracle_attention.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_long, ctypes.c_int, P,
                                       ctypes.c_int, P, P, ctypes.c_long, ctypes.c_long, ctypes.c_long, P,
                                       ctypes.c_long, ctypes.c_double, P, P, ctypes.c_int]
        L.oracle_mxfp4_quantize.argtypes = [P, ctypes.c_long, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_mxfp8_quantize.argtypes = [P, ctypes.c_long, ctypes.c_int, P, P]
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e8m0_value.argtypes = [ctypes.c_int]
        L.oracle_e8m0_value.restype = ctypes.c_double
        _lib = L
    return _lib


def default_threads():
    return max(1, len(os.sched_getaffinity(0)))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(x):
    """bf16 storage words as a contiguous uint16 array (accepts torch bf16 or numpy uint16)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.asarray(x)
    assert a.dtype == np.uint16, a.dtype
    return np.ascontiguousarray(a)


def _u8(x):
    if hasattr(x, "numpy"):
        x = x.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(np.asarray(x))
    assert a.dtype == np.uint8, a.dtype
    return a


def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e8m0_value(byte):
    return lib().oracle_e8m0_value(int(byte))


def n_vis(t, m):
    """Number of compressed entries visible to absolute position t: block j covers
    [j*m, j*m+m-1] and is visible when j*m+m-1 <= t."""
    return (np.asarray(t, dtype=np.int64) + 1) // m


def compress(K, V, Z, B, m, nthreads=None):
    """Softmax-gated per-channel pooling of K and V over blocks of m tokens.
    K, V, Z: [T, d] bf16; B: [m, d] float32.  Returns (Kc, Vc) float64 [T//m, d]."""
    K, V, Z = _u16(K), _u16(V), _u16(Z)
    B = np.ascontiguousarray(np.asarray(B.cpu().numpy() if hasattr(B, "cpu") else B, dtype=np.float32))
    T, d = K.shape
    assert B.shape == (m, d)
    nb = T // m
    Kc = np.zeros((nb, d), np.float64)
    Vc = np.zeros((nb, d), np.float64)
    rc = lib().oracle_compress(_p(K), _p(V), _p(Z), _p(B), T, d, m, _p(Kc), _p(Vc), nthreads or default_threads())
    assert rc == 0
    return Kc, Vc


def indexer(q_codes, q_scales, w_codes, k_codes, k_scales, t0, m, rows=None, nthreads=None):
    """Exact lightning-indexer scores (float64) for the given local query rows.
    q_codes [T,HI,dI/2] u8, q_scales [T,HI,dI/32] u8, w_codes [T,HI] u8,
    k_codes [Nc,dI/2] u8, k_scales [Nc,dI/32] u8.  Returns I [len(rows), Nc] with
    -inf where j >= n_vis(t0 + row)."""
    qc, qs, wc, kc, ks = _u8(q_codes), _u8(q_scales), _u8(w_codes), _u8(k_codes), _u8(k_scales)
    T, HI, half = qc.shape
    dI = half * 2
    Nc = kc.shape[0]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(np.asarray(rows, np.int64))
    out = np.zeros((len(rows), Nc), np.float64)
    rc = lib().oracle_indexer(_p(qc), _p(qs), _p(wc), _p(kc), _p(ks), t0, Nc, HI, dI, m, _p(rows), len(rows),
                              _p(out), nthreads or default_threads())
    assert rc == 0
    return out


def topk(scores, nvis, k, nthreads=None):
    """Top-k per row over the first nvis[i] entries; ties -> smaller index.
    Returns (idx int32 [n,k] with -1 padding, top float64 [n,k] with -inf padding)."""
    S = np.ascontiguousarray(np.asarray(scores, np.float64))
    n, Nc = S.shape
    nv = np.ascontiguousarray(np.broadcast_to(np.asarray(nvis, np.int64), (n,)).copy())
    idx = np.zeros((n, k), np.int32)
    top = np.zeros((n, k), np.float64)
    rc = lib().oracle_topk(_p(S), n, Nc, _p(nv), k, _p(idx), _p(top), nthreads or default_threads())
    assert rc == 0
    return idx, top


def attention(Q, Kc, Vc, Kraw, Vraw, t0, m, W, scale, sel=None, rows=None, raw_pos0=0, nthreads=None):
    """Joint-softmax attention over compressed entries plus the raw window.
    Q [T,H,d] bf16; Kc,Vc [Nc,d] bf16; Kraw,Vraw bf16 rows for absolute positions
    raw_pos0...; sel [len(rows), nsel] int32 (-1 = unused) or None for every
    visible entry (HCA).  Returns (O float64 [n,H,d], lse float64 [n,H])."""
    Qa = _u16(Q)
    T, H, d = Qa.shape
    Kca = _u16(Kc).reshape(-1, d) if Kc is not None else np.zeros((0, d), np.uint16)
    Vca = _u16(Vc).reshape(-1, d) if Vc is not None else np.zeros((0, d), np.uint16)
    Nc = Kca.shape[0]
    Kr = _u16(Kraw).reshape(-1, d) if Kraw is not None else None
    Vr = _u16(Vraw).reshape(-1, d) if Vraw is not None else None
    rows = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(np.asarray(rows, np.int64))
    n = len(rows)
    if sel is not None:
        sel = np.ascontiguousarray(np.asarray(sel, np.int32)).reshape(n, -1)
        nsel = sel.shape[1]
    else:
        nsel = 0
    O = np.zeros((n, H, d), np.float64)
    lse = np.zeros((n, H), np.float64)
    rc = lib().oracle_attention(_p(Qa), H, d, _p(Kca), _p(Vca), Nc, m, _p(sel), nsel, _p(Kr), _p(Vr), raw_pos0,
                                W, t0, _p(rows), n, float(scale), _p(O), _p(lse), nthreads or default_threads())
    assert rc == 0
    return O, lse


def csa_layer(inp, m, k, W, scale, rows=None, Kc=None, Vc=None, nthreads=None):
    """Whole CSA prefill for the given rows: compress (unless Kc/Vc given as bf16),
    indexer, top-k, attention.  `inp` holds Q,K,V,Z,B,qI_codes,qI_scales,w_codes,
    kI_codes,kI_scales.  Returns dict with Kc/Vc (float64 or the given bf16), idx,
    top, O, lse."""
    T = inp["Q"].shape[0]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = {}
    if Kc is None:
        Kc64, Vc64 = compress(inp["K"], inp["V"], inp["Z"], inp["B"], m, nthreads)
        out["Kc"], out["Vc"] = Kc64, Vc64
        Kc, Vc = to_bf16_words(Kc64), to_bf16_words(Vc64)
    I = indexer(inp["qI_codes"], inp["qI_scales"], inp["w_codes"], inp["kI_codes"], inp["kI_scales"], 0, m, rows,
                nthreads)
    idx, top = topk(I, n_vis(rows, m), k, nthreads)
    O, lse = attention(inp["Q"], Kc, Vc, inp["K"], inp["V"], 0, m, W, scale, sel=idx, rows=rows, nthreads=nthreads)
    out.update(idx=idx, top=top, O=O, lse=lse, I=I)
    return out


def mxfp4_quantize(x, mode=0):
    """bf16 [rows, n] -> (codes uint8 [rows, n/2], scales uint8 [rows, n/32]) by
    the OCP MX rule: per 32-element block X = floor(log2 max|x|) - 2, codes the
    E2M1 values nearest to x / 2^X (ties to even, saturating at 6, sign kept).
    mode 1 clamps X to [-2, 1] (scale bytes 125..128)."""
    xa = _u16(x)
    shape = xa.shape
    n = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    xa = np.ascontiguousarray(xa.reshape(rows, n))
    codes = np.zeros((rows, n // 2), np.uint8)
    scales = np.zeros((rows, n // 32), np.uint8)
    rc = lib().oracle_mxfp4_quantize(_p(xa), rows, n, mode, _p(codes), _p(scales))
    assert rc == 0
    return codes.reshape(shape[:-1] + (n // 2,)), scales.reshape(shape[:-1] + (n // 32,))


def mxfp8_quantize(x):
    """bf16 [rows, n] -> (E4M3 codes uint8 [rows, n], E8M0 scales uint8 [rows, n/32])
    by the OCP MX rule: per 32-element block X = floor(log2 max|x|) - 8, codes the
    E4M3 values nearest to x / 2^X (ties to even, saturating at 448, sign kept)."""
    xa = _u16(x)
    shape = xa.shape
    n = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    xa = np.ascontiguousarray(xa.reshape(rows, n))
    codes = np.zeros((rows, n), np.uint8)
    scales = np.zeros((rows, n // 32), np.uint8)
    rc = lib().oracle_mxfp8_quantize(_p(xa), rows, n, _p(codes), _p(scales))
    assert rc == 0
    return codes.reshape(shape), scales.reshape(shape[:-1] + (n // 32,))


def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def mxfp8_dequantize(codes, scales):
    """E4M3 codes [..., n] and E8M0 scales [..., n/32] -> float64 values."""
    c = np.asarray(codes.cpu().numpy() if hasattr(codes, "cpu") else codes)
    s = np.asarray(scales.cpu().numpy() if hasattr(scales, "cpu") else scales)
    table = np.array([e4m3_value(i) for i in range(256)])
    sv = np.array([e8m0_value(b) for b in range(256)])
    return table[c] * np.repeat(sv[s], 32, axis=-1)


def to_bf16_words(x):
    """Round float64 values straight to bf16 (8 significant bits, round to nearest,
    ties to even; normal range) and return the uint16 storage words."""
    x = np.asarray(x, np.float64)
    mant, ex = np.frexp(x)                      # x = mant * 2**ex, 0.5 <= |mant| < 1
    r = np.ldexp(np.rint(np.ldexp(mant, 8)), ex - 8)   # np.rint rounds half to even
    f = np.ascontiguousarray(r.astype(np.float32))     # exact: r has 8 significant bits
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_words_to_f64(w):
    w = np.asarray(w, np.uint16).astype(np.uint32) << 16
    return w.view(np.float32).astype(np.float64)
