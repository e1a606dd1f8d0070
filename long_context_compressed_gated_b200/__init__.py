"""Python binding of libcsa.so -- the DeepSeek-V4 CSA/HCA hot path on B200.

Argument marshalling only: every step runs in the CUDA kernels of libcsa.so
(declared in include/csa.h).  Functions carry the C ABI names and take torch
tensors that already live on the current CUDA device; outputs are allocated
here when not supplied, scratch memory is a torch uint8 workspace sized by the
library's *_workspace_bytes() query, and work is enqueued on torch's current
stream.  A non-zero status from the library raises CsaError.  There is no CPU
path: importing works without a GPU, but every call needs the CUDA library.
"""
import ctypes
import os

import torch

__all__ = [
    "CsaError", "lib", "csa_compress", "csa_indexer_topk", "csa_sparse_attn", "hca_attn", "csa_decode",
    "hca_decode", "csa_check_status", "csa_status_string", "csa_version", "LIB_PATH", "csa_decode_append",
    "hca_decode_append", "csa_mxfp4_quantize", "csa_mxfp8_quantize", "csa_decode_fp8", "csa_peak_mma",
    "csa_decode_search", "csa_topk_merge", "csa_decode_attend", "csa_attn_combine",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa.so")

_lib = None


class CsaError(RuntimeError):
    def __init__(self, code, what):
        super().__init__("%s failed: %s (status %d)" % (what, csa_status_string(code), code))
        self.code = code


def lib():
    """The loaded libcsa.so. Raises if the CUDA library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libcsa.so not found at %s; build it with "
                               "`python -m long_context_compressed_gated_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        sig = {
            "csa_status_string": ([I], ctypes.c_char_p),
            "csa_last_cuda_error": ([], I),
            "csa_version": ([], I),
            "csa_check_status": ([P, P], I),
            "csa_debug_inject": ([I], I),
            "csa_decode_append": ([P, P, P, P, P, P, P, I, I64, I, I, I, I, P, P, P, P, P, P, P, P, P, P], I),
            "hca_decode_append": ([P, P, P, P, P, I, I64, I, I, I, P, P, P, P, P, P, P, P], I),
            "csa_mxfp4_quantize": ([P, I64, I, I, P, P, P], I),
            "csa_mxfp8_quantize": ([P, I64, I, P, P, P], I),
            "csa_peak_mma": ([I, I64, I, P, SZ, P, P], I),
            "csa_compress": ([P, P, P, P, I64, I, I, P, P, P], I),
            "csa_indexer_topk_workspace_bytes": ([I64, I64, I, I, I], SZ),
            "csa_indexer_topk": ([P, P, P, P, P, I64, I64, I64, I, I, I, I, P, P, P, SZ, P], I),
            "csa_sparse_attn_workspace_bytes": ([I64, I, I, I, I], SZ),
            "csa_sparse_attn": ([P, P, P, P, P, P, I64, I64, I64, I, I, I, I, F, P, I, P, P, SZ, P], I),
            "hca_attn_workspace_bytes": ([I64, I, I, I], SZ),
            "hca_attn": ([P, P, P, P, P, I64, I64, I64, I, I, I, I, F, P, I, P, P, SZ, P], I),
            "csa_decode_workspace_bytes": ([I, I64, I, I, I, I, I, I], SZ),
            "csa_decode": ([P, P, P, P, P, P, P, P, P, P, P, I, I64, I, I, I, I, I, I, I, F, P, I, P, P, P, P, SZ,
                            P], I),
            "csa_decode_fp8": ([P, P, P, P, P, P, P, P, P, P, P, P, P, I, I64, I, I, I, I, I, I, I, F, P, I, P, P, P,
                                P, SZ, P], I),
            "hca_decode_workspace_bytes": ([I, I64, I, I, I], SZ),
            "csa_decode_search_workspace_bytes": ([I, I64, I], SZ),
            "csa_decode_search": ([P, P, P, P, P, P, I, I64, I64, I, I, I, I, P, P, SZ, P], I),
            "csa_topk_merge_workspace_bytes": ([I, I], SZ),
            "csa_topk_merge": ([P, I, I, I, P, P, P, P, SZ, P], I),
            "csa_decode_attend": ([P, P, P, P, I64, P, P, P, I, I64, I, I, I, I, I, F, P, I, P, P, SZ, P], I),
            "csa_attn_combine": ([P, P, I, I, I, I, P, I, P, P], I),
            "hca_decode": ([P, P, P, P, P, P, I, I64, I, I, I, I, F, P, I, P, P, SZ, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def csa_status_string(code):
    return lib().csa_status_string(int(code)).decode()


def csa_version():
    return lib().csa_version()


_ODTYPE = {torch.bfloat16: 0, torch.float32: 1}  # csa_dtype_t


def _out(O, like, shape, out_dtype, name="O"):
    """Output tensor of the given dtype (bf16 or fp32): allocated when O is None."""
    if out_dtype not in _ODTYPE:
        raise TypeError("%s dtype must be torch.bfloat16 or torch.float32" % name)
    if O is None:
        return torch.empty(shape, dtype=out_dtype, device=like.device)
    return _dev(O, out_dtype, name)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %d" % (name, ndim, t.dim()))
    return t


def _check(code, what):
    if code != 0:
        raise CsaError(code, what)


def _workspace(nbytes, device, workspace=None):
    if workspace is not None:
        if workspace.numel() < nbytes:
            raise ValueError("workspace too small: %d < %d bytes" % (workspace.numel(), nbytes))
        return workspace
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:4].zero_()  # status word
    return ws


def csa_check_status(workspace):
    """Synchronise the current stream, return and clear the device status word."""
    return lib().csa_check_status(_ptr(workspace), _stream())


def csa_peak_mma(kind, iters, ctas=None, workspace=None):
    """Enqueue the tensor-pipe peak loop (kind 0 = bf16, 1 = MXFP4) on the current
    stream; returns (flops of the launch, workspace).  ctas defaults to the SM count."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if ctas is None:
        ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    ws = _workspace(256, dev, workspace)
    fl = ctypes.c_double(0.0)
    _check(lib().csa_peak_mma(int(kind), int(iters), int(ctas), _ptr(ws), ws.numel(), ctypes.byref(fl), _stream()),
           "csa_peak_mma")
    return fl.value, ws


MX_OCP, MX_INDEXER = 0, 1


def csa_mxfp4_quantize(x, mode=MX_OCP, codes=None, scales=None):
    """bf16 [..., n] (n % 32 == 0) -> MXFP4 (codes uint8 [..., n/2], scales uint8
    [..., n/32]).  mode MX_INDEXER keeps the scale bytes in 125..128."""
    _dev(x, torch.bfloat16, "x")
    n = x.shape[-1]
    rows = x.numel() // n if n else 0
    lead = tuple(x.shape[:-1])
    codes = torch.empty(lead + (n // 2,), dtype=torch.uint8, device=x.device) if codes is None else \
        _dev(codes, torch.uint8, "codes")
    scales = torch.empty(lead + (n // 32,), dtype=torch.uint8, device=x.device) if scales is None else \
        _dev(scales, torch.uint8, "scales")
    _check(lib().csa_mxfp4_quantize(_ptr(x), rows, n, int(mode), _ptr(codes), _ptr(scales), _stream()),
           "csa_mxfp4_quantize")
    return codes, scales


def csa_mxfp8_quantize(x, codes=None, scales=None):
    """bf16 [..., n] (n % 32 == 0) -> MXFP8 (E4M3 codes uint8 [..., n], E8M0 scales
    uint8 [..., n/32]): the FP8 form of the compressed K/V cache."""
    _dev(x, torch.bfloat16, "x")
    n = x.shape[-1]
    rows = x.numel() // n if n else 0
    lead = tuple(x.shape[:-1])
    codes = torch.empty(lead + (n,), dtype=torch.uint8, device=x.device) if codes is None else \
        _dev(codes, torch.uint8, "codes")
    scales = torch.empty(lead + (n // 32,), dtype=torch.uint8, device=x.device) if scales is None else \
        _dev(scales, torch.uint8, "scales")
    _check(lib().csa_mxfp8_quantize(_ptr(x), rows, n, _ptr(codes), _ptr(scales), _stream()), "csa_mxfp8_quantize")
    return codes, scales


def csa_compress(K, V, Z, B, m, Kc=None, Vc=None):
    """Gated pooling of every complete block of m tokens. K,V,Z [T,d] bf16, B [m,d] f32.
    Returns (Kc, Vc) [T//m, d] bf16."""
    _dev(K, torch.bfloat16, "K", 2), _dev(V, torch.bfloat16, "V", 2), _dev(Z, torch.bfloat16, "Z", 2)
    _dev(B, torch.float32, "B", 2)
    T, d = K.shape
    nb = T // m
    Kc = torch.empty(nb, d, dtype=torch.bfloat16, device=K.device) if Kc is None else _dev(Kc, torch.bfloat16, "Kc")
    Vc = torch.empty(nb, d, dtype=torch.bfloat16, device=K.device) if Vc is None else _dev(Vc, torch.bfloat16, "Vc")
    _check(lib().csa_compress(_ptr(K), _ptr(V), _ptr(Z), _ptr(B), T, d, m, _ptr(Kc), _ptr(Vc), _stream()),
           "csa_compress")
    return Kc, Vc


def csa_indexer_topk(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, m, k, t0=0, idx=None, scores=None,
                     want_scores=True, workspace=None):
    """MXFP4 lightning indexer + causal top-k. Returns (idx [T,k] int32, scores [T,k] f32 or None, workspace)."""
    _dev(qI_codes, torch.uint8, "qI_codes", 3), _dev(qI_scales, torch.uint8, "qI_scales", 3)
    _dev(w_codes, torch.uint8, "w_codes", 2), _dev(kI_codes, torch.uint8, "kI_codes", 2)
    _dev(kI_scales, torch.uint8, "kI_scales", 2)
    T, HI, half = qI_codes.shape
    dI = half * 2
    Nc = kI_codes.shape[0]
    dev = qI_codes.device
    idx = torch.empty(T, k, dtype=torch.int32, device=dev) if idx is None else _dev(idx, torch.int32, "idx")
    if want_scores and scores is None:
        scores = torch.empty(T, k, dtype=torch.float32, device=dev)
    elif scores is not None:
        _dev(scores, torch.float32, "scores")
    ws = _workspace(lib().csa_indexer_topk_workspace_bytes(T, Nc, HI, dI, k), dev, workspace)
    _check(lib().csa_indexer_topk(_ptr(qI_codes), _ptr(qI_scales), _ptr(w_codes), _ptr(kI_codes), _ptr(kI_scales),
                                  T, t0, Nc, HI, dI, m, k, _ptr(idx), _ptr(scores), _ptr(ws), ws.numel(),
                                  _stream()), "csa_indexer_topk")
    return idx, scores, ws


def csa_sparse_attn(Q, Kc, Vc, idx, Kraw, Vraw, W, scale, t0=0, O=None, lse=None, want_lse=True, workspace=None,
                    out_dtype=torch.bfloat16):
    """CSA attention over the selected entries plus the raw window. Returns (O, lse, workspace).
    out_dtype: torch.bfloat16 (default) or torch.float32 for O."""
    _dev(Q, torch.bfloat16, "Q", 3), _dev(Kc, torch.bfloat16, "Kc", 2), _dev(Vc, torch.bfloat16, "Vc", 2)
    _dev(idx, torch.int32, "idx", 2), _dev(Kraw, torch.bfloat16, "Kraw", 2), _dev(Vraw, torch.bfloat16, "Vraw", 2)
    T, H, d = Q.shape
    k = idx.shape[1]
    dev = Q.device
    O = _out(O, Q, Q.shape, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    ws = _workspace(lib().csa_sparse_attn_workspace_bytes(T, H, d, k, W), dev, workspace)
    _check(lib().csa_sparse_attn(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(idx), _ptr(Kraw), _ptr(Vraw), T, t0,
                                 Kc.shape[0], H, d, k, W, float(scale), _ptr(O), _ODTYPE[out_dtype], _ptr(lse),
                                 _ptr(ws), ws.numel(), _stream()), "csa_sparse_attn")
    return O, lse, ws


def hca_attn(Q, Kc, Vc, Kraw, Vraw, m, W, scale, t0=0, O=None, lse=None, want_lse=True, workspace=None,
             out_dtype=torch.bfloat16):
    """HCA attention over every visible compressed entry plus the raw window. Returns (O, lse, workspace).
    out_dtype: torch.bfloat16 (default) or torch.float32 for O."""
    _dev(Q, torch.bfloat16, "Q", 3), _dev(Kc, torch.bfloat16, "Kc", 2), _dev(Vc, torch.bfloat16, "Vc", 2)
    _dev(Kraw, torch.bfloat16, "Kraw", 2), _dev(Vraw, torch.bfloat16, "Vraw", 2)
    T, H, d = Q.shape
    dev = Q.device
    O = _out(O, Q, Q.shape, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    ws = _workspace(lib().hca_attn_workspace_bytes(T, H, d, W), dev, workspace)
    _check(lib().hca_attn(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(Kraw), _ptr(Vraw), T, t0, Kc.shape[0], H, d, m, W,
                          float(scale), _ptr(O), _ODTYPE[out_dtype], _ptr(lse), _ptr(ws), ws.numel(), _stream()),
           "hca_attn")
    return O, lse, ws


def csa_decode(q, qI_codes, qI_scales, w_codes, Kc, Vc, kI_codes, kI_scales, Kwin, Vwin, pos, m, k, scale,
               O=None, lse=None, idx=None, scores=None, want_lse=True, want_sel=True, workspace=None,
               out_dtype=torch.bfloat16):
    """One new token per sequence against its compressed cache (indexer, top-k,
    sparse + window attention). pos: list of absolute positions (host).
    Returns (O [B,H,d], lse, idx [B,k], scores [B,k], workspace)."""
    _dev(q, torch.bfloat16, "q", 3), _dev(qI_codes, torch.uint8, "qI_codes", 3)
    _dev(qI_scales, torch.uint8, "qI_scales", 3), _dev(w_codes, torch.uint8, "w_codes", 2)
    _dev(Kc, torch.bfloat16, "Kc", 3), _dev(Vc, torch.bfloat16, "Vc", 3)
    _dev(kI_codes, torch.uint8, "kI_codes", 3), _dev(kI_scales, torch.uint8, "kI_scales", 3)
    _dev(Kwin, torch.bfloat16, "Kwin", 3), _dev(Vwin, torch.bfloat16, "Vwin", 3)
    B, H, d = q.shape
    HI, dI = qI_codes.shape[1], qI_codes.shape[2] * 2
    Ncap = Kc.shape[1]
    W = Kwin.shape[1]
    dev = q.device
    O = _out(O, q, q.shape, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    if want_sel:
        idx = torch.empty(B, k, dtype=torch.int32, device=dev) if idx is None else idx
        scores = torch.empty(B, k, dtype=torch.float32, device=dev) if scores is None else scores
    posa = (ctypes.c_int64 * B)(*[int(p) for p in pos])
    ws = _workspace(lib().csa_decode_workspace_bytes(B, Ncap, H, d, HI, dI, k, W), dev, workspace)
    _check(lib().csa_decode(_ptr(q), _ptr(qI_codes), _ptr(qI_scales), _ptr(w_codes), _ptr(Kc), _ptr(Vc),
                            _ptr(kI_codes), _ptr(kI_scales), _ptr(Kwin), _ptr(Vwin), posa, B, Ncap, H, d, HI, dI,
                            m, k, W, float(scale), _ptr(O), _ODTYPE[out_dtype], _ptr(lse), _ptr(idx),
                            _ptr(scores), _ptr(ws), ws.numel(), _stream()), "csa_decode")
    return O, lse, idx, scores, ws


def csa_decode_fp8(q, qI_codes, qI_scales, w_codes, Kc_codes, Kc_scales, Vc_codes, Vc_scales, kI_codes, kI_scales,
                   Kwin, Vwin, pos, m, k, scale, O=None, lse=None, idx=None, scores=None, want_lse=True,
                   want_sel=True, workspace=None, out_dtype=torch.bfloat16):
    """csa_decode over an MXFP8 compressed cache: Kc/Vc codes [B,Ncap,d] uint8 (E4M3)
    and scales [B,Ncap,d/32] uint8 (E8M0).  Returns (O, lse, idx, scores, workspace)."""
    _dev(q, torch.bfloat16, "q", 3), _dev(qI_codes, torch.uint8, "qI_codes", 3)
    _dev(qI_scales, torch.uint8, "qI_scales", 3), _dev(w_codes, torch.uint8, "w_codes", 2)
    for t, n in ((Kc_codes, "Kc_codes"), (Kc_scales, "Kc_scales"), (Vc_codes, "Vc_codes"), (Vc_scales, "Vc_scales"),
                 (kI_codes, "kI_codes"), (kI_scales, "kI_scales")):
        _dev(t, torch.uint8, n, 3)
    _dev(Kwin, torch.bfloat16, "Kwin", 3), _dev(Vwin, torch.bfloat16, "Vwin", 3)
    B, H, d = q.shape
    HI, dI = qI_codes.shape[1], qI_codes.shape[2] * 2
    Ncap = Kc_codes.shape[1]
    W = Kwin.shape[1]
    dev = q.device
    O = _out(O, q, q.shape, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    if want_sel:
        idx = torch.empty(B, k, dtype=torch.int32, device=dev) if idx is None else idx
        scores = torch.empty(B, k, dtype=torch.float32, device=dev) if scores is None else scores
    posa = (ctypes.c_int64 * B)(*[int(p) for p in pos])
    ws = _workspace(lib().csa_decode_workspace_bytes(B, Ncap, H, d, HI, dI, k, W), dev, workspace)
    _check(lib().csa_decode_fp8(_ptr(q), _ptr(qI_codes), _ptr(qI_scales), _ptr(w_codes), _ptr(Kc_codes),
                                _ptr(Kc_scales), _ptr(Vc_codes), _ptr(Vc_scales), _ptr(kI_codes), _ptr(kI_scales),
                                _ptr(Kwin), _ptr(Vwin), posa, B, Ncap, H, d, HI, dI, m, k, W, float(scale), _ptr(O),
                                _ODTYPE[out_dtype], _ptr(lse), _ptr(idx), _ptr(scores), _ptr(ws), ws.numel(),
                                _stream()), "csa_decode_fp8")
    return O, lse, idx, scores, ws


def hca_decode(q, Kc, Vc, Kwin, Vwin, pos, m, scale, O=None, lse=None, want_lse=True, workspace=None,
               out_dtype=torch.bfloat16):
    """HCA decode: one token per sequence, dense over its visible cache + window."""
    _dev(q, torch.bfloat16, "q", 3), _dev(Kc, torch.bfloat16, "Kc", 3), _dev(Vc, torch.bfloat16, "Vc", 3)
    _dev(Kwin, torch.bfloat16, "Kwin", 3), _dev(Vwin, torch.bfloat16, "Vwin", 3)
    B, H, d = q.shape
    Ncap, W = Kc.shape[1], Kwin.shape[1]
    dev = q.device
    O = _out(O, q, q.shape, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    posa = (ctypes.c_int64 * B)(*[int(p) for p in pos])
    ws = _workspace(lib().hca_decode_workspace_bytes(B, Ncap, H, d, W), dev, workspace)
    _check(lib().hca_decode(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(Kwin), _ptr(Vwin), posa, B, Ncap, H, d, m, W,
                            float(scale), _ptr(O), _ODTYPE[out_dtype], _ptr(lse), _ptr(ws), ws.numel(), _stream()),
           "hca_decode")
    return O, lse, ws


def csa_decode_append(K_new, V_new, Z_new, B, pos, Kwin, Vwin, Kblk, Vblk, Zblk, Kc, Vc, kI_codes_new=None,
                      kI_scales_new=None, kI_codes=None, kI_scales=None):
    """Append one token per sequence to the decode state (window, block staging,
    and on block completion the compressed entry and its indexer key), in place.
    K_new/V_new/Z_new [Bseq,d] bf16; B [m,d] f32; pos: host positions of the new
    tokens; Kwin/Vwin [Bseq,W,d]; Kblk/Vblk/Zblk [Bseq,m,d]; Kc/Vc [Bseq,Ncap,d];
    kI_* (all or none): the completed entry's MXFP4 key [Bseq,dI/2]/[Bseq,dI/32]
    and the cache's key tensors [Bseq,Ncap,dI/2]/[Bseq,Ncap,dI/32]."""
    for t, n in ((K_new, "K_new"), (V_new, "V_new"), (Z_new, "Z_new"), (Kwin, "Kwin"), (Vwin, "Vwin"),
                 (Kblk, "Kblk"), (Vblk, "Vblk"), (Zblk, "Zblk"), (Kc, "Kc"), (Vc, "Vc")):
        _dev(t, torch.bfloat16, n)
    _dev(B, torch.float32, "B", 2)
    nb, d = K_new.shape
    m = Kblk.shape[1]
    W = Kwin.shape[1]
    Ncap = Kc.shape[1]
    posa = (ctypes.c_int64 * nb)(*[int(p) for p in pos])
    dI = 0
    if kI_codes is not None:
        for t, n in ((kI_codes_new, "kI_codes_new"), (kI_scales_new, "kI_scales_new"), (kI_codes, "kI_codes"),
                     (kI_scales, "kI_scales")):
            _dev(t, torch.uint8, n)
        dI = kI_codes.shape[-1] * 2
    _check(lib().csa_decode_append(_ptr(K_new), _ptr(V_new), _ptr(Z_new), _ptr(B), _ptr(kI_codes_new),
                                   _ptr(kI_scales_new), posa, nb, Ncap, d, dI, m, W, _ptr(Kwin), _ptr(Vwin),
                                   _ptr(Kblk), _ptr(Vblk), _ptr(Zblk), _ptr(Kc), _ptr(Vc), _ptr(kI_codes),
                                   _ptr(kI_scales), _stream()), "csa_decode_append")


def hca_decode_append(K_new, V_new, Z_new, B, pos, Kwin, Vwin, Kblk, Vblk, Zblk, Kc, Vc):
    """csa_decode_append without indexer keys (the HCA layer's cache, ratio m')."""
    csa_decode_append(K_new, V_new, Z_new, B, pos, Kwin, Vwin, Kblk, Vblk, Zblk, Kc, Vc)


def csa_decode_search(qI_codes, qI_scales, w_codes, kI_codes, kI_scales, pos, m, k, j_base=0, keys=None,
                      workspace=None):
    """The k best entries of a cache slice (global indices j_base + local) as exact
    uint64 keys [B, k] (torch.int64 storage; 0 = none).  Returns (keys, workspace)."""
    B, HI, half = qI_codes.shape
    dI = half * 2
    Nloc = kI_codes.shape[1]
    dev = qI_codes.device
    keys = torch.empty(B, k, dtype=torch.int64, device=dev) if keys is None else _dev(keys, torch.int64, "keys")
    posa = (ctypes.c_int64 * B)(*[int(p) for p in pos])
    ws = _workspace(lib().csa_decode_search_workspace_bytes(B, Nloc, k), dev, workspace)
    _check(lib().csa_decode_search(_ptr(qI_codes), _ptr(qI_scales), _ptr(w_codes), _ptr(kI_codes), _ptr(kI_scales),
                                   posa, B, Nloc, int(j_base), HI, dI, m, k, _ptr(keys), _ptr(ws), ws.numel(),
                                   _stream()), "csa_decode_search")
    return keys, ws


def csa_topk_merge(keys, k, idx=None, scores=None, workspace=None):
    """keys [B, L, k] (int64 storage of the uint64 keys) -> (idx [B,k], scores [B,k])."""
    _dev(keys, torch.int64, "keys", 3)
    B, L, kk = keys.shape
    assert kk == k
    dev = keys.device
    idx = torch.empty(B, k, dtype=torch.int32, device=dev) if idx is None else idx
    scores = torch.empty(B, k, dtype=torch.float32, device=dev) if scores is None else scores
    ws = _workspace(lib().csa_topk_merge_workspace_bytes(B, L), dev, workspace)
    _check(lib().csa_topk_merge(_ptr(keys), B, L, k, _ptr(idx), _ptr(scores), None, _ptr(ws), ws.numel(), _stream()),
           "csa_topk_merge")
    return idx, scores


def csa_decode_attend(q, Kc, Vc, idx, Kwin, Vwin, pos, m, W, scale, j_base=0, O=None, lse=None,
                      out_dtype=torch.float32, workspace=None):
    """Attention over the selected entries inside a cache slice [B, Nloc, d] (+ the
    window when W > 0).  Returns (O, lse) for merging with csa_attn_combine."""
    B, H, d = q.shape
    Nloc = Kc.shape[1]
    k = idx.shape[1]
    dev = q.device
    O = _out(O, q, q.shape, out_dtype)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev) if lse is None else lse
    posa = (ctypes.c_int64 * B)(*[int(p) for p in pos])
    ws = _workspace(lib().csa_decode_workspace_bytes(B, Nloc, H, d, 16, 128, k, W), dev, workspace)
    _check(lib().csa_decode_attend(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(idx), int(j_base), _ptr(Kwin) if W else None,
                                   _ptr(Vwin) if W else None, posa, B, Nloc, H, d, m, k, W, float(scale), _ptr(O),
                                   _ODTYPE[out_dtype], _ptr(lse), _ptr(ws), ws.numel(), _stream()),
           "csa_decode_attend")
    return O, lse


def csa_attn_combine(O_parts, lse_parts, out_dtype=torch.bfloat16, O=None, lse=None):
    """O_parts [L, B, H, d] f32, lse_parts [L, B, H] f32 -> (O [B, H, d], lse [B, H])."""
    _dev(O_parts, torch.float32, "O_parts", 4), _dev(lse_parts, torch.float32, "lse_parts", 3)
    L, B, H, d = O_parts.shape
    O = _out(O, O_parts, (B, H, d), out_dtype)
    lse = torch.empty(B, H, dtype=torch.float32, device=O_parts.device) if lse is None else lse
    _check(lib().csa_attn_combine(_ptr(O_parts), _ptr(lse_parts), L, B, H, d, _ptr(O), _ODTYPE[out_dtype], _ptr(lse),
                                  _stream()), "csa_attn_combine")
    return O, lse
