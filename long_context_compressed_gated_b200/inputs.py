"""Seeded synthetic inputs for the CSA / HCA hot path.

This module holds no arithmetic of the method: it only draws random tensors with
the shapes and value distributions of the five workloads, so that the CUDA path
and the CPU oracle are fed identical bytes.

Distributions (as the workloads state them):
  Q, K, V        bf16, drawn N(0,1) in float32 and rounded to nearest-even bf16
  Z (gate logits) bf16 N(0,1), per token and channel, shared by K and V
  B (gate bias)  float32 N(0, 0.5^2) -- 0.5 read as the standard deviation
  MXFP4 codes    uint8 bytes uniform over 0..255 (two E2M1 nibbles, all 16
                 codes equally likely, -0 included)
  E8M0 scales    uint8 uniform over 125..128 (2^-2 .. 2^1)
  w codes        one E2M1 code per byte, uniform over 0..15
  projection P   bf16 N(0, 1/d)

Every tensor has its own generator seeded from (workload seed, tensor name), so
one tensor can be regenerated without the others.
"""
from dataclasses import dataclass, field
import zlib

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int = 0              # query tokens (prefill)
    H: int = 4              # query heads (one shared K/V head, MQA)
    d: int = 64             # head dim
    m: int = 4              # CSA compression ratio
    k: int = 16             # top-k
    W: int = 64             # sliding window
    HI: int = 4             # indexer heads
    dI: int = 64            # indexer head dim
    m_hca: int = 64         # HCA compression ratio m'
    W_hca: int = 64
    batch: int = 0          # decode: sequences
    context: int = 0        # decode: context length L (new token at L-1)
    chunk: int = 0          # chunked prefill chunk length
    seed: int = 0
    layers: tuple = field(default_factory=tuple)


# The five workloads of the method's specification.
TINY = Workload("tiny_csa_hca_T1024", T=1024, H=4, d=64, m=4, k=16, W=64, HI=4, dI=64, m_hca=64, W_hca=64, seed=0,
                layers=("csa", "hca"))
CSA_PREFILL = Workload("csa_prefill_T32768", T=32768, H=64, d=128, m=4, k=512, W=128, HI=64, dI=128, seed=1,
                       layers=("csa",))
HCA_PREFILL = Workload("hca_prefill_T131072", T=131072, H=64, d=128, m_hca=128, W_hca=128, seed=2, layers=("hca",))
CSA_DECODE = Workload("csa_decode_B16_L1M", H=64, d=128, m=4, k=1024, W=128, HI=16, dI=128, batch=16,
                      context=1048576, seed=3, layers=("csa",))
STACK = Workload("csa_hca_stack_T262144_chunk16384", T=262144, H=64, d=128, m=4, k=1024, W=128, HI=16, dI=128,
                 m_hca=128, W_hca=128, chunk=16384, seed=4, layers=("csa", "hca"))

WORKLOADS = [TINY, CSA_PREFILL, HCA_PREFILL, CSA_DECODE, STACK]


def _gen(seed, name, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + zlib.crc32(name.encode())) & 0x7FFFFFFFFFFFFFFF)
    return g


def normal_bf16(shape, seed, name, std=1.0, device="cpu"):
    g = _gen(seed, name, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def normal_f32(shape, seed, name, std=1.0, device="cpu"):
    g = _gen(seed, name, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def uniform_u8(shape, seed, name, lo, hi, device="cpu"):
    """Integers uniform over [lo, hi] inclusive, stored as uint8."""
    g = _gen(seed, name, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def mxfp4(rows_shape, dI, seed, name, device="cpu"):
    """Packed E2M1 codes [..., dI/2] and E8M0 scales [..., dI/32]."""
    codes = uniform_u8(tuple(rows_shape) + (dI // 2,), seed, name + ".codes", 0, 255, device)
    scales = uniform_u8(tuple(rows_shape) + (dI // 32,), seed, name + ".scales", 125, 128, device)
    return codes, scales


def prefill_layer(wl: Workload, T=None, seed=None, device="cpu", prefix="", with_indexer=True, with_q=True):
    """Inputs of one CSA/HCA prefill layer: Q,K,V,Z,B (+ indexer tensors)."""
    T = wl.T if T is None else T
    s = wl.seed if seed is None else seed
    p = prefix
    out = {}
    if with_q:
        out["Q"] = normal_bf16((T, wl.H, wl.d), s, p + "Q", device=device)
    out["K"] = normal_bf16((T, wl.d), s, p + "K", device=device)
    out["V"] = normal_bf16((T, wl.d), s, p + "V", device=device)
    out["Z"] = normal_bf16((T, wl.d), s, p + "Z", device=device)
    out["B"] = normal_f32((wl.m, wl.d), s, p + "B", std=0.5, device=device)
    out["B_hca"] = normal_f32((wl.m_hca, wl.d), s, p + "B_hca", std=0.5, device=device)
    if with_indexer:
        out["qI_codes"], out["qI_scales"] = mxfp4((T, wl.HI), wl.dI, s, p + "qI", device)
        out["w_codes"] = uniform_u8((T, wl.HI), s, p + "w", 0, 15, device)
        nc = T // wl.m
        out["kI_codes"], out["kI_scales"] = mxfp4((nc,), wl.dI, s, p + "kI", device)
    return out


def decode_batch(wl: Workload, device="cpu", n_entries=None, batch=None):
    """Decode inputs: per sequence a compressed cache (Kc,Vc bf16; kI MXFP4), the
    raw window of the last W tokens (newest last), one query token and its
    indexer query."""
    B = wl.batch if batch is None else batch
    L = wl.context
    N = (L // wl.m) if n_entries is None else n_entries
    s = wl.seed
    out = {
        "q": normal_bf16((B, wl.H, wl.d), s, "q", device=device),
        "Kc": normal_bf16((B, N, wl.d), s, "Kc", device=device),
        "Vc": normal_bf16((B, N, wl.d), s, "Vc", device=device),
        "Kwin": normal_bf16((B, wl.W, wl.d), s, "Kwin", device=device),
        "Vwin": normal_bf16((B, wl.W, wl.d), s, "Vwin", device=device),
    }
    out["qI_codes"], out["qI_scales"] = mxfp4((B, wl.HI), wl.dI, s, "qI", device)
    out["w_codes"] = uniform_u8((B, wl.HI), s, "w", 0, 15, device)
    out["kI_codes"], out["kI_scales"] = mxfp4((B, N), wl.dI, s, "kI", device)
    return out


def projection(wl: Workload, device="cpu"):
    """Per-head projection P [d, d] bf16 N(0, 1/d) shared by all heads (layer-1
    output -> layer-2 query in the two-layer stack)."""
    return normal_bf16((wl.d, wl.d), wl.seed, "P", std=wl.d ** -0.5, device=device)
