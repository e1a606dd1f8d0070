"""GPU parity of the MXFP4 quantiser (csa_mxfp4_quantize) against the oracle:
codes and scales bit for bit, in both modes, on blocks of every magnitude
(zeros, subnormal bf16, normal, huge, mixed signs, non-finite); then bf16
indexer activations quantised on the GPU in the indexer range feed the
indexer, whose top-k must equal the oracle's on the oracle's own quantisation.
The indexer's query-key path on MXFP4: m.youleyou.com/wenzhang/2906406.html
section 1."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import assert_topk_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import long_context_compressed_gated_b200 as m
    m.lib()
    return m


def _mixed_blocks(rows, n, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, n, generator=g)
    # per-block magnitude from 2^-140 (bf16 subnormal) to 2^100
    nb = n // 32
    e = torch.randint(-140, 100, (rows, nb), generator=g).float()
    x = x * torch.pow(2.0, e).repeat_interleave(32, dim=1)
    x[0, :32] = 0.0                       # an all-zero block
    x[1, :32] = -0.0
    x[2, 5] = float("inf")                # non-finite blocks
    x[3, 40] = float("nan")
    x[4, :32] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4)  # ties at scale 2^0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("rows,n,seed", [(1000, 128, 1), (333, 64, 2), (4096, 256, 3)])
def test_quantize_bit_exact(csa, mode, rows, n, seed):
    x = _mixed_blocks(rows, n, seed)
    codes, scales = csa.csa_mxfp4_quantize(x.cuda(), mode=mode)
    torch.cuda.synchronize()
    c_want, s_want = oracle.mxfp4_quantize(x, mode=mode)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_want, err_msg="scales")
    np.testing.assert_array_equal(codes.cpu().numpy(), c_want, err_msg="codes")


def test_quantized_activations_feed_the_indexer(csa):
    """bf16 indexer queries [T, HI, dI] and keys [Nc, dI], N(0, 1) like the layer's
    activations, quantised in the indexer range on the GPU; the selection is
    compared with the oracle's indexer + top-k over the oracle's quantisation."""
    T, Nc, HI, dI, m, k = 512, 1024, 16, 128, 4, 64
    t0 = 4 * Nc - T
    qf = inputs.normal_bf16((T, HI, dI), 5, "qf")
    kf = inputs.normal_bf16((Nc, dI), 5, "kf")
    w = inputs.uniform_u8((T, HI), 5, "w", 0, 15)
    qc, qs = csa.csa_mxfp4_quantize(qf.cuda(), mode=1)
    kc, ks = csa.csa_mxfp4_quantize(kf.cuda(), mode=1)
    qc_x, qs_x = oracle.mxfp4_quantize(qf, mode=1)
    kc_x, ks_x = oracle.mxfp4_quantize(kf, mode=1)
    np.testing.assert_array_equal(qc.cpu().numpy(), qc_x)
    np.testing.assert_array_equal(ks.cpu().numpy(), ks_x)
    idx, sc, ws = csa.csa_indexer_topk(qc, qs, w.cuda(), kc, ks, m, k, t0=t0)
    assert csa.csa_check_status(ws) == 0  # every scale byte in the exact range
    I = oracle.indexer(qc_x, qs_x, w, kc_x, ks_x, t0, m)
    want_idx, want_top = oracle.topk(I, np.minimum(oracle.n_vis(t0 + np.arange(T), m), Nc), k)
    assert_topk_exact(idx, sc, want_idx, want_top, "indexer on quantised activations")
