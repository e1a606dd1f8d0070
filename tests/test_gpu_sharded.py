"""The token-sharded prefill on one GPU with emulated ranks (each rank's phases
run in turn; the all-gather is a concatenation, so no kernel waits on another
rank).  The sharded result must equal the chunked single-GPU stack: layer-1
outputs bit for bit (the compressed entries, the selection and the attention of
a row do not depend on how the sequence is split), layer-2 outputs within the
tolerance (the projection between the layers is a library bf16 matmul over
differently shaped row blocks)."""
import numpy as np
import pytest
import torch

from long_context_compressed_gated_b200 import inputs
from long_context_compressed_gated_b200.sharded import EmulatedRanks, ShardedPrefill, chunks_of, shard_inputs
from long_context_compressed_gated_b200.stack import stack_inputs, stack_prefill_chunked
from tests.parity import assert_attention_close

pytestmark = pytest.mark.gpu

SMALL = inputs.Workload("sharded_gpu_small", T=4096, H=64, d=128, m=4, k=64, W=128, HI=16, dI=128, m_hca=128,
                        W_hca=128, seed=58)


@pytest.mark.parametrize("wl,world", [(SMALL, 2), (SMALL, 4), (SMALL, 8), (inputs.STACK, 8)])
def test_emulated_ranks_equal_the_single_gpu_stack(wl, world):
    l1, l2, P = stack_inputs(wl, device="cuda")
    chunk = wl.chunk if wl.chunk else wl.T // 4
    O2_ref, O1_ref = stack_prefill_chunked(l1, l2, P, chunk, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca, return_o1=True)
    sp = ShardedPrefill(wl.T, world, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca)
    xs = [shard_inputs(l1, l2, P, r, world, wl.T, wl.m) for r in range(world)]
    O2, O1 = EmulatedRanks(world).run(sp, xs)
    torch.cuda.synchronize()
    C = wl.T // (2 * world)
    for r in range(world):
        for c in chunks_of(r, world):
            sl = slice(c * C, (c + 1) * C)
            assert torch.equal(O1[r][c], O1_ref[sl]), "layer 1 differs on chunk %d of %d ranks" % (c, world)
            if c in (0, 2 * world - 1):
                assert_attention_close(O2[r][c], O2_ref[sl].float().cpu().double().numpy(),
                                       "layer 2, chunk %d of %d ranks" % (c, world))


@pytest.mark.parametrize("world", [2, 4])
def test_split_cache_decode_emulated_ranks(world):
    """Split-cache decode with the ranks emulated on one GPU, against csa_decode
    over the whole cache: selection bit for bit, output within the tolerance."""
    import math
    import long_context_compressed_gated_b200 as csa
    from long_context_compressed_gated_b200.sharded import SplitCacheDecode, emulated_split_decode, split_cache
    wl = inputs.Workload("split_dec", H=64, d=128, m=4, k=1024, W=128, HI=16, dI=128, batch=4, context=1 << 18,
                         seed=62)
    g = {key: v.cuda() for key, v in inputs.decode_batch(wl).items()}
    pos = [wl.context - 1, 200000, 70001, 4100]
    scale = 1.0 / math.sqrt(wl.d)
    O_ref, lse_ref, idx_ref, sc_ref, ws = csa.csa_decode(g["q"], g["qI_codes"], g["qI_scales"], g["w_codes"], g["Kc"],
                                                         g["Vc"], g["kI_codes"], g["kI_scales"], g["Kwin"], g["Vwin"],
                                                         pos, wl.m, wl.k, scale, out_dtype=torch.float32)
    assert csa.csa_check_status(ws) == 0
    dec = SplitCacheDecode(wl.m, wl.k, wl.W, scale)
    xs = []
    for r in range(world):
        x = split_cache(g, r, world)
        x["pos"] = pos
        xs.append(x)
    O, lse, idx, sc = emulated_split_decode(dec, xs)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref) and torch.equal(sc, sc_ref)
    assert_attention_close(O, O_ref.double().cpu().numpy(), "split-cache decode over %d ranks" % world)
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), atol=1e-4)
