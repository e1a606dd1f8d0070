"""The token-sharded prefill's exchange on two CPU ranks (gloo): each rank
compresses its own chunks, one all-gather per layer brings every rank's
compressed entries, indexer keys and window halos, and each rank attends for
its own rows.  The compute steps are the oracle here (tests/oracle_ops.py), so
the result must equal the oracle's unsharded chain: layer-1 outputs bit for
bit, layer-2 outputs within the attention tolerance (the projection between
the layers is a bf16 matmul over differently shaped row blocks)."""
import math
import os
import socket
import tempfile

import numpy as np
import torch
import torch.multiprocessing as mp

import oracle
from long_context_compressed_gated_b200 import inputs
from long_context_compressed_gated_b200.sharded import EmulatedRanks, ShardedPrefill, TorchComm, chunks_of, shard_inputs
from long_context_compressed_gated_b200.stack import stack_inputs
from tests.parity import assert_attention_close

WL = inputs.Workload("sharded_small", T=512, H=4, d=64, m=4, k=16, W=32, HI=4, dI=64, m_hca=32, W_hca=32, seed=57)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, outdir):
    import torch.distributed as dist
    from tests import oracle_ops
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        l1, l2, P = stack_inputs(WL)
        sp = ShardedPrefill(WL.T, world, WL.m, WL.k, WL.W, WL.m_hca, WL.W_hca, ops=oracle_ops)
        x = shard_inputs(l1, l2, P, rank, world, WL.T, WL.m)
        O2, O1 = sp.run(x, TorchComm())
        torch.save({"O1": O1, "O2": O2}, os.path.join(outdir, "rank%d.pt" % rank))
    finally:
        dist.destroy_process_group()


def _oracle_chain(l1, l2, P):
    """Unsharded reference: every row's layer-1 selection and output, Q2 = bf16(O1 P)
    in fp64 from the bf16 O1, then layer 2."""
    wl = WL
    scale = 1.0 / math.sqrt(wl.d)
    Kc, Vc = oracle.compress(l1["K"], l1["V"], l1["Z"], l1["B"], wl.m)
    Kw, Vw = oracle.to_bf16_words(Kc), oracle.to_bf16_words(Vc)
    I = oracle.indexer(l1["qI_codes"], l1["qI_scales"], l1["w_codes"], l1["kI_codes"], l1["kI_scales"], 0, wl.m)
    sel, _ = oracle.topk(I, oracle.n_vis(np.arange(wl.T), wl.m), wl.k)
    O1, _ = oracle.attention(l1["Q"], Kw, Vw, l1["K"], l1["V"], 0, wl.m, wl.W, scale, sel=sel)
    O1w = oracle.to_bf16_words(O1)
    Pf = oracle.bf16_words_to_f64(oracle._u16(P)).reshape(wl.d, wl.d)
    Q2 = oracle.to_bf16_words(oracle.bf16_words_to_f64(O1w) @ Pf)
    K2, V2 = oracle.compress(l2["K"], l2["V"], l2["Z"], l2["B"], wl.m_hca)
    O2, _ = oracle.attention(Q2, oracle.to_bf16_words(K2), oracle.to_bf16_words(V2), l2["K"], l2["V"], 0,
                             wl.m_hca, wl.W_hca, scale)
    return O1w, O2


def test_two_gloo_ranks_equal_the_unsharded_oracle():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        res = [torch.load(os.path.join(d, "rank%d.pt" % r)) for r in range(world)]
    l1, l2, P = stack_inputs(WL)
    O1w, O2 = _oracle_chain(l1, l2, P)
    C = WL.T // (2 * world)
    for r in range(world):
        for c in chunks_of(r, world):
            sl = slice(c * C, (c + 1) * C)
            got1 = res[r]["O1"][c].contiguous().view(torch.int16).numpy().view(np.uint16)
            np.testing.assert_array_equal(got1, O1w[sl], err_msg="layer 1, chunk %d (rank %d)" % (c, r))
            assert_attention_close(res[r]["O2"][c], O2[sl], "layer 2, chunk %d (rank %d)" % (c, r))


def test_zigzag_chunks_cover_the_sequence_once():
    for world in (1, 2, 3, 8):
        owned = sorted(c for r in range(world) for c in chunks_of(r, world))
        assert owned == list(range(2 * world))
        # the zig-zag pairs an early chunk with a late one: equal causal work per rank
        work = [sum(c + 0.5 for c in chunks_of(r, world)) for r in range(world)]
        assert max(work) == min(work)


def test_emulated_ranks_equal_torch_ranks_on_cpu():
    """The single-process emulation (used on one GPU) gives the same layer-1
    results as the real collective."""
    from tests import oracle_ops
    world = 2
    l1, l2, P = stack_inputs(WL)
    sp = ShardedPrefill(WL.T, world, WL.m, WL.k, WL.W, WL.m_hca, WL.W_hca, ops=oracle_ops)
    xs = [shard_inputs(l1, l2, P, r, world, WL.T, WL.m) for r in range(world)]
    O2e, O1e = EmulatedRanks(world).run(sp, xs)
    O1w, _ = _oracle_chain(l1, l2, P)
    C = WL.T // (2 * world)
    for r in range(world):
        for c in chunks_of(r, world):
            got = O1e[r][c].contiguous().view(torch.int16).numpy().view(np.uint16)
            np.testing.assert_array_equal(got, O1w[c * C:(c + 1) * C])


# ------------------------------------------------------------------ split-cache decode on two gloo ranks
DEC = inputs.Workload("split_dec_small", H=4, d=64, m=4, k=16, W=32, HI=4, dI=64, batch=2, context=4096, seed=61)


def _decode_rank_main(rank, world, port, outdir):
    import torch.distributed as dist
    from long_context_compressed_gated_b200.sharded import SplitCacheDecode, split_cache
    from tests import oracle_ops
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        batch = inputs.decode_batch(DEC)
        batch["pos"] = [DEC.context - 1, 3000]
        dec = SplitCacheDecode(DEC.m, DEC.k, DEC.W, 1.0 / math.sqrt(DEC.d), ops=oracle_ops)
        x = split_cache(batch, rank, world)
        x["pos"] = batch["pos"]
        O, lse, idx, sc = dec.run(x, TorchComm())
        torch.save({"O": O, "idx": idx}, os.path.join(outdir, "dec%d.pt" % rank))
    finally:
        dist.destroy_process_group()


def test_split_cache_decode_on_two_gloo_ranks():
    """Each rank searches its half of the cache; one all-gather of candidates, an
    identical merge, attention over its own selected entries (+ the window on the
    last rank), an all-gather of the partial outputs and their log-sum-exp combine:
    equal to the oracle's decode over the whole cache."""
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_decode_rank_main, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        res = [torch.load(os.path.join(d, "dec%d.pt" % r)) for r in range(world)]
    batch = inputs.decode_batch(DEC)
    pos = [DEC.context - 1, 3000]
    scale = 1.0 / math.sqrt(DEC.d)
    for b, t in enumerate(pos):
        I = oracle.indexer(batch["qI_codes"][b:b + 1], batch["qI_scales"][b:b + 1], batch["w_codes"][b:b + 1],
                           batch["kI_codes"][b], batch["kI_scales"][b], t, DEC.m)
        want_idx, _ = oracle.topk(I, oracle.n_vis([t], DEC.m), DEC.k)
        o, _ = oracle.attention(batch["q"][b:b + 1], batch["Kc"][b], batch["Vc"][b], batch["Kwin"][b],
                                batch["Vwin"][b], t, DEC.m, DEC.W, scale, sel=want_idx, rows=[0],
                                raw_pos0=t - DEC.W + 1)
        for r in range(world):
            np.testing.assert_array_equal(res[r]["idx"][b].numpy(), want_idx[0])
            np.testing.assert_allclose(res[r]["O"][b].numpy(), o[0], atol=1e-5)
