"""A device-side wait that runs out: the indexer launch that follows
csa_debug_inject(CSA_FAULT_INDEXER_STALL) never receives its first key tile,
so its MMA and epilogue waits give up after their deadline (~0.14 s).  The
launch must come back with CSA_ERR_DEVICE_TIMEOUT in the status word, and the
CUDA context must stay usable: the same call afterwards gives the oracle's
selection.  Nothing is read or written out of bounds and no GPU fault is raised;
the injected fault only withholds one copy."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_gated_b200 import inputs
from tests.parity import assert_topk_exact

pytestmark = pytest.mark.gpu

CSA_FAULT_INDEXER_STALL = 1
CSA_ERR_DEVICE_TIMEOUT = -6


def test_indexer_stall_times_out_and_the_context_survives():
    import long_context_compressed_gated_b200 as csa
    T, Nc, HI, dI, m, k, seed = 64, 1024, 16, 128, 4, 32, 61
    qc, qs = inputs.mxfp4((T, HI), dI, seed, "qI")
    w = inputs.uniform_u8((T, HI), seed, "w", 0, 15)
    kc, ks = inputs.mxfp4((Nc,), dI, seed, "kI")
    g = [x.cuda() for x in (qc, qs, w, kc, ks)]
    t0 = 4 * Nc - T  # every row sees all Nc entries: eight key tiles per row
    assert csa.lib().csa_debug_inject(CSA_FAULT_INDEXER_STALL) == 0
    idx, sc, ws = csa.csa_indexer_topk(*g, m, k, t0=t0)
    torch.cuda.synchronize()
    assert csa.csa_check_status(ws) == CSA_ERR_DEVICE_TIMEOUT
    # the status word was cleared by the check; the next launch runs normally
    idx, sc, ws = csa.csa_indexer_topk(*g, m, k, t0=t0, workspace=ws)
    assert csa.csa_check_status(ws) == 0
    I = oracle.indexer(qc, qs, w, kc, ks, t0, m)
    want_idx, want_top = oracle.topk(I, np.minimum(oracle.n_vis(t0 + np.arange(T), m), Nc), k)
    assert_topk_exact(idx, sc, want_idx, want_top, "indexer after a timed-out launch")

