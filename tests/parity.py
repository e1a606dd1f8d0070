"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import oracle

# Attention tolerance of the specification: max-abs 1e-2, relative Frobenius 5e-3.
ATTN_MAX_ABS = 1e-2
ATTN_REL_FRO = 5e-3


def bf16_to_f64(t):
    return t.detach().float().cpu().double().numpy()


def words(t):
    """torch bf16 tensor -> numpy uint16 storage words."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_words(w, device):
    return torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).view(torch.bfloat16).to(device)


def _pool_exp2_depth(d, m):
    """N, the most exp2 factors on the path of one gate weight in the GPU
    pooling of a block (its launch rule): S slices of R = m/S rows (S = 1 up to
    16 rows, else the largest power of two with >= 16 rows per slice, m a
    multiple of 8S and d/8 * S <= 512 threads), pooled in chunks of 2 rows;
    groups of d/8 * S threads merge in-warp pairwise over log2 levels, then the
    first warp of a group merges the other warps in turn.  A weight meets its own exp2, the rescales
    after its chunk (at most chunks - 1), one factor per in-warp level and at
    most nw - 1 factors in the cross-warp merge."""
    S = 1
    while 2 * S <= m // 16 and m % (8 * S) == 0 and 2 * S * (d // 8) <= 512:
        S *= 2
    chunks = -(-(m // S) // 2)
    CG = d // 8
    gsize = CG * S
    levels, mask = 0, CG
    while mask < 32 and mask < gsize:
        levels += 1
        mask <<= 1
    nw = gsize // 32 if gsize > 32 else 1
    return chunks + levels + nw - 1


def fp32_pool_slack(x_bf16, m, Z, B):
    """Worst-case absolute error of the fp32 gated pooling, per (block, channel),
    with u = 2^-24, X = max |x| over the block, G = max |z + b| over the block,
    and N = _pool_exp2_depth(d, m):
      the kernel takes logits in base 2, g2 = RN(RN(z + b) * RN(log2 e)), so every
      logit carries 3uG (the sum, the rounded constant, the product; an error
      common to all logits of a block cancels in the normalised mean), and
      every weight a relative error of at most
        3*u*G + N * (2*u*G + 4*u)
      (each of its N exp2 factors - its own, the in-slice rescales after it and
      the slice merges on its path - is one exp2 of a rounded difference: 2uG
      for the difference, 4u for exp2f's 2-ulp bound); a relative weight error
      eta moves a weighted mean by at most 2*eta*X; the sums of numerator and
      denominator (m terms, each through at most m - 1 additions in any order,
      and at most N rescale products) add (m + N) * u * X each; the division and
      the final product 2*u*X.  Total:
        u * X * (2*G*(3 + 2*N) + 8*N + 2*(m + N) + 2).
    When the weighted sum cancels, this can exceed one bf16 ulp of the (small)
    result; otherwise the bf16 ulp dominates."""
    xf = x_bf16.detach().float().cpu().double().numpy() if hasattr(x_bf16, "detach") else oracle.bf16_words_to_f64(x_bf16)
    zf = Z.detach().float().cpu().double().numpy() if hasattr(Z, "detach") else oracle.bf16_words_to_f64(Z)
    bf = B.detach().float().cpu().double().numpy() if hasattr(B, "detach") else np.asarray(B, np.float64)
    T, d = xf.shape
    nb = T // m
    X = np.abs(xf[: nb * m]).reshape(nb, m, d).max(axis=1)
    g = zf[: nb * m].reshape(nb, m, d) + bf[None, :, :]
    G = np.abs(g).max(axis=1)
    N = _pool_exp2_depth(d, m)
    u = 2.0 ** -24
    return u * X * (2 * G * (3 + 2 * N) + 8 * N + 2 * (m + N) + 2)


def assert_within_bf16_ulp(got_bf16, exact_f64, what, slack=None):
    """|got - exact| <= 1 ulp of bf16 at |exact| (+ an optional fp32 evaluation
    slack): the GPU rounds an fp32 result to nearest-even bf16; the exact value is
    the oracle's fp64 result."""
    got = bf16_to_f64(got_bf16)
    ex = np.asarray(exact_f64, np.float64)
    mag = np.maximum(np.abs(ex), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    if slack is not None:
        ulp = ulp + slack
    err = np.abs(got - ex)
    bad = err > ulp
    assert not bad.any(), "%s: %d of %d elements off by more than 1 bf16 ulp (max err/ulp %.3f)" % (
        what, int(bad.sum()), bad.size, float((err / ulp).max()))


def assert_attention_close(got_bf16, want_f64, what):
    """Spec tolerance on an attention output (bf16 or fp32 tensor); prints the
    margins used (max |O|, max-abs and rel-Frobenius as fractions of the bound)."""
    got = bf16_to_f64(got_bf16)
    want = np.asarray(want_f64, np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    fro = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-30)) if diff.size else 0.0
    omax = float(np.abs(want).max()) if want.size else 0.0
    print("[margin] %s (%s): max|O| %.3f, max-abs %.3e (%.0f%% of bound), rel-Fro %.3e (%.0f%% of bound)" % (
        what, str(getattr(got_bf16, "dtype", "?")).replace("torch.", ""), omax, max_abs,
        100 * max_abs / ATTN_MAX_ABS, fro, 100 * fro / ATTN_REL_FRO))
    assert max_abs <= ATTN_MAX_ABS and fro <= ATTN_REL_FRO, "%s: max-abs %.3e (<= %.0e), rel-Frobenius %.3e (<= %.0e)" % (
        what, max_abs, ATTN_MAX_ABS, fro, ATTN_REL_FRO)
    return max_abs, fro


def assert_topk_exact(idx_gpu, scores_gpu, idx_want, top_want, what):
    ig = idx_gpu.cpu().numpy()
    np.testing.assert_array_equal(ig, idx_want, err_msg=what + ": top-k indices differ")
    if scores_gpu is not None:
        sg = scores_gpu.cpu().numpy()
        sw = np.asarray(top_want, np.float64).astype(np.float32)  # round-to-nearest of the exact score
        np.testing.assert_array_equal(sg, sw, err_msg=what + ": top-k scores differ")


def sample_rows(T, n, special, seed):
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in special if 0 <= r < T)
    rows.update(int(r) for r in rng.choice(T, size=min(n, T), replace=False))
    return np.array(sorted(rows), dtype=np.int64)
