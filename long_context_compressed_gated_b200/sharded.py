"""Token-sharded CSA -> HCA prefill over G ranks (one process per GPU).

The method's prefill shards by query tokens (blog.nickys.cn/?p=150 "1. CSA" /
"2. HCA": a query needs the compressed entries of every block that ends at or
before it, its k selected ones or all of them, plus the raw tokens of its
window).  The sequence of T tokens is cut into 2G chunks of C = T / (2G)
tokens, and rank r owns chunks r and 2G-1-r (zig-zag), which balances the
causal work.  Per layer:

  1. compress   each rank pools the blocks of its own chunks (C is a multiple
                of m and m', so no block straddles two chunks);
  2. exchange   ONE all-gather of every rank's compressed entries (K/V, and
                for CSA the entries' MXFP4 indexer keys) and of the last W-1
                raw K/V rows of each of its chunks (the halo the next chunk's
                window reaches into);
  3. attend     each rank assembles the compressed cache in position order and
                the raw rows its windows need, then runs the indexer + top-k and
                sparse attention (CSA) or dense attention (HCA) for its own
                query rows against the entries that precede them.

Between the layers each rank projects its own CSA outputs (Q2 = O1 P, outside
the method) and the HCA layer repeats steps 1-3 with m', no indexer.  Every
compute step is a libcsa call (`ops`); this module only moves tensors.  The
collective goes through `comm`: TorchComm (torch.distributed: NCCL on GPUs,
gloo on CPU) or EmulatedRanks, which runs the G ranks one after another in one
process (a single GPU) with the all-gather done by concatenation.
"""
import math

import torch


class TorchComm:
    """The all-gather of the sharded path over torch.distributed."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, flat):
        out = [torch.empty_like(flat) for _ in range(self.world)]
        self.dist.all_gather(out, flat, group=self.group)
        return out


def chunks_of(rank, world):
    """The two chunk indices (of 2*world) that rank owns: r and 2G-1-r."""
    return (rank, 2 * world - 1 - rank)


def owner_of(chunk, world):
    return chunk if chunk < world else 2 * world - 1 - chunk


def _pack(tensors):
    """Flatten a list of tensors into one uint8 buffer (all ranks pack the same shapes)."""
    return torch.cat([t.contiguous().view(torch.uint8).reshape(-1) for t in tensors])


def _unpack(flat, like):
    out, off = [], 0
    for t in like:
        n = t.numel() * t.element_size()
        out.append(flat[off:off + n].view(t.dtype).reshape(t.shape))
        off += n
    return out


class ShardedPrefill:
    """The sharded two-layer prefill of one rank.

    x: the rank's inputs -- dict of per-chunk slices {c: {...}} for its two chunks
    with, per chunk c (positions c*C .. c*C+C-1):
      Q [C,H,d], K, V, Z [C,d] (layer 1), qI_codes [C,HI,dI/2], qI_scales
      [C,HI,dI/32], w_codes [C,HI], kI_codes [C/m,dI/2], kI_scales [C/m,dI/32]
      (the indexer keys of the chunk's blocks), K2, V2, Z2 [C,d] (layer 2);
    shared: B [m,d], B2 [m2,d] f32, P [d,d] bf16.
    """

    def __init__(self, T, world, m, k, W, m2, W2, scale=None, ops=None):
        assert T % (2 * world) == 0
        self.T, self.G = T, world
        self.C = T // (2 * world)
        assert self.C % m == 0 and self.C % m2 == 0 and self.C >= max(W, W2)
        self.m, self.k, self.W, self.m2, self.W2 = m, k, W, m2, W2
        self.scale = scale
        if ops is None:
            import long_context_compressed_gated_b200 as ops
        self.ops = ops

    # --------------------------------------------------------------- layer 1 (CSA)
    def csa_parts(self, x):
        """Step 1 for the CSA layer: this rank's compressed entries, indexer keys and halos."""
        parts = []
        for c in sorted(x["chunks"]):
            ch = x["chunks"][c]
            Kc, Vc = self.ops.csa_compress(ch["K"], ch["V"], ch["Z"], x["B"], self.m)
            halo = max(self.W - 1, 0)
            parts += [Kc, Vc, ch["kI_codes"], ch["kI_scales"], ch["K"][self.C - halo:], ch["V"][self.C - halo:]]
        return parts

    def csa_attend(self, x, gathered):
        """Step 3 for the CSA layer: returns {chunk: O1 [C,H,d]}."""
        ch0 = next(iter(x["chunks"].values()))
        cache = self._assemble(gathered, per_chunk=6, m=self.m, with_keys=True)
        out = {}
        d = ch0["K"].shape[1]
        scale = self.scale if self.scale is not None else 1.0 / math.sqrt(d)
        for c in sorted(x["chunks"]):
            ch = x["chunks"][c]
            s0 = c * self.C
            e = (s0 + self.C) // self.m
            Kraw, Vraw = self._raw_rows(cache, ch["K"], ch["V"], c, self.W)
            idx, _, _ = self.ops.csa_indexer_topk(ch["qI_codes"], ch["qI_scales"], ch["w_codes"],
                                                  cache["kI_codes"][:e], cache["kI_scales"][:e], self.m, self.k,
                                                  t0=s0, want_scores=False)
            O, _, _ = self.ops.csa_sparse_attn(ch["Q"], cache["Kc"][:e], cache["Vc"][:e], idx, Kraw, Vraw, self.W,
                                               scale, t0=s0, want_lse=False)
            out[c] = O
        return out

    # --------------------------------------------------------------- layer 2 (HCA)
    def hca_parts(self, x):
        parts = []
        for c in sorted(x["chunks"]):
            ch = x["chunks"][c]
            Kc, Vc = self.ops.csa_compress(ch["K2"], ch["V2"], ch["Z2"], x["B2"], self.m2)
            halo = max(self.W2 - 1, 0)
            parts += [Kc, Vc, ch["K2"][self.C - halo:], ch["V2"][self.C - halo:]]
        return parts

    def hca_attend(self, x, gathered, Q2):
        ch0 = next(iter(x["chunks"].values()))
        cache = self._assemble(gathered, per_chunk=4, m=self.m2, with_keys=False)
        d = ch0["K2"].shape[1]
        scale = self.scale if self.scale is not None else 1.0 / math.sqrt(d)
        out = {}
        for c in sorted(x["chunks"]):
            ch = x["chunks"][c]
            s0 = c * self.C
            e = (s0 + self.C) // self.m2
            Kraw, Vraw = self._raw_rows(cache, ch["K2"], ch["V2"], c, self.W2)
            O, _, _ = self.ops.hca_attn(Q2[c], cache["Kc"][:e], cache["Vc"][:e], Kraw, Vraw, self.m2, self.W2, scale,
                                        t0=s0, want_lse=False)
            out[c] = O
        return out

    # --------------------------------------------------------------- helpers
    def _assemble(self, gathered, per_chunk, m, with_keys):
        """Compressed cache in position order from every rank's parts (each rank
        lists its chunks in increasing order)."""
        G, C = self.G, self.C
        slots = {}
        for r, parts in enumerate(gathered):
            for i, c in enumerate(sorted(chunks_of(r, G))):
                slots[c] = parts[i * per_chunk:(i + 1) * per_chunk]
        order = [slots[c] for c in range(2 * G)]
        cache = {"Kc": torch.cat([p[0] for p in order]), "Vc": torch.cat([p[1] for p in order]),
                 "halo_K": {c: order[c][-2] for c in range(2 * G)}, "halo_V": {c: order[c][-1] for c in range(2 * G)}}
        if with_keys:
            cache["kI_codes"] = torch.cat([p[2] for p in order])
            cache["kI_scales"] = torch.cat([p[3] for p in order])
        return cache

    def _raw_rows(self, cache, K, V, c, W):
        """Raw K/V addressed by absolute position (row s at index s) for chunk c:
        the previous chunk's halo rows and the chunk's own rows; nothing earlier is
        read by the chunk's windows."""
        s0 = c * self.C
        Kr = K.new_zeros(s0 + self.C, K.shape[1])
        Vr = V.new_zeros(s0 + self.C, V.shape[1])
        Kr[s0:] = K
        Vr[s0:] = V
        h = max(W - 1, 0)
        if c > 0 and h > 0:
            Kr[s0 - h:s0] = cache["halo_K"][c - 1]
            Vr[s0 - h:s0] = cache["halo_V"][c - 1]
        return Kr, Vr

    # --------------------------------------------------------------- one rank, end to end
    def run(self, x, comm):
        """Both layers for this rank (comm: rank, world, all_gather)."""
        parts = self.csa_parts(x)
        gathered = [_unpack(f, parts) for f in comm.all_gather(_pack(parts))]
        O1 = self.csa_attend(x, gathered)
        Q2 = {c: self._project(O1[c], x["P"]) for c in O1}
        parts2 = self.hca_parts(x)
        gathered2 = [_unpack(f, parts2) for f in comm.all_gather(_pack(parts2))]
        return self.hca_attend(x, gathered2, Q2), O1

    @staticmethod
    def _project(O1, P):
        # glue between the layers (outside the method): Q2[t,h] = bf16(O1[t,h] P)
        C, H, d = O1.shape
        return torch.matmul(O1.reshape(-1, d), P).reshape(C, H, d)


def shard_inputs(l1, l2, P, rank, world, T, m):
    """The rank's view of full-sequence inputs (for tests and benchmarks; a
    deployment would hold only its chunks).  l1/l2 as in stack.stack_inputs; m is
    the CSA ratio (the indexer keys are per block of m tokens)."""
    C = T // (2 * world)
    chunks = {}
    for c in chunks_of(rank, world):
        sl = slice(c * C, (c + 1) * C)
        b1 = slice(c * C // m, (c + 1) * C // m)
        chunks[c] = {"Q": l1["Q"][sl], "K": l1["K"][sl], "V": l1["V"][sl], "Z": l1["Z"][sl],
                     "qI_codes": l1["qI_codes"][sl], "qI_scales": l1["qI_scales"][sl], "w_codes": l1["w_codes"][sl],
                     "kI_codes": l1["kI_codes"][b1], "kI_scales": l1["kI_scales"][b1],
                     "K2": l2["K"][sl], "V2": l2["V"][sl], "Z2": l2["Z"][sl]}
    return {"chunks": chunks, "B": l1["B"], "B2": l2["B"], "P": P}


class EmulatedRanks:
    """Runs the G ranks' phases one after another in one process (one GPU): the
    all-gather is the list of every rank's parts.  No kernel of one rank waits on
    another rank's."""

    def __init__(self, world):
        self.world = world

    def run(self, sp, xs):
        parts = [sp.csa_parts(x) for x in xs]
        O1 = [sp.csa_attend(x, parts) for x in xs]
        Q2 = [{c: sp._project(o[c], x["P"]) for c in o} for o, x in zip(O1, xs)]
        parts2 = [sp.hca_parts(x) for x in xs]
        O2 = [sp.hca_attend(x, parts2, q) for x, q in zip(xs, Q2)]
        return O2, O1


# ------------------------------------------------------------------ split-cache decode
class SplitCacheDecode:
    """Decode of B sequences whose compressed caches are split over the ranks by
    entry ranges: rank r holds entries [j_base, j_base + Nloc) of every sequence,
    the last rank also the raw window (the newest tokens).  Per step:

      1. search     the k best entries of the rank's slice, as exact 64-bit keys
                    with global entry numbers (csa_decode_search);
      2. exchange   all-gather of the keys ([L, B, k]);
      3. merge      the exact top-k of the L lists, identical on every rank
                    (csa_topk_merge);
      4. attend     attention over the selected entries inside the slice, plus
                    the window on the last rank: an fp32 partial output and its
                    log-sum-exp (csa_decode_attend);
      5. exchange   all-gather of the partials, then their log-sum-exp combine
                    (csa_attn_combine).

    x: dict with q [B,H,d], qI_codes, qI_scales, w_codes, Kc, Vc [B,Nloc,d] (the
    slice), kI_codes [B,Nloc,dI/2], kI_scales, Kwin, Vwin [B,W,d], pos (host list),
    j_base, has_window.  The result equals csa_decode on the whole cache: the
    selection bit for bit, O within the attention tolerance.
    """

    def __init__(self, m, k, W, scale, ops=None):
        self.m, self.k, self.W, self.scale = m, k, W, scale
        if ops is None:
            import long_context_compressed_gated_b200 as ops
        self.ops = ops

    def search(self, x):
        keys, _ = self.ops.csa_decode_search(x["qI_codes"], x["qI_scales"], x["w_codes"], x["kI_codes"],
                                             x["kI_scales"], x["pos"], self.m, self.k, j_base=x["j_base"])
        return keys

    def merge(self, gathered_keys):
        return self.ops.csa_topk_merge(torch.stack(gathered_keys, dim=1), self.k)

    def attend(self, x, idx):
        W = self.W if x["has_window"] else 0
        return self.ops.csa_decode_attend(x["q"], x["Kc"], x["Vc"], idx, x["Kwin"], x["Vwin"], x["pos"], self.m, W,
                                          self.scale, j_base=x["j_base"])

    def combine(self, gathered_O, gathered_lse, out_dtype=torch.float32):
        return self.ops.csa_attn_combine(torch.stack(gathered_O), torch.stack(gathered_lse), out_dtype=out_dtype)

    def run(self, x, comm, out_dtype=torch.float32):
        """One decode step on this rank; returns (O, lse, idx, scores), the same on every rank."""
        keys = self.search(x)
        idx, scores = self.merge(comm.all_gather(keys))
        O_r, lse_r = self.attend(x, idx)
        O, lse = self.combine(comm.all_gather(O_r), comm.all_gather(lse_r), out_dtype)
        return O, lse, idx, scores


def split_cache(batch, rank, world):
    """The rank's slice of full decode inputs (for tests and benchmarks): entries
    [r*N/G, (r+1)*N/G) of every sequence's cache; the last rank keeps the window."""
    N = batch["Kc"].shape[1]
    lo, hi = rank * N // world, (rank + 1) * N // world
    x = {k: batch[k] for k in ("q", "qI_codes", "qI_scales", "w_codes", "Kwin", "Vwin")}
    for key in ("Kc", "Vc", "kI_codes", "kI_scales"):
        x[key] = batch[key][:, lo:hi].contiguous()
    x["j_base"] = lo
    x["has_window"] = rank == world - 1
    return x


def emulated_split_decode(dec, xs, out_dtype=torch.float32):
    """All ranks' steps in one process (one GPU): the all-gathers are lists."""
    keys = [dec.search(x) for x in xs]
    merged = [dec.merge(keys) for _ in xs]
    parts = [dec.attend(x, m[0]) for x, m in zip(xs, merged)]
    O, lse = dec.combine([p[0] for p in parts], [p[1] for p in parts], out_dtype)
    return O, lse, merged[0][0], merged[0][1]
