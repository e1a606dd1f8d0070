"""Benchmark of the CSA/HCA hot path on B200 (one JSON line on rank 0).

Step = one pass of the whole CSA prefill path (gated compression m=4, MXFP4
indexer + causal top-k, sparse + window attention) over one sequence of the
T=32768, 64x128 workload, inputs resident in HBM.  The HCA prefill
(T=131072, m'=128) and the 1M-context CSA decode (B=16) are measured the same
way and reported under "workloads".  With --gpus N each rank runs its own
sequence (independent problems, no collective): weak scaling.

--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_compressed_gated_b200 import inputs  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
METRIC = "CSA/HCA prefill tokens/s & TFLOP/s; 1M-ctx decode GB/s; % of B200 roofline"
NOMINAL_FP4_TFLOPS = 9000.0  # NVIDIA's dense FP4 figure for B200 (context only)
# DRAM bytes per call (dram__bytes_read.sum + dram__bytes_write.sum) of each phase's
# kernels on the T=32768 CSA prefill, from the ncu captures summarised under profiles/;
# to be refreshed whenever those kernels change.
E2E_CHUNKS = 16  # query chunks of the pipelined end-to-end step

PHASE_TRAFFIC = {
    # DRAM bytes (read + written) of one full-size launch, from the one-pass ncu capture
    # of the bench's launch list (summary under profiles/); the indexer phase is the
    # indexer kernel plus the finalize kernel
    "indexer_topk": (145393664 + 87410432 + 130292736 + 30677248,
                     "ncu dram__bytes_read.sum + dram__bytes_write.sum of the full-size indexer and finalize "
                     "launches (one-pass capture of the bench's launch list, profiles/)"),
    "sparse_attn": (626069504 + 487205632,
                    "ncu dram__bytes_read.sum + dram__bytes_write.sum of a full-size attention launch "
                    "(one-pass capture of the bench's launch list, profiles/)"),
}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------- tensor-pipe peaks
def measure_tensor_peaks(csa, sustained_s=0.0, sampler=None):
    """The MXFP4 and bf16 ceilings of this GPU's tensor pipe: csa_peak_mma (one
    CTA per SM, back-to-back tcgen05.mma on shared-memory operands), each launch
    ~20 ms, best of 10 (burst); with sustained_s > 0 also a back-to-back run of
    that many seconds per kind (mean rate)."""
    out = {}
    for kind, name in ((1, "mxf4"), (0, "bf16")):
        probe = 4096
        fl, ws = csa.csa_peak_mma(kind, probe)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fl, ws = csa.csa_peak_mma(kind, probe, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        per_iter_ms = e0.elapsed_time(e1) / probe
        iters = max(1024, int(20.0 / max(per_iter_ms, 1e-9)))
        best = 0.0
        for _ in range(10):
            e0.record()
            fl, ws = csa.csa_peak_mma(kind, iters, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            best = max(best, fl / (e0.elapsed_time(e1) * 1e-3) / 1e12)
        rec = {"burst_tflops": best, "iters_per_cta": iters}
        if sustained_s > 0:
            n = max(1, int(sustained_s * 1000 / 20))
            if sampler is not None:
                sampler.start()
            e0.record()
            for _ in range(n):
                fl, ws = csa.csa_peak_mma(kind, iters, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            if sampler is not None:
                sampler.stop()
                rec["clocks"] = sampler.summary()
                sampler.samples = []
            rec["sustained_tflops"] = fl * n / (e0.elapsed_time(e1) * 1e-3) / 1e12
            rec["sustained_s"] = e0.elapsed_time(e1) * 1e-3
        rec["status"] = csa.csa_check_status(ws)
        out[name] = rec
    return out


# ----------------------------------------------------------------- algorithmic work
def csa_prefill_work(wl):
    t = np.arange(wl.T, dtype=np.int64)
    nv = (t + 1) // wl.m
    pairs = int(nv.sum())
    visits = int((np.minimum(nv, wl.k) + np.minimum(t + 1, wl.W)).sum())
    return {
        "indexer_flop": 2.0 * pairs * wl.HI * wl.dI,
        "attn_flop": 4.0 * visits * wl.H * wl.d,
        "compress_bytes": 3 * wl.T * wl.d * 2 + 2 * (wl.T // wl.m) * wl.d * 2 + wl.m * wl.d * 4,
        "pairs": pairs, "visits": visits,
    }


def hca_prefill_work(wl):
    t = np.arange(wl.T, dtype=np.int64)
    nv = (t + 1) // wl.m_hca
    visits = int((nv + np.minimum(t + 1, wl.W_hca)).sum())
    return {"attn_flop": 4.0 * visits * wl.H * wl.d,
            "compress_bytes": 3 * wl.T * wl.d * 2 + 2 * (wl.T // wl.m_hca) * wl.d * 2 + wl.m_hca * wl.d * 4,
            "visits": visits}


def decode_bytes(wl, B=None):
    B = wl.batch if B is None else B
    n = wl.context // wl.m
    per = (n * (wl.dI // 2 + wl.dI // 32)            # every visible indexer key: codes + scales
           + wl.k * wl.d * 2 * 2                      # gathered compressed K and V rows
           + wl.W * wl.d * 2 * 2                      # raw window K and V
           + wl.H * wl.d * 2 + wl.HI * (wl.dI // 2 + wl.dI // 32) + wl.HI  # q, qI, w
           + wl.H * wl.d * 2 + wl.k * 4)              # O, idx
    return per * B


# ----------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[5 + i].lower() == "active"})
        under = [v for v in sm if v > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(under) if under else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------- timing helpers
class Timer:
    """CUDA events on the current stream around each named phase of a step."""

    def __init__(self, names):
        self.names = names
        self.events = []

    def step(self):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.names) + 1)]
        self.events.append(ev)
        return ev

    def per_phase_ms(self):
        out = {n: 0.0 for n in self.names}
        for ev in self.events:
            for i, n in enumerate(self.names):
                out[n] += ev[i].elapsed_time(ev[i + 1])
        k = max(1, len(self.events))
        return {n: v / k for n, v in out.items()}


def barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, dist_on, device="cuda"):
    """Max of a per-rank scalar over all ranks (the job's time is its slowest rank's)."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


def rank_seed(wl, rank):
    """Each rank runs its own sequence (independent problems, weak scaling)."""
    return wl.seed + 1000 * rank


# ----------------------------------------------------------------- workloads (ours)
def run_csa_prefill(csa, wl, steps, warmup, dist_on, rank):
    d = inputs.prefill_layer(wl, device="cuda", seed=rank_seed(wl, rank))
    scale = 1.0 / math.sqrt(wl.d)
    T, H = wl.T, wl.H
    Kc = torch.empty(T // wl.m, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    idx = torch.empty(T, wl.k, dtype=torch.int32, device="cuda")
    O = torch.empty_like(d["Q"])
    ws_bytes = max(csa.lib().csa_indexer_topk_workspace_bytes(T, T // wl.m, wl.HI, wl.dI, wl.k),
                   csa.lib().csa_sparse_attn_workspace_bytes(T, H, wl.d, wl.k, wl.W))
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    timer = Timer(["compress", "indexer_topk", "sparse_attn"])

    def step(ev=None):
        if ev: ev[0].record()
        csa.csa_compress(d["K"], d["V"], d["Z"], d["B"], wl.m, Kc=Kc, Vc=Vc)
        if ev: ev[1].record()
        csa.csa_indexer_topk(d["qI_codes"], d["qI_scales"], d["w_codes"], d["kI_codes"], d["kI_scales"], wl.m,
                             wl.k, idx=idx, want_scores=False, workspace=ws)
        if ev: ev[2].record()
        csa.csa_sparse_attn(d["Q"], Kc, Vc, idx, d["K"], d["V"], wl.W, scale, O=O, want_lse=False, workspace=ws)
        if ev: ev[3].record()

    for _ in range(warmup):
        step()
    barrier(dist_on)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step(timer.step())
    t1.record()
    barrier(dist_on)
    ms = t0.elapsed_time(t1) / steps
    status = csa.csa_check_status(ws)
    phases = timer.per_phase_ms()
    # e2e through the public API with host buffers: H2D of the step's inputs, D2H of O.
    # The step is pipelined over query chunks on three streams: the inputs every
    # chunk needs (K, V, Z, B, the indexer keys) go first and are compressed; then
    # chunk c's queries are copied in while chunk c-1 is scored and attended, and
    # chunk c-1's output is copied out (chunked calls give the unchunked result).
    host = {k: v.cpu().pin_memory() for k, v in d.items() if k != "B_hca"}
    O_host = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = O.numel() * O.element_size()
    dev = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
    shared = ("K", "V", "Z", "B", "kI_codes", "kI_scales")
    per_row = [k for k in host if k not in shared]  # query-row tensors: Q, qI codes / scales, w
    n_chunks = E2E_CHUNKS if T % E2E_CHUNKS == 0 and (T // E2E_CHUNKS) % wl.m == 0 else 1
    C = T // n_chunks
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step():
        main = torch.cuda.current_stream()
        for s_ in (s_in, s_comp, s_out):
            s_.wait_stream(main)
        ev_shared = torch.cuda.Event()
        ev_in = [torch.cuda.Event() for _ in range(n_chunks)]
        ev_done = [torch.cuda.Event() for _ in range(n_chunks)]
        with torch.cuda.stream(s_in):
            for k in shared:
                dev[k].copy_(host[k], non_blocking=True)
            ev_shared.record()
            for c in range(n_chunks):
                sl = slice(c * C, (c + 1) * C)
                for k in per_row:
                    dev[k][sl].copy_(host[k][sl], non_blocking=True)
                ev_in[c].record()
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_shared)
            csa.csa_compress(dev["K"], dev["V"], dev["Z"], dev["B"], wl.m, Kc=Kc, Vc=Vc)
            for c in range(n_chunks):
                t0c = c * C
                sl = slice(t0c, t0c + C)
                e1 = (t0c + C) // wl.m
                s_comp.wait_event(ev_in[c])
                csa.csa_indexer_topk(dev["qI_codes"][sl], dev["qI_scales"][sl], dev["w_codes"][sl],
                                     dev["kI_codes"][:e1], dev["kI_scales"][:e1], wl.m, wl.k, t0=t0c, idx=idx[sl],
                                     want_scores=False, workspace=ws)
                csa.csa_sparse_attn(dev["Q"][sl], Kc[:e1], Vc[:e1], idx[sl], dev["K"][: t0c + C],
                                    dev["V"][: t0c + C], wl.W, scale, t0=t0c, O=O[sl], want_lse=False, workspace=ws)
                ev_done[c].record()
        with torch.cuda.stream(s_out):
            for c in range(n_chunks):
                sl = slice(c * C, (c + 1) * C)
                s_out.wait_event(ev_done[c])
                O_host[sl].copy_(O[sl], non_blocking=True)
        for s_ in (s_in, s_comp, s_out):
            main.wait_stream(s_)

    O_dev_ref = O.clone()  # output of the device-resident (timed) path, same inputs
    e2e_step()
    barrier(dist_on)
    e2e_matches = bool(torch.equal(O_host, O_dev_ref.cpu()))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(steps, 3))
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    barrier(dist_on)
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    del dev, host
    return {"ms": ms, "phases": phases, "status": status, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h,
            "launches_per_step": 4,  # compress, indexer, top-k sort (finalize), attention
            "e2e_chunks": n_chunks, "e2e_matches": e2e_matches}


def run_hca_prefill(csa, wl, steps, warmup):
    d = inputs.prefill_layer(wl, device="cuda", with_indexer=False)
    scale = 1.0 / math.sqrt(wl.d)
    Kc = torch.empty(wl.T // wl.m_hca, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)
    O = torch.empty_like(d["Q"])
    ws = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    timer = Timer(["compress", "hca_attn"])

    def step(ev=None):
        if ev: ev[0].record()
        csa.csa_compress(d["K"], d["V"], d["Z"], d["B_hca"], wl.m_hca, Kc=Kc, Vc=Vc)
        if ev: ev[1].record()
        csa.hca_attn(d["Q"], Kc, Vc, d["K"], d["V"], wl.m_hca, wl.W_hca, scale, O=O, want_lse=False, workspace=ws)
        if ev: ev[2].record()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step(timer.step())
    t1.record()
    torch.cuda.synchronize()
    return {"ms": t0.elapsed_time(t1) / steps, "phases": timer.per_phase_ms(), "status": csa.csa_check_status(ws)}


def run_decode(csa, wl, steps, warmup):
    d = inputs.decode_batch(wl, device="cuda")
    scale = 1.0 / math.sqrt(wl.d)
    pos = [wl.context - 1] * wl.batch
    O = torch.empty_like(d["q"])
    idx = torch.empty(wl.batch, wl.k, dtype=torch.int32, device="cuda")
    ws = None

    def step():
        nonlocal ws
        _, _, _, _, ws = csa.csa_decode(d["q"], d["qI_codes"], d["qI_scales"], d["w_codes"], d["Kc"], d["Vc"],
                                        d["kI_codes"], d["kI_scales"], d["Kwin"], d["Vwin"], pos, wl.m, wl.k, scale,
                                        O=O, idx=idx, want_lse=False, want_sel=True, workspace=ws)

    for _ in range(warmup):
        step()
    # L2 is smaller than the streamed indexer keys (285 MB), so back-to-back steps read HBM.
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    return {"ms": t0.elapsed_time(t1) / steps, "status": csa.csa_check_status(ws)}


def stack_work(wl):
    t = np.arange(wl.T, dtype=np.int64)
    nv1 = (t + 1) // wl.m
    nv2 = (t + 1) // wl.m_hca
    win = np.minimum(t + 1, wl.W)
    return {"indexer_flop": 2.0 * float(nv1.sum()) * wl.HI * wl.dI,
            "csa_attn_flop": 4.0 * float((np.minimum(nv1, wl.k) + win).sum()) * wl.H * wl.d,
            "hca_attn_flop": 4.0 * float((nv2 + np.minimum(t + 1, wl.W_hca)).sum()) * wl.H * wl.d,
            "projection_flop": 2.0 * wl.T * wl.H * wl.d * wl.d}


def run_stack(csa, wl, steps, warmup):
    from long_context_compressed_gated_b200.stack import stack_inputs, stack_prefill_chunked
    l1, l2, P = stack_inputs(wl, device="cuda")
    O2 = torch.empty_like(l1["Q"])

    def step(events=None):
        stack_prefill_chunked(l1, l2, P, wl.chunk, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca, out=O2,
                              phase_events=events)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    events = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step(events)
    t1.record()
    torch.cuda.synchronize()
    phases = {}
    for name, e0, e1 in events:
        phases[name] = phases.get(name, 0.0) + e0.elapsed_time(e1) / steps
    return {"ms": t0.elapsed_time(t1) / steps, "phases": phases}


class _OneRank:
    """The all-gather of a single rank (no process group)."""
    rank, world = 0, 1

    def all_gather(self, flat):
        return [flat]


def run_sharded_stack(csa, wl, steps, warmup, dist_on, rank, world):
    """The two-layer stack of ONE sequence token-sharded over the ranks (zig-zag
    chunks, one all-gather of compressed entries + halos per layer): strong
    scaling, the job's time is its slowest rank's."""
    from long_context_compressed_gated_b200.sharded import ShardedPrefill, TorchComm, shard_inputs
    from long_context_compressed_gated_b200.stack import stack_inputs
    l1, l2, P = stack_inputs(wl, device="cuda")
    sp = ShardedPrefill(wl.T, world, wl.m, wl.k, wl.W, wl.m_hca, wl.W_hca)
    x = shard_inputs(l1, l2, P, rank, world, wl.T, wl.m)
    comm = TorchComm() if dist_on else _OneRank()
    for _ in range(warmup):
        sp.run(x, comm)
    barrier(dist_on)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        sp.run(x, comm)
    t1.record()
    barrier(dist_on)
    return max_over_ranks(t0.elapsed_time(t1) / steps, dist_on)


# ----------------------------------------------------------------- CPU oracle (reference arm / baseline)
def _boundary_rows(wl):
    """Rows every CPU sample includes: 0, m-1, m, W-1, W, the rows where the
    visible count reaches k, and T-1."""
    r = {0, wl.m - 1, wl.m, wl.W - 1, wl.W, wl.k * wl.m - 1, wl.k * wl.m, wl.T - 1}
    return sorted(x for x in r if 0 <= x < wl.T)


class OracleCSA:
    """The CPU oracle on the CSA prefill workload: compression of every block
    once, then indexer + top-k + attention for batches of query rows (boundary
    rows first, then a seeded permutation)."""

    def __init__(self, wl):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.d = inputs.prefill_layer(wl)
        self.scale = 1.0 / math.sqrt(wl.d)
        self.nthreads = oracle.default_threads()
        t = time.perf_counter()
        Kc64, Vc64 = oracle.compress(self.d["K"], self.d["V"], self.d["Z"], self.d["B"], wl.m, self.nthreads)
        self.Kcw, self.Vcw = oracle.to_bf16_words(Kc64), oracle.to_bf16_words(Vc64)
        self.t_comp = time.perf_counter() - t
        b = _boundary_rows(wl)
        rest = np.random.default_rng(0).permutation(wl.T)
        self.order = np.concatenate([np.array(b, np.int64), rest[~np.isin(rest, b)]])
        self.done = 0

    def rows(self, n):
        r = np.sort(self.order[self.done:self.done + n])
        self.done += len(r)
        return r

    def run_rows(self, rows):
        o, d, wl = self.oracle, self.d, self.wl
        I = o.indexer(d["qI_codes"], d["qI_scales"], d["w_codes"], d["kI_codes"], d["kI_scales"], 0, wl.m, rows,
                      self.nthreads)
        sel, _ = o.topk(I, o.n_vis(rows, wl.m), wl.k, self.nthreads)
        o.attention(d["Q"], self.Kcw, self.Vcw, d["K"], d["V"], 0, wl.m, wl.W, self.scale, sel=sel, rows=rows,
                    nthreads=self.nthreads)

    def timed(self, seconds, batch=None):
        """Rows processed in about `seconds`; returns (rows, seconds)."""
        batch = batch or max(8, self.nthreads)
        n, t_rows = 0, 0.0
        while t_rows < seconds and self.done < self.wl.T:
            r = self.rows(batch)
            t1 = time.perf_counter()
            self.run_rows(r)
            t_rows += time.perf_counter() - t1
            n += len(r)
        return n, t_rows


def oracle_sample(wl, seconds=8.0):
    """Time the CPU oracle on a bounded sample of the CSA prefill workload and
    extrapolate the full step as compress + T * (time per row)."""
    oc = OracleCSA(wl)
    n, t_rows = oc.timed(seconds)
    total_s = oc.t_comp + t_rows / n * wl.T
    return {"tokens_per_s": wl.T / total_s, "rows": n, "seconds": oc.t_comp + t_rows, "cores": oc.nthreads,
            "sample": "compression of all %d blocks + indexer/top-k/attention of %d query rows of %d (the boundary "
                      "rows %s, then seeded random rows; %.1f s of CPU time); full step extrapolated as compress + "
                      "T x time per row" % (wl.T // wl.m, n, wl.T, _boundary_rows(wl), oc.t_comp + t_rows)}


def oracle_other_configs():
    """The oracle on the other workloads: the tiny layer and the 1M-context decode
    in full, the HCA prefill and the two-layer stack on seeded rows that include
    the boundary rows (time per row and an extrapolated full time, so labelled)."""
    import oracle
    out = {}
    nth = oracle.default_threads()
    # tiny CSA + HCA layer, in full
    wl = inputs.TINY
    d = inputs.prefill_layer(wl)
    sc = 1.0 / math.sqrt(wl.d)
    t = time.perf_counter()
    oracle.csa_layer(d, wl.m, wl.k, wl.W, sc, nthreads=nth)
    K2, V2 = oracle.compress(d["K"], d["V"], d["Z"], d["B_hca"], wl.m_hca, nth)
    oracle.attention(d["Q"], oracle.to_bf16_words(K2), oracle.to_bf16_words(V2), d["K"], d["V"], 0, wl.m_hca,
                     wl.W_hca, sc, nthreads=nth)
    out[wl.name] = {"seconds": time.perf_counter() - t, "scope": "full (CSA and HCA layer, all %d rows)" % wl.T}
    # 1M-context decode, all 16 sequences, generated on the GPU and copied to the host
    wl = inputs.CSA_DECODE
    g = inputs.decode_batch(wl, device="cuda")
    h = {k: v.cpu() for k, v in g.items()}
    del g
    torch.cuda.empty_cache()
    sc = 1.0 / math.sqrt(wl.d)
    t = time.perf_counter()
    pos = wl.context - 1

    def one_sequence(b):  # one query row per sequence: the sequences go to separate threads
        I = oracle.indexer(h["qI_codes"][b:b + 1], h["qI_scales"][b:b + 1], h["w_codes"][b:b + 1], h["kI_codes"][b],
                           h["kI_scales"][b], pos, wl.m, nthreads=1)
        sel, _ = oracle.topk(I, oracle.n_vis([pos], wl.m), wl.k, 1)
        oracle.attention(h["q"][b:b + 1], h["Kc"][b], h["Vc"][b], h["Kwin"][b], h["Vwin"][b], pos, wl.m, wl.W, sc,
                         sel=sel, rows=[0], raw_pos0=pos - wl.W + 1, nthreads=1)

    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(max_workers=min(nth, wl.batch)) as ex:
        list(ex.map(one_sequence, range(wl.batch)))
    dt = time.perf_counter() - t
    out[wl.name] = {"seconds": dt, "us_per_step": dt * 1e6, "threads": min(nth, wl.batch),
                    "scope": "full (16 sequences, one step, a thread per sequence)"}
    del h
    # HCA prefill, 128 rows
    wl = inputs.HCA_PREFILL
    d = inputs.prefill_layer(wl, with_indexer=False)
    sc = 1.0 / math.sqrt(wl.d)
    t = time.perf_counter()
    K2, V2 = oracle.compress(d["K"], d["V"], d["Z"], d["B_hca"], wl.m_hca, nth)
    t_comp = time.perf_counter() - t
    rows = np.array(sorted(set([0, wl.m_hca - 1, wl.m_hca, wl.W_hca - 1, wl.W_hca, wl.T - 1]) |
                           set(np.random.default_rng(2).choice(wl.T, 122, replace=False).tolist())), np.int64)
    t = time.perf_counter()
    oracle.attention(d["Q"], oracle.to_bf16_words(K2), oracle.to_bf16_words(V2), d["K"], d["V"], 0, wl.m_hca,
                     wl.W_hca, sc, rows=rows, nthreads=nth)
    per_row = (time.perf_counter() - t) / len(rows)
    out[wl.name] = {"rows": len(rows), "s_per_row": per_row, "compress_s": t_comp,
                    "extrapolated_full_s": t_comp + per_row * wl.T,
                    "tokens_per_s_extrapolated": wl.T / (t_comp + per_row * wl.T),
                    "scope": "compression of all blocks + attention of %d rows incl. boundary rows; extrapolated"
                             % len(rows)}
    del d
    return out


EXTRA_CASES = ("hca_prefill", "csa_decode", "stack", "fp8_decode", "append", "quantize", "compress")


def _event_ms(fn, reps, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_fp8_decode(csa, wl, steps, warmup):
    """The 1M-context decode over the MXFP8 compressed cache (E4M3 + E8M0 per 32)."""
    d = inputs.decode_batch(wl, device="cuda")
    scale = 1.0 / math.sqrt(wl.d)
    pos = [wl.context - 1] * wl.batch
    Kq, Ks = csa.csa_mxfp8_quantize(d["Kc"])
    Vq, Vs = csa.csa_mxfp8_quantize(d["Vc"])
    del d["Kc"], d["Vc"]
    torch.cuda.empty_cache()
    O = torch.empty_like(d["q"])
    idx = torch.empty(wl.batch, wl.k, dtype=torch.int32, device="cuda")
    ws = [None]

    def step():
        r = csa.csa_decode_fp8(d["q"], d["qI_codes"], d["qI_scales"], d["w_codes"], Kq, Ks, Vq, Vs, d["kI_codes"],
                               d["kI_scales"], d["Kwin"], d["Vwin"], pos, wl.m, wl.k, scale, O=O, idx=idx,
                               want_lse=False, workspace=ws[0])
        ws[0] = r[4]

    ms = _event_ms(step, max(5, steps), warmup)
    return {"ms": ms, "status": csa.csa_check_status(ws[0])}


def run_append(csa, wl, steps):
    """One decode-append step for B sequences: the tokens complete a block, so the
    window shifts, the block is pooled into the cache and its indexer key copied."""
    B, d, m, W = wl.batch, wl.d, wl.m, wl.W
    Ncap = 4096
    g = lambda *s: torch.randn(*s, device="cuda").to(torch.bfloat16)
    Kn, Vn, Zn = g(B, d), g(B, d), g(B, d)
    Bias = torch.randn(m, d, device="cuda") * 0.5
    Kw, Vw = g(B, W, d), g(B, W, d)
    Kb, Vb, Zb = g(B, m, d), g(B, m, d), g(B, m, d)
    Kc, Vc = g(B, Ncap, d), g(B, Ncap, d)
    kn = torch.zeros(B, wl.dI // 2, dtype=torch.uint8, device="cuda")
    ksn = torch.full((B, wl.dI // 32), 127, dtype=torch.uint8, device="cuda")
    kc = torch.zeros(B, Ncap, wl.dI // 2, dtype=torch.uint8, device="cuda")
    ks = torch.zeros(B, Ncap, wl.dI // 32, dtype=torch.uint8, device="cuda")
    pos = [m * 100 - 1] * B  # completes block 99
    ms = _event_ms(lambda: csa.csa_decode_append(Kn, Vn, Zn, Bias, pos, Kw, Vw, Kb, Vb, Zb, Kc, Vc, kI_codes_new=kn,
                                                 kI_scales_new=ksn, kI_codes=kc, kI_scales=ks), max(20, steps))
    # bytes: new rows in, window read + written, staged rows read, entry and key written
    by = B * (3 * d * 2 + 2 * 2 * (W - 1) * d * 2 + 2 * d * 2 + 3 * (m - 1) * d * 2 + 2 * d * 2 + wl.dI // 2 + wl.dI // 32)
    return {"us_per_step": ms * 1e3, "bytes": by}


def run_quantize(csa, steps):
    """The two quantisers on large bf16 tensors: MXFP4 of the cfg1 indexer queries
    [32768, 64, 128] and MXFP8 of one sequence's 1M-context cache [262144, 128] x 16."""
    out = {}
    x4 = torch.randn(32768, 64, 128, device="cuda").to(torch.bfloat16)
    ms = _event_ms(lambda: csa.csa_mxfp4_quantize(x4, mode=1), max(5, steps))
    by = x4.numel() * 2 + x4.numel() // 2 + x4.numel() // 32
    out["mxfp4_indexer_q_32768x64x128"] = {"ms": ms, "gbs": by / (ms * 1e-3) / 1e9}
    del x4
    x8 = torch.randn(16 * 262144, 128, device="cuda").to(torch.bfloat16)
    ms = _event_ms(lambda: csa.csa_mxfp8_quantize(x8), max(5, steps))
    by = x8.numel() * 2 + x8.numel() + x8.numel() // 32
    out["mxfp8_cache_16x262144x128"] = {"ms": ms, "gbs": by / (ms * 1e-3) / 1e9}
    return out


def run_compress(csa, wl, steps):
    """The gated compression of the HCA prefill workload alone (m' = 128, 131072
    tokens: 100 MB of K, V, Z).  The inputs fit in L2, so the launches cycle
    through three copies of them (303 MB, more than twice L2): every launch reads
    inputs that the two launches before it have evicted, and L2 then holds only
    clean lines (a flush by writing a large buffer leaves dirty lines whose
    write-back would land in the timed kernel).  The launches are queued behind a
    short device-side sleep so that the host's call time stays out of the
    measurement."""
    sets = [inputs.prefill_layer(wl, device="cuda", with_indexer=False, with_q=False) for _ in range(3)]
    Kc = torch.empty(wl.T // wl.m_hca, wl.d, dtype=torch.bfloat16, device="cuda")
    Vc = torch.empty_like(Kc)

    def launch(i):
        d = sets[i % len(sets)]
        csa.csa_compress(d["K"], d["V"], d["Z"], d["B_hca"], wl.m_hca, Kc=Kc, Vc=Vc)

    reps = 3 * max(50, steps)
    for i in range(6):
        launch(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(20_000_000)  # ~10 ms at 2 GHz: the host queues all launches meanwhile
    e0.record()
    for i in range(reps):
        launch(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    by = 3 * wl.T * wl.d * 2 + 2 * (wl.T // wl.m_hca) * wl.d * 2 + wl.m_hca * wl.d * 4
    return {"ms": ms, "bytes": by}


def run_extra(name, csa, peaks, steps, warmup, T=None):
    """One of the workloads reported under "workloads" (T overrides its length)."""
    import dataclasses
    if name == "hca_prefill":
        w2 = inputs.HCA_PREFILL if T is None else dataclasses.replace(inputs.HCA_PREFILL, T=T)
        r2 = run_hca_prefill(csa, w2, max(3, steps // 2), warmup)
        hw = hca_prefill_work(w2)
        return {"hca_prefill_T%d" % w2.T: {
            "tokens_per_s": w2.T / (r2["ms"] * 1e-3), "ms_per_step": r2["ms"],
            "attn_tflops": hw["attn_flop"] / (r2["phases"]["hca_attn"] * 1e-3) / 1e12,
            "attn_frac_bf16": hw["attn_flop"] / (r2["phases"]["hca_attn"] * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "compress_gbs": hw["compress_bytes"] / (r2["phases"]["compress"] * 1e-3) / 1e9,
            "phases_ms": r2["phases"], "status": r2["status"]}}
    if name == "csa_decode":
        w3 = inputs.CSA_DECODE if T is None else dataclasses.replace(inputs.CSA_DECODE, context=T)
        r3 = run_decode(csa, w3, max(5, steps), warmup)
        by = decode_bytes(w3)
        return {"csa_decode_B%d_L%s" % (w3.batch, "1M" if w3.context == 1 << 20 else str(w3.context)): {
            "us_per_step": r3["ms"] * 1e3, "algorithmic_bytes": by, "gbs": by / (r3["ms"] * 1e-3) / 1e9,
            "frac_hbm": by / (r3["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], "status": r3["status"]}}
    if name == "fp8_decode":
        w3 = inputs.CSA_DECODE if T is None else dataclasses.replace(inputs.CSA_DECODE, context=T)
        r = run_fp8_decode(csa, w3, steps, warmup)
        n = w3.context // w3.m
        # as the bf16 decode's bytes, with the gathered entries in 1 byte + 1/32 scale byte per channel
        by = decode_bytes(w3) - w3.batch * w3.k * w3.d * 2 * 2 + w3.batch * w3.k * (w3.d + w3.d // 32) * 2
        return {"csa_decode_fp8cache_B%d_L%s" % (w3.batch, "1M" if w3.context == 1 << 20 else str(w3.context)): {
            "us_per_step": r["ms"] * 1e3, "algorithmic_bytes": by, "gbs": by / (r["ms"] * 1e-3) / 1e9,
            "frac_hbm": by / (r["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], "entries_per_sequence": n,
            "status": r["status"]}}
    if name == "append":
        r = run_append(csa, inputs.CSA_DECODE, steps)
        return {"csa_decode_append_B16": {"us_per_step": r["us_per_step"], "bytes": r["bytes"],
                                          "gbs": r["bytes"] / (r["us_per_step"] * 1e-6) / 1e9}}
    if name == "compress":
        w2 = inputs.HCA_PREFILL if T is None else dataclasses.replace(inputs.HCA_PREFILL, T=T)
        r = run_compress(csa, w2, steps)
        gbs = r["bytes"] / (r["ms"] * 1e-3) / 1e9
        return {"compress_hca_T%d_m%d" % (w2.T, w2.m_hca): {"ms": r["ms"], "bytes": r["bytes"], "gbs": gbs,
                                                           "frac_hbm": gbs / peaks["hbm_gbs"],
                                                           "l2": "three input copies in turn (303 MB)"}}
    if name == "quantize":
        return {"quantize": {k: dict(v, frac_hbm=v["gbs"] / peaks["hbm_gbs"]) for k, v in run_quantize(csa, steps).items()}}
    if name == "stack":
        w4 = inputs.STACK if T is None else dataclasses.replace(inputs.STACK, T=T)
        r4 = run_stack(csa, w4, 2, 1)
        sw = stack_work(w4)
        ph4 = r4["phases"]
        method_ms = r4["ms"] - ph4.get("projection", 0.0)
        return {"csa_hca_stack_T%d_chunk%d" % (w4.T, w4.chunk): {
            "tokens_per_s": w4.T / (r4["ms"] * 1e-3), "ms_per_step": r4["ms"],
            "tokens_per_s_without_projection": w4.T / (method_ms * 1e-3),
            "indexer_tflops": sw["indexer_flop"] / (ph4["indexer_topk"] * 1e-3) / 1e12,
            "csa_attn_tflops": sw["csa_attn_flop"] / (ph4["sparse_attn"] * 1e-3) / 1e12,
            "hca_attn_tflops": sw["hca_attn_flop"] / (ph4["hca_attn"] * 1e-3) / 1e12,
            "phases_ms": ph4, "projection_excluded_from_method": True}}
    raise ValueError(name)


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the HCA and decode workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default="all", choices=("all", "csa_prefill", "peaks", "sharded_stack") + EXTRA_CASES,
                    help="all: the CSA prefill line plus the other workloads; csa_prefill: that line alone; "
                         "otherwise one other workload alone, on one GPU (for profiling)")
    ap.add_argument("--T", type=int, default=None,
                    help="with --case: override the sequence length (the context length for csa_decode)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = inputs.CSA_PREFILL
    if args.case == "csa_prefill" and args.T is not None:
        import dataclasses
        wl = dataclasses.replace(wl, T=args.T)

    if args.impl == "reference":
        if rank != 0:
            return
        # each step = one bounded sample of the workload's query rows (a budget that
        # keeps the whole --steps K --warmup W run within a few minutes); the value
        # is the workload's tokens/s extrapolated from the rows done per second
        oc = OracleCSA(wl)
        budget = min(8.0, 150.0 / max(1, args.steps + args.warmup))
        for _ in range(args.warmup):
            oc.timed(budget / 4)
        step_s, rows_done = [], 0
        for _ in range(args.steps):
            n, t_rows = oc.timed(budget)
            if n == 0:
                break
            step_s.append(t_rows)
            rows_done += n
        t_rows = sum(step_s)
        per_row = t_rows / max(1, rows_done)
        v = wl.T / (oc.t_comp + per_row * wl.T)
        sample = ("each step: indexer/top-k/attention of a batch of query rows for ~%.1f s (boundary rows %s first, "
                  "then seeded random rows); %d rows over %d steps; compression of all %d blocks (%.2f s) once; "
                  "tokens/s extrapolated as T / (compress + T x time per row)"
                  % (budget, _boundary_rows(wl), rows_done, len(step_s), wl.T // wl.m, oc.t_comp))
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": len(step_s), "warmup": args.warmup,
                "ms_per_step": 1000.0 * t_rows / max(1, len(step_s)), "rows_per_step": rows_done / max(1, len(step_s)),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "d": wl.d, "m": wl.m,
                                                 "k": wl.k, "W": wl.W, "HI": wl.HI, "dI": wl.dI},
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oc.nthreads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    import long_context_compressed_gated_b200 as csa
    csa.lib()
    peaks = load_peaks()
    if args.case == "peaks":
        if rank == 0:
            sm = ClockSampler(local)
            print(json.dumps({"case": "peaks", "tensor_peaks": measure_tensor_peaks(csa, sustained_s=4.0, sampler=sm),
                              "cublas_bf16_measured": peaks}), flush=True)
        if dist_on:
            torch.distributed.destroy_process_group()
        return
    tensor_peaks = measure_tensor_peaks(csa)
    peaks["mxf4_tflops"] = tensor_peaks["mxf4"]["burst_tflops"]
    peaks["mxf4_source"] = "measured: csa_peak_mma loop, best of 10"
    peaks["bf16_mma_loop_tflops"] = tensor_peaks["bf16"]["burst_tflops"]
    if args.case == "sharded_stack":
        wls = inputs.STACK if args.T is None else __import__("dataclasses").replace(inputs.STACK, T=args.T)
        ms = run_sharded_stack(csa, wls, args.steps, args.warmup, dist_on, rank, world)
        if rank == 0:
            print(json.dumps({"case": "sharded_stack", "metric": METRIC, "value": wls.T / (ms * 1e-3),
                              "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": ms, "scaling": "strong",
                              "config": {"workload": wls.name, "T": wls.T, "parallelism": "token-sharded zig-zag, "
                                         "one all-gather of compressed entries + halos per layer"}}), flush=True)
        if dist_on:
            torch.distributed.destroy_process_group()
        return
    if args.case in EXTRA_CASES:
        if rank == 0:
            print(json.dumps({"case": args.case, "workloads": run_extra(args.case, csa, peaks, args.steps,
                                                                         args.warmup, args.T)}), flush=True)
        if dist_on:
            torch.distributed.destroy_process_group()
        return
    work = csa_prefill_work(wl)

    sampler = ClockSampler(local)
    sampler.start()
    res = run_csa_prefill(csa, wl, args.steps, args.warmup, dist_on, rank)
    sampler.stop()
    ms = max_over_ranks(res["ms"], dist_on)
    e2e_ms = max_over_ranks(res["e2e_ms"], dist_on)

    extra = {}
    if not args.no_extra and args.case == "all" and rank == 0:
        for name in EXTRA_CASES:
            extra.update(run_extra(name, csa, peaks, args.steps, args.warmup))
            torch.cuda.empty_cache()

    ph = res["phases"]
    dominant = max(ph, key=ph.get)
    idx_tf = work["indexer_flop"] / (ph["indexer_topk"] * 1e-3) / 1e12
    attn_tf = work["attn_flop"] / (ph["sparse_attn"] * 1e-3) / 1e12
    comp_gbs = work["compress_bytes"] / (ph["compress"] * 1e-3) / 1e9
    fp4_peak = peaks["mxf4_tflops"]
    same_cfg = wl.T == inputs.CSA_PREFILL.T
    if dominant == "indexer_topk":
        roof = {"kernel": "indexer_topk", "bound": "tensor", "achieved": idx_tf, "peak": fp4_peak,
                "unit": "TFLOP/s", "frac": idx_tf / fp4_peak,
                "traffic": PHASE_TRAFFIC["indexer_topk"][0] if same_cfg else None,
                "traffic_source": PHASE_TRAFFIC["indexer_topk"][1],
                "peak_note": "measured kind::mxf4 peak (tcgen05 MMA loop on this GPU, burst, best of 10); "
                             "NVIDIA's dense FP4 figure %.0f TFLOP/s for context" % NOMINAL_FP4_TFLOPS}
    elif dominant == "sparse_attn":
        roof = {"kernel": "sparse_attn", "bound": "tensor", "achieved": attn_tf, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": attn_tf / peaks["bf16_tflops"],
                "traffic": PHASE_TRAFFIC["sparse_attn"][0] if same_cfg else None,
                "traffic_source": PHASE_TRAFFIC["sparse_attn"][1],
                "peak_note": "bf16 burst, %s" % peaks["source"]}
    else:
        roof = {"kernel": "compress", "bound": "hbm", "achieved": comp_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": comp_gbs / peaks["hbm_gbs"], "traffic": None}
    total_tokens = wl.T * world
    value = job_throughput(wl.T, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16+mxfp4", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "d": wl.d, "m": wl.m, "k": wl.k, "W": wl.W,
                   "HI": wl.HI, "dI": wl.dI, "sequences_per_gpu": 1, "parallelism": "independent sequences per GPU",
                   "l2": "inputs larger than L2 (Q alone %d MiB), no flush" % (wl.T * wl.H * wl.d * 2 >> 20)},
        "roofline": roof,
        "kernels": {"compress_ms": ph["compress"], "compress_gbs": comp_gbs,
                    "indexer_topk_ms": ph["indexer_topk"], "indexer_tflops": idx_tf,
                    "indexer_frac_fp4": idx_tf / fp4_peak,
                    "sparse_attn_ms": ph["sparse_attn"], "sparse_attn_tflops": attn_tf,
                    "sparse_attn_frac_bf16": attn_tf / peaks["bf16_tflops"]},
        "e2e": {"value": job_throughput(wl.T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"], "pipelined_chunks": res["e2e_chunks"],
                "output_equals_device_path": res["e2e_matches"]},
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": sampler.summary(),
        "device_status": res["status"],
        "peaks": peaks,
        "tensor_peaks": tensor_peaks,
        "workloads": extra,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample(wl, seconds=8.0)
        line["cpu_baseline"] = {"value": r["tokens_per_s"], "unit": "tokens/s", "cores": r["cores"],
                                "kind": "oracle", "sample": r["sample"]}
        if args.case == "all" and not args.no_extra:
            line["cpu_baseline"]["other_workloads"] = oracle_other_configs()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
