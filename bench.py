"""Benchmark of the CSA layer hot path on B200.

Headline: CSA decode queries/s at 128K context (32 sequences, one new token
each, 32,768 compressed entries per sequence, top-k 1024, window 128, 64
query heads x 512, BF16). One step = one decode step of the layer:
  compressor projection of the new token (main entries and index keys),
  preparation of its window row into the ring, lightning indexer + top-k
  over all visible entries, sparse shared-KV attention with window and sink.
Secondary (same JSON line, key "prefill"): CSA prefill tokens/s at T=8192.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own batch (weak scaling, no data-path
collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import compressed_sparse_attention_17_b200 as csa  # noqa: E402
from compressed_sparse_attention_17_b200 import synth  # noqa: E402

L2_FLUSH_BYTES = 256 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- device helpers
def to_dev(spec: synth.Spec, device) -> torch.Tensor:
    st = spec.storage()
    t = torch.from_numpy(st)
    if spec.dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device, non_blocking=False)


def to_pinned(spec: synth.Spec) -> torch.Tensor:
    st = spec.storage()
    t = torch.from_numpy(st)
    if spec.dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.pin_memory()


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "20"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *exc):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        for line in Path(self.f.name).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- decode workload
class Decode:
    """The decode workload on one GPU: caches resident in HBM, per-step inputs."""

    def __init__(self, w: synth.Workload, device):
        self.w, self.dev = w, device
        B, N, c, cI, m = w.B, w.n_entries, w.c, w.c_I, w.m
        s = w.specs()
        self.s = s
        t0 = time.time()
        self.g = csa.geom(c=c, rope_dims=w.rope_dims, win_ring=1, n_win=w.n_win)
        self.gI = csa.geom(c=cI, rope_dims=0)
        self.ldE = N + 8
        mixed = w.kv_mixed
        # compressed main entries: raw rows prepared (RMSNorm, RoPE at i*m) on the GPU
        raw = to_dev(s["E_raw"], device)
        if mixed:
            self.E = torch.zeros(B, self.ldE, csa.MIXED_ROW_BYTES, dtype=torch.uint8, device=device)
        else:
            self.E = torch.zeros(B, self.ldE, c, dtype=torch.bfloat16, device=device)
        for b in range(B):
            csa.rmsnorm_rope(raw[b], self.g, pos0=0, pos_step=m, out=self.E[b, :N],
                             out_dtype=csa.CSA_FP8_MIXED if mixed else None)
        del raw
        self.KI = torch.zeros(B, self.ldE, cI, dtype=torch.bfloat16, device=device)
        self.KI[:, :N] = to_dev(s["KI"], device)
        # window ring: slot j mod n_win holds position j, prepared at j
        p = w.L
        slots = np.arange(w.n_win)
        wpos = p - ((p - slots) % w.n_win)
        win_raw = to_dev(s["win_raw"], device)
        self.ring = torch.empty(B, w.n_win, c, dtype=torch.bfloat16, device=device)
        for b in range(B):
            csa.rmsnorm_rope(win_raw[b], self.g, pos=torch.from_numpy(wpos).to(device),
                             out=self.ring[b])
        self.kv_new = win_raw[:, p % w.n_win].contiguous()
        # per-step inputs (host copies are pinned for the end-to-end leg)
        self.host = {n: to_pinned(s[n]) for n in ("q", "qI", "w", "h")}
        self.host["kv_new"] = self.kv_new.cpu().pin_memory()
        self.host["pos"] = torch.full((B,), p, dtype=torch.int64).pin_memory()
        self.host["out_row"] = (torch.arange(B, dtype=torch.int64) * w.n_win + p % w.n_win).pin_memory()
        self.inp = {n: t.to(device) for n, t in self.host.items()}
        self.W = {n: to_dev(s[n], device) for n in ("W_aKV", "W_bKV", "W_aZ", "W_bZ", "WI_aKV",
                                                     "WI_bKV", "WI_aZ", "WI_bZ")}
        self.bias = to_dev(s["bias"], device)
        self.biasI = to_dev(s["biasI"], device)
        self.sink = to_dev(s["sink"], device)
        self.state = csa.decode_state(B, self.g, device)
        self.stateI = csa.decode_state(B, self.gI, device)
        self.seq = torch.arange(B, dtype=torch.int32, device=device)
        self.ne = torch.full((B,), N, dtype=torch.int64, device=device)
        self.idx = torch.empty(B, w.k, dtype=torch.int32, device=device)
        self.O = torch.empty(B, w.H_q, c, dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(max(16, csa.load().csa_index_topk_workspace_size(B, self.ldE, w.k)),
                              dtype=torch.uint8, device=device)
        self.host_O = torch.empty_like(self.O, device="cpu").pin_memory()
        torch.cuda.synchronize(device)
        log(f"[decode] setup {time.time() - t0:.1f}s: B={B} entries={N} "
            f"{'mixed FP8' if mixed else 'BF16'} cache")

    def step(self, inp, ev=None, O=None):
        W = self.W
        csa.compress_decode(inp["h"], inp["pos"], W["W_aKV"], W["W_aZ"], self.bias, self.state,
                            self.E, self.g, W_bKV=W["W_bKV"], W_bZ=W["W_bZ"])
        csa.compress_decode(inp["h"], inp["pos"], W["WI_aKV"], W["WI_aZ"], self.biasI,
                            self.stateI, self.KI, self.gI, W_bKV=W["WI_bKV"], W_bZ=W["WI_bZ"])
        csa.rmsnorm_rope(inp["kv_new"], self.g, pos=inp["pos"], out=self.ring.view(-1, self.w.c),
                         out_row=inp["out_row"])
        if ev is not None:
            ev[0].record()
        csa.index_topk(inp["qI"], inp["w"], self.KI, self.seq, inp["pos"], self.ne, self.w.k,
                       self.g, workspace=self.ws, out=self.idx)
        if ev is not None:
            ev[1].record()
        csa.attend(inp["q"], self.sink, self.E, self.idx, self.ring, self.seq, inp["pos"],
                   self.ne, self.g, out=self.O if O is None else O)
        if ev is not None and len(ev) > 2:
            ev[2].record()

    def capture(self):
        """Record one decode step (all of its library launches) as a CUDA
        graph; replays launch the same kernels on the same buffers."""
        self.step(self.inp)
        torch.cuda.synchronize(self.dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step(self.inp)
        torch.cuda.synchronize(self.dev)

    def step_graph(self, ev=None):
        self.graph.replay()

    def setup_pipeline(self):
        """A second set of step inputs and outputs (and, with graphs, a second
        graph on them), so that one step's copies overlap another's kernels."""
        second = {n: t.clone() for n, t in self.inp.items()}
        self.inp2 = [self.inp, second]
        self.O2 = [self.O, torch.empty_like(self.O)]
        self.host_O2 = [self.host_O, torch.empty_like(self.host_O).pin_memory()]
        self.graphs = None
        if getattr(self, "graph", None) is not None:
            self.step(second, O=self.O2[1])
            torch.cuda.synchronize(self.dev)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                self.step(second, O=self.O2[1])
            self.graphs = [self.graph, g2]
        self.s_h2d = torch.cuda.Stream(self.dev)
        self.s_d2h = torch.cuda.Stream(self.dev)
        torch.cuda.synchronize(self.dev)

    def run_pipelined(self, nsteps):
        """nsteps decode steps through the public API from pinned host
        buffers, the way a serving loop runs them: step i's inputs are copied
        host->device on one stream while step i-1's kernels run on the current
        stream, and each step's output is copied back on a third stream. The
        two buffer sets alternate; events keep a set from being overwritten
        while a step still reads it. Returns events around the whole run
        (first input copy to last output copy)."""
        sc = torch.cuda.current_stream(self.dev)
        sh, sd = self.s_h2d, self.s_d2h
        ev = lambda: torch.cuda.Event()
        h_done, c_done, d_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(sh)
        for i in range(nsteps):
            b = i & 1
            with torch.cuda.stream(sh):
                if i >= 2:
                    sh.wait_event(c_done[b])  # step i-2 no longer reads these inputs
                for n, t in self.host.items():
                    self.inp2[b][n].copy_(t, non_blocking=True)
                h_done[b].record(sh)
            sc.wait_event(h_done[b])
            if i >= 2:
                sc.wait_event(d_done[b])  # step i-2's output has been copied out
            if self.graphs is not None:
                self.graphs[b].replay()
            else:
                self.step(self.inp2[b], O=self.O2[b])
            c_done[b].record(sc)
            with torch.cuda.stream(sd):
                sd.wait_event(c_done[b])
                self.host_O2[b].copy_(self.O2[b], non_blocking=True)
                d_done[b].record(sd)
        end.record(sd)
        return start, end

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host.values())

    @property
    def d2h_bytes(self):
        return self.O.numel() * self.O.element_size()

    def attend_bytes(self):
        """Algorithmic bytes of one attention launch: the selected entry rows
        and the window rows of every query, its queries in and outputs out."""
        w = self.w
        row = csa.MIXED_ROW_BYTES if w.kv_mixed else 2 * w.c
        return w.B * (w.k * row + w.n_win * 2 * w.c) + 2 * w.B * w.H_q * w.c * 2

    def index_bytes(self):
        """Algorithmic bytes of one indexer launch: every visible index key
        once, the queries and weights, the selected indices."""
        w = self.w
        return (w.B * w.n_entries * w.c_I * 2 + w.B * w.H_I * w.c_I * 2 + w.B * w.H_I * 4 +
                w.B * w.k * 4)


# ---------------------------------------------------------------- prefill workload
class Prefill:
    def __init__(self, w: synth.Workload, device):
        self.w, self.dev = w, device
        t0 = time.time()
        s = w.specs()
        self.g = csa.geom(c=w.c, rope_dims=w.rope_dims)
        self.gI = csa.geom(c=w.c_I, rope_dims=0)
        self.t = {n: to_dev(s[n], device) for n in s}
        T = w.T
        self.pos = torch.arange(T, dtype=torch.int64, device=device)
        self.seq = torch.zeros(T, dtype=torch.int32, device=device)
        self.ne = torch.tensor([T // w.m], dtype=torch.int64, device=device)
        self.idx = torch.empty(T, w.k, dtype=torch.int32, device=device)
        self.O = torch.empty(T, w.H_q, w.c, dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize(device)
        log(f"[prefill] setup {time.time() - t0:.1f}s: T={T}")

    def time_scores(self, reps, warmup, flush):
        """Device ms of the indexer alone (csa_index_scores on the step's
        index keys), L2 flushed before each launch, outside the events."""
        t = self.t
        sc = torch.empty(self.w.T, self.KI.shape[0], device=self.dev)
        call = lambda: csa.index_scores(t["qI"], t["w"], self.KI[None], self.seq, self.pos,
                                        self.ne, self.g, out=sc)
        for _ in range(warmup):
            flush_l2(flush)
            call()
        ev = []
        for _ in range(reps):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            ev.append((a, b))
        torch.cuda.synchronize(self.dev)
        return [a.elapsed_time(b) for a, b in ev]

    def index_flops(self):
        """Algorithmic FLOPs of the prefill indexer: 2 H_I c_I per visible
        (query, entry) pair, entry s visible to token t when s < (t + 1) / m."""
        w = self.w
        t = np.arange(w.T, dtype=np.int64)
        nvis = np.minimum((t + self.g.vis_offset) // w.m, w.T // w.m)
        return int(nvis.sum()) * 2 * w.H_I * w.c_I

    def step(self, ev=None):
        t, w = self.t, self.w
        E = csa.compress(t["H"], t["W_aKV"], t["W_aZ"], t["bias"], self.g, W_bKV=t["W_bKV"],
                         W_bZ=t["W_bZ"])
        KI = csa.compress(t["H"], t["WI_aKV"], t["WI_aZ"], t["biasI"], self.gI, W_bKV=t["WI_bKV"],
                          W_bZ=t["WI_bZ"])
        win = csa.rmsnorm_rope(t["kv_win"], self.g, pos0=0, pos_step=1)
        if ev:
            ev[0].record()
        csa.index_topk(t["qI"], t["w"], KI[None], self.seq, self.pos, self.ne, w.k, self.g,
                       out=self.idx)
        if ev:
            ev[1].record()
        self.KI = KI
        csa.attend(t["q"], t["sink"], E[None], self.idx, win[None], self.seq, self.pos, self.ne,
                   self.g, out=self.O)


class HcaPrefill:
    """HCA prefill: non-overlapping m'=128 compressor, window preparation,
    dense attention over every visible entry plus the window."""

    def __init__(self, w: synth.Workload, device):
        self.w, self.dev = w, device
        t0 = time.time()
        s = w.specs()
        self.g = csa.geom(m=w.m, overlap=0, c=w.c, rope_dims=w.rope_dims)
        self.t = {n: to_dev(s[n], device) for n in s}
        T = w.T
        self.pos = torch.arange(T, dtype=torch.int64, device=device)
        self.seq = torch.zeros(T, dtype=torch.int32, device=device)
        self.ne = torch.tensor([T // w.m], dtype=torch.int64, device=device)
        self.O = torch.empty(T, w.H_q, w.c, dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize(device)
        log(f"[hca prefill] setup {time.time() - t0:.1f}s: T={T}")

    def step(self):
        t = self.t
        E = csa.compress(t["H"], t["W_KV"], t["W_Z"], t["bias"], self.g)
        win = csa.rmsnorm_rope(t["kv_win"], self.g, pos0=0, pos_step=1)
        csa.hca_attend(t["q"], t["sink"], E[None], win[None], self.seq, self.pos, self.ne, self.g,
                       out=self.O)


# ---------------------------------------------------------------- timing
def flush_l2(buf):
    buf.zero_()


def time_steps(fn, steps, warmup, device, flush, extra_events=0):
    """Per-step device time with CUDA events (L2 flushed before each step,
    outside the events). Returns (list of step ms, list of extra-event ms)."""
    for _ in range(warmup):
        flush_l2(flush)
        fn(None)
    torch.cuda.synchronize(device)
    st, sub = [], []
    for _ in range(steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(extra_events)] or None
        e0.record()
        fn(ev)
        e1.record()
        st.append((e0, e1, ev))
    torch.cuda.synchronize(device)
    ms = [a.elapsed_time(b) for a, b, _ in st]
    sub_ms = [ev[0].elapsed_time(ev[1]) for _, _, ev in st] if extra_events else []
    return ms, sub_ms


def max_over_ranks(x: float) -> float:
    """Largest value over all ranks (the slowest rank's time); identity
    without a process group. NCCL groups reduce on the current GPU, others
    (gloo) on the CPU."""
    if torch.distributed.is_initialized():
        dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return x


def whole_job_rate(units_per_rank: int, n_ranks: int, ms_max: float) -> float:
    """Units per second of the whole job: every rank processes its own
    units (weak scaling), the job takes as long as its slowest rank."""
    return n_ranks * units_per_rank / (ms_max / 1e3)


def barrier():
    if torch.distributed.is_initialized():
        torch.distributed.barrier()


# ---------------------------------------------------------------- CPU oracle leg
def oracle_decode_sample(w: synth.Workload, nq: int):
    """The FP64 oracle (as it stands) on the first nq sequences of the decode
    workload: index + top-k over all visible entries, then attention over the
    selected entries (prepared from the raw rows) and the window ring."""
    import oracle as orc
    s = w.specs()
    N, c, cI, m = w.n_entries, w.c, w.c_I, w.m
    p = w.L
    t0 = time.time()
    KI = s["KI"].rows(np.arange(nq * N)).reshape(nq, N, cI)
    qI = s["qI"].rows(np.arange(nq * w.H_I)).reshape(nq, w.H_I, cI)
    wv = s["w"].rows(np.arange(nq)).reshape(nq, w.H_I)
    q = s["q"].rows(np.arange(nq * w.H_q)).reshape(nq, w.H_q, c)
    sink = s["sink"].values()
    win_raw = s["win_raw"].rows(np.arange(nq * w.n_win)).reshape(nq, w.n_win, c)
    gen_s = time.time() - t0
    t1 = time.time()
    pos = np.full(nq, p)
    ref = orc.index_topk(qI, wv, KI, np.arange(nq), pos, np.full(nq, N), m=m, k=w.k)
    sel = ref["idx"]
    slots = np.arange(w.n_win)
    wpos = p - ((p - slots) % w.n_win)
    Osum = 0.0
    for b in range(nq):
        rows = sel[b][sel[b] >= 0]
        Eraw = s["E_raw"].rows(b * N + rows)
        Eb = np.zeros((1, N, c))
        Eb[0, rows] = orc.rmsnorm_rope(Eraw, rows * m, w.rope_dims)
        ring = orc.rmsnorm_rope(win_raw[b], wpos, w.rope_dims)[None]
        O = orc.attend(q[b:b + 1], sink, Eb, ring, [0], [p], [N], rope_dims=w.rope_dims,
                       idx=sel[b:b + 1], win_ring=1)
        Osum += float(np.abs(O).sum())
    el = time.time() - t1
    return nq / el, el, gen_s


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill secondary line")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel of a decode step from the host instead of "
                         "replaying the step as a CUDA graph")
    ap.add_argument("--cpu-queries", type=int, default=32,
                    help="queries in the CPU-oracle sample (decode workload); 0 skips it")
    ap.add_argument("--workload", default="csa_decode_bf16",
                    choices=["csa_decode_bf16", "csa_decode_long_mixed"],
                    help="decode workload of the headline line")
    ap.add_argument("--batch", type=int, default=0, help="override the decode batch size")
    ap.add_argument("--prefill-workload", default="csa_prefill_bf16",
                    choices=["csa_prefill_bf16", "hca_prefill_bf16"])
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    w = synth.WORKLOADS[args.workload]()
    if args.batch > 0:
        w = synth.WORKLOADS[args.workload](B=args.batch)
    config = {"workload": w.name, "launch": "host" if args.no_graph else "cuda_graph", "batch": w.B, "context": w.L, "entries_per_seq": w.n_entries,
              "m": w.m, "top_k": w.k, "window": w.n_win, "query_heads": w.H_q, "head_dim": w.c,
              "indexer_heads": w.H_I, "indexer_dim": w.c_I, "parallelism": f"dp{args.gpus}",
              "l2": "flushed (256 MiB write) before every timed step",
              "e2e": "pinned host inputs copied in and the output copied back every step; "
                     "steps pipelined over three streams; no flush (each step streams > L2)"}

    if args.impl == "reference":
        if rank != 0:
            return
        nq = 2
        vals = []
        for _ in range(args.warmup):
            oracle_decode_sample(w, 1)
        for _ in range(args.steps):
            qps, el, _ = oracle_decode_sample(w, nq)
            vals.append(el)
        ms = 1e3 * sum(vals) / len(vals)
        value = nq / (ms / 1e3)
        cores = min(nq, os.cpu_count() or 1)
        line = {"metric": "CSA decode queries/s", "value": value, "unit": "queries/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference",
                "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores,
                                 "kind": "oracle",
                                 "sample": f"{nq} queries of the workload per step (FP64 oracle: "
                                           "index+top-k over 32,768 entries, attention over "
                                           "1,024 selected + 128 window rows)"},
                "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    hbm, tflops, peak_kind = peaks()

    dec = Decode(w, device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    launches0 = csa.kernel_launches()
    dec.step(dec.inp)
    torch.cuda.synchronize(device)
    per_step_launches = csa.kernel_launches() - launches0
    # the indexer launch alone, for the roofline (events on the launching stream)
    _, idx_ms = time_steps(lambda ev: dec.step(dec.inp, ev), max(5, args.steps // 2), args.warmup,
                           device, flush, extra_events=2)
    # the indexer and the attention together (csa_index_topk then csa_attend,
    # events before the first and after the second), in a loop of their own
    ia_ms = None
    try:
        evs = []
        for i in range(args.warmup + max(5, args.steps // 2)):
            flush_l2(flush)
            e3 = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            dec.step(dec.inp, e3)
            if i >= args.warmup:
                evs.append(e3)
        torch.cuda.synchronize(device)
        ia_ms = statistics.mean(e3[0].elapsed_time(e3[2]) for e3 in evs)
    except Exception as ex:  # optional figure: reported as absent rather than failing the run
        log(f"[decode] indexer + attention timing unavailable: {ex}")
    if not args.no_graph:
        dec.capture()
    barrier()
    clk = Clocks(device.index).__enter__()
    step_fn = (lambda ev: dec.step(dec.inp)) if args.no_graph else dec.step_graph
    step_ms, _ = time_steps(step_fn, args.steps, args.warmup, device, flush)
    ms = statistics.mean(step_ms)
    ms_max = max_over_ranks(ms)
    value = whole_job_rate(w.B, args.gpus, ms_max)

    # end to end through the public API from pinned host memory: steps
    # pipelined over three streams (copies of one step overlap the kernels of
    # the previous one); no L2 flush between steps, each of which streams more
    # than 300 MB of cache through L2
    e2e_ms = None
    if not args.no_e2e:
        dec.setup_pipeline()
        dec.run_pipelined(args.warmup)
        torch.cuda.synchronize(device)
        a, b = dec.run_pipelined(args.steps)
        torch.cuda.synchronize(device)
        e2e_ms = max_over_ranks(a.elapsed_time(b) / args.steps)
    h2d_bytes, d2h_bytes = dec.h2d_bytes, dec.d2h_bytes

    # roofline of the dominant kernel (the indexer)
    idx_avg = statistics.mean(idx_ms)
    idx_bytes = dec.index_bytes()
    achieved = idx_bytes / (idx_avg / 1e3) / 1e9
    traffic = None
    prof = ROOT / "profiles" / "index_topk_decode_traffic.json"
    if prof.exists() and w.name == "csa_decode_bf16" and w.B == 32:
        # ncu DRAM bytes of the call, valid only while the kernels' sources are
        # the ones that were captured
        try:
            rec = json.loads(prof.read_text())
            same = all(hashlib.sha256((ROOT / f).read_bytes()).hexdigest() == digest
                       for f, digest in rec.get("sources_sha256", {}).items())
            traffic = rec.get("dram_bytes_per_launch") if same else None
        except (ValueError, OSError):
            traffic = None
    index_attention = None
    if ia_ms is not None:
        ia_ms = max_over_ranks(ia_ms)
        ia_bytes = idx_bytes + dec.attend_bytes()
        ia_ach = ia_bytes / (ia_ms / 1e3) / 1e9
        index_attention = {"bound": "hbm", "achieved": ia_ach, "peak": hbm, "unit": "GB/s",
                           "frac": ia_ach / hbm, "ms": ia_ms, "algorithmic_bytes": ia_bytes,
                           "calls": "csa_index_topk + csa_attend (decode step)"}
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic,
                "kernel": f"csa_index_topk (decode, all {w.B} queries)",
                "kernel_ms": idx_avg, "algorithmic_bytes": idx_bytes,
                "peak_source": f"{peak_kind} HBM copy bandwidth"}

    # secondary: prefill tokens/s
    prefill = None
    if not args.no_prefill:
        del dec
        torch.cuda.empty_cache()
        pw = synth.WORKLOADS[args.prefill_workload]()
        pre = (Prefill if pw.kind == "csa_prefill" else HcaPrefill)(pw, device)
        csa_pre = pw.kind == "csa_prefill"
        pms, ims = time_steps((lambda ev: pre.step(ev)) if csa_pre else (lambda ev: pre.step()),
                              max(3, args.steps // 4), 3, device, flush,
                              extra_events=2 if csa_pre else 0)
        pms_max = max_over_ranks(statistics.mean(pms))
        prefill = {"metric": ("CSA" if pw.kind == "csa_prefill" else "HCA") + " prefill tokens/s",
                   "value": args.gpus * pw.T / (pms_max / 1e3),
                   "unit": "tokens/s", "ms_per_step": pms_max,
                   "config": {"workload": pw.name, "T": pw.T, "d": pw.d, "top_k": pw.k}}
        if csa_pre:
            # tensor roofline of the indexer: the score kernel alone
            # (csa_index_scores, timed in its own loop), and the step's whole
            # csa_index_topk call (score launch + top-k launch) beside it
            sms = max_over_ranks(statistics.mean(pre.time_scores(max(5, args.steps // 2), 3, flush)))
            ims_max = max_over_ranks(statistics.mean(ims))
            fl = pre.index_flops()
            ach = fl / (sms / 1e3) / 1e12
            prefill["indexer_roofline"] = {
                "bound": "tensor", "achieved": ach, "peak": tflops, "unit": "TFLOP/s",
                "frac": ach / tflops,
                "kernel": f"csa_index_scores (prefill, {pw.T} queries)",
                "kernel_ms": sms, "algorithmic_flop": fl,
                "index_topk_call_ms": ims_max,
                "index_topk_call_frac": fl / (ims_max / 1e3) / 1e12 / tflops,
                "peak_source": f"{peak_kind} dense BF16 GEMM (burst)"}
        del pre

    clk.__exit__(None, None, None)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_queries > 0:
        nq = max(1, min(args.cpu_queries, w.B))
        qps, el, gen = oracle_decode_sample(w, nq)
        cpu = {"value": qps, "unit": "queries/s", "cores": min(nq, os.cpu_count() or 1),
               "kind": "oracle",
               "sample": f"{nq} of the 32 decode queries (index+top-k over 32,768 entries and "
                         f"attention over 1,024 selected + 128 window rows, FP64), {el:.1f}s"}

    clocks = clk.summary()
    if rank == 0:
        line = {"metric": "CSA decode queries/s", "value": value, "unit": "queries/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": None if e2e_ms is None else
                       {"value": args.gpus * w.B / (e2e_ms / 1e3), "unit": "queries/s",
                        "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes},
                "gpu_launches": per_step_launches * args.steps,
                "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
                "decode_index_attention": index_attention,
                "prefill": prefill}
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
