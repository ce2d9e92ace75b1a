#!/usr/bin/env python
"""Benchmark of one Lookahead Sparse Attention indexer trigger on B200.

One step = the whole indexer path for a batch of B sequences and the three indexer
layers: low-rank query projection, head-fused gated score + threshold (tcgen05), OR-union,
fetch-list compaction, cold-pool -> hot-pool gather of the newly fetched compressed-KV
rows over the host link (on a side stream, overlapped with the next layer's scoring),
compaction of the union and the top-k inside the fetched set.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (weak scaling, no collective on the data
path); the timed region is bracketed by a barrier and a synchronisation, and the time
is the maximum over ranks.  Rank 0 prints one JSON line.  `--impl reference` times the
fp64 CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import workloads as W  # noqa: E402

METRIC = "LSA entries scored+selected/sec at 1M ctx (B=32, 3 layers); % of roofline"
UNIT = "entry-layer scorings/s"
DEFAULT_WORKLOAD = "lsa_step_1m_b32_fp8"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "score_tc_fp8_1m_b32_traffic.txt")
# the score kernel's source: the kernel file and the tcgen05 / TMA wrappers it includes
SCORE_SRC = [os.path.join(ROOT, "lookahead_sparse_kv_score_b200", "csrc", f) for f in ("score_tc.cu", "tc_ptx.cuh")]
PROFILE_GATHER = os.path.join(ROOT, "profiles", "gather_cold_1m_host_link.txt")
GATHER_SRC = [os.path.join(ROOT, "lookahead_sparse_kv_score_b200", "csrc", "gather.cu")]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's B); smaller batches are for profiling")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-vote", action="store_true", help="skip the vote-label measurement")
    ap.add_argument("--no-hot-pool", action="store_true", help="skip the residency measurement")
    ap.add_argument("--select-only", action="store_true",
                    help="profiling mode: time only the main-stream part of the step (projection, scoring, "
                         "selection, top-k) without the cold pool, the gathers or the secondary measurements")
    ap.add_argument("--schedule", choices=["batched", "per_layer"], default="batched",
                    help="fetch schedule of the timed step (batched: all layers scored in one launch, then the "
                         "selection, then the gathers; per_layer: each layer's gather runs beside the next "
                         "layer's scoring; both are timed side by side in gather_overlap)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- ranks

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_pg(world: int, local: int, backend: str):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local) if backend == "nccl" else None)
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job(units_local: int, ms_local: float, dist, device):
    """(total units over ranks, max device time over ranks in ms, whole-job units/s)."""
    if dist is None:
        return units_local, ms_local, units_local / (ms_local * 1e-3)
    t = torch.tensor([float(units_local)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    ms = max_over_ranks(ms_local, dist, device)
    units = int(t.item())
    return units, ms, units / (ms * 1e-3)


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)


# ----------------------------------------------------------------------------- inputs

def device_inputs(w: W.ScoreWorkload, device):
    """All inputs of the scoring step, generated on the device from the seeded streams."""
    bias, direction = W.load_params(w.name)
    h = W.hidden_states(w, device).transpose(0, 1).contiguous()           # [L][B][D]
    Wd, Wu, Ww = W.all_layer_weights(w, device)
    kdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[w.kdtype]
    K = torch.empty(w.L, w.B, w.N, w.dI, dtype=kdt, device=device)
    ks = torch.empty(w.L, w.B, w.N, dtype=torch.float32, device=device) if w.kdtype == "e4m3" else None
    for l in range(w.L):
        for b in range(w.B):
            k, s = W.keys(w, b, l, direction[b, l].double(), 0, w.N, device)
            K[l, b] = k
            if ks is not None:
                ks[l, b] = s
    return dict(h=h, Wd=Wd, Wu=Wu, Ww=Ww, bias=bias.to(device), K=K, kscale=ks)


def cold_pool(w: W.ScoreWorkload, device, chunk_rows=1 << 15):
    """Pinned, device-mapped host memory [B][N][row_bytes] filled with the seeded rows."""
    cold = torch.empty(w.B, w.N, w.row_bytes, dtype=torch.uint8, pin_memory=True)
    for b in range(w.B):
        for s0 in range(0, w.N, chunk_rows):
            n = min(chunk_rows, w.N - s0)
            cold[b, s0:s0 + n].copy_(W.cold_rows(w, b, s0, n, device), non_blocking=False)
    return cold


# ----------------------------------------------------------------------------- the step

class Trigger:
    """Buffers and streams of one indexer trigger; run() enqueues one step."""

    def __init__(self, lsa, w: W.ScoreWorkload, inp, cold, device):
        self.lsa, self.w, self.inp, self.cold, self.dev = lsa, w, inp, cold, device
        B, L, N = w.B, w.L, w.N
        self.Nw = (N + 31) // 32
        self.cap = N
        self.wdt = lsa.dtype_code(inp["h"])
        self.kdt = lsa.dtype_code(inp["K"])
        self.q = torch.empty(L, B, w.H, w.dI, dtype=inp["h"].dtype, device=device)
        self.wv = torch.empty(L, B, w.H, dtype=torch.float32, device=device)
        self.mask = torch.empty(L, B, self.Nw, dtype=torch.int32, device=device)
        self.logit = torch.empty(L, B, N, dtype=torch.float32, device=device)
        self.U = torch.zeros(B, self.Nw, dtype=torch.int32, device=device)
        self.new = torch.empty(L, B, self.Nw, dtype=torch.int32, device=device)
        self.idx_new = torch.empty(L, B, self.cap, dtype=torch.int32, device=device)
        self.cnt_new = torch.zeros(L, B, dtype=torch.int32, device=device)
        # the hot pool (one region per layer's new rows); not needed without a cold pool
        self.hot = (torch.empty(L, B, self.cap, w.row_bytes, dtype=torch.uint8, device=device)
                    if cold is not None else None)
        self.idx_U = torch.empty(B, N, dtype=torch.int32, device=device)
        self.cnt_U = torch.zeros(B, dtype=torch.int32, device=device)
        self.key_U = torch.empty(B, N, dtype=torch.int32, device=device)   # the union's top-k keys (uint32 bits)
        self.topk = torch.empty(B, w.k, dtype=torch.int32, device=device)
        self.topk_cnt = torch.zeros(B, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws_proj = lsa.workspace(lsa.lsa_index_project_workspace_bytes(B, L, w.D, w.r, w.H, w.dI, self.wdt),
                                     device)
        self.ws_score = lsa.workspace(lsa.lsa_index_score_workspace_bytes(B, L, N, w.D, w.r, w.H, w.dI,
                                                                          self.wdt, self.kdt), device)
        self.ws_topk = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, N), device)
        self.ws_sel = lsa.workspace(lsa.lsa_select_fetch_workspace_bytes(B, N), device)
        # The main stream runs at a higher priority than the side stream: where the two
        # overlap (the residency measurement), the SMs a retiring gather block frees go to
        # the selection first.
        self.main = torch.cuda.Stream(device, priority=-1)
        self.side = torch.cuda.Stream(device, priority=0)
        self.timing = []     # per recorded step: the events of its score, gather and main-stream spans
        self.schedule = "batched"

    def run(self, record=False, schedule=None):
        """One trigger on the chosen fetch schedule (self.schedule unless given)."""
        if (schedule or self.schedule) == "per_layer":
            return self.run_per_layer(record)
        return self.run_batched(record)

    def _events(self, record):
        L = self.w.L
        mk = lambda: torch.cuda.Event(enable_timing=record)
        return {"score": [(mk(), mk()) for _ in range(L)], "gather": [(mk(), mk()) for _ in range(L)],
                "select": (mk(), mk())}

    def run_batched(self, record=False):
        """One trigger, all layers scored in one launch (HBM-bound, ~0.55 ms), then one
        call forms the union, the per-layer new sets, all fetch lists and the union's top-k
        keys, and the top-k runs on those keys (it ranks by the indexer logits, so it does
        not wait for the rows); then the side stream gathers the new rows of each layer
        over the host link (tens of ms)."""
        lsa, w, inp = self.lsa, self.w, self.inp
        B, L, N = w.B, w.L, w.N
        m, sd = self.main, self.side
        e = self._events(record)
        if record:
            e["select"][0].record(m)
        lsa.lsa_index_project(B, L, w.D, w.r, w.H, w.dI, self.wdt, inp["h"], inp["Wd"], inp["Wu"], inp["Ww"], -1,
                              self.q, self.wv, self.ws_proj, stream=m)
        if record:
            e["score"][0][0].record(m)
        lsa.lsa_index_score(B, L, N, w.D, w.r, w.H, w.dI, self.wdt, None, None, None, None, inp["bias"],
                            self.kdt, inp["K"], inp["kscale"], -1, self.q, self.wv, None, None,
                            self.mask, self.logit, None, self.ws_score, status=self.status, stream=m)
        if record:
            e["score"][0][1].record(m)
            for l in range(1, L):       # one launch covers every layer
                e["score"][l][0].record(m)
                e["score"][l][1].record(m)
        lsa.lsa_select_fetch(B, L, N, self.mask, self.U, self.new, self.cap, self.idx_new, self.cnt_new,
                             self.idx_U, self.cnt_U, self.ws_sel, logit=self.logit, key_U=self.key_U,
                             status=self.status, stream=m)
        lsa.lsa_topk_keyed(B, w.k, self.idx_U, N, self.cnt_U, self.key_U, self.topk, self.topk_cnt, stream=m)
        if record:
            e["select"][1].record(m)
        selected = torch.cuda.Event()
        selected.record(m)
        sd.wait_event(selected)
        for l in range(L):
            if record:
                e["gather"][l][0].record(sd)
            lsa.lsa_gather_cold(B, N, w.row_bytes, self.cold, self.idx_new[l], self.cnt_new[l], self.cap,
                                self.hot[l], self.status, stream=sd)
            if record:
                e["gather"][l][1].record(sd)
        done = torch.cuda.Event()
        done.record(sd)
        m.wait_event(done)
        if record:
            self.timing.append(e)

    def select_only(self):
        """The main stream's part of a trigger alone (projection, scoring, union, fetch
        lists, top-k), without the gathers."""
        lsa, w, inp = self.lsa, self.w, self.inp
        B, L, N = w.B, w.L, w.N
        m = self.main
        lsa.lsa_index_project(B, L, w.D, w.r, w.H, w.dI, self.wdt, inp["h"], inp["Wd"], inp["Wu"], inp["Ww"], -1,
                              self.q, self.wv, self.ws_proj, stream=m)
        lsa.lsa_index_score(B, L, N, w.D, w.r, w.H, w.dI, self.wdt, None, None, None, None, inp["bias"],
                            self.kdt, inp["K"], inp["kscale"], -1, self.q, self.wv, None, None,
                            self.mask, self.logit, None, self.ws_score, status=self.status, stream=m)
        lsa.lsa_select_fetch(B, L, N, self.mask, self.U, self.new, self.cap, self.idx_new, self.cnt_new,
                             self.idx_U, self.cnt_U, self.ws_sel, logit=self.logit, key_U=self.key_U,
                             status=self.status, stream=m)
        lsa.lsa_topk_keyed(B, w.k, self.idx_U, N, self.cnt_U, self.key_U, self.topk, self.topk_cnt, stream=m)
        torch.cuda.current_stream().wait_stream(m)

    def run_per_layer(self, record=False):
        """One trigger on the schedule the pages describe (the fetch asynchronous and
        overlapped with compute): layer l is scored alone, its new rows are unioned and
        compacted, and their gather starts on the side stream while layer l + 1 is
        scored; the union's fetch list and the top-k follow the last layer."""
        lsa, w, inp = self.lsa, self.w, self.inp
        B, L, N = w.B, w.L, w.N
        m, sd = self.main, self.side
        e = self._events(record)
        if record:
            e["select"][0].record(m)
        lsa.lsa_index_project(B, L, w.D, w.r, w.H, w.dI, self.wdt, inp["h"], inp["Wd"], inp["Wu"], inp["Ww"], -1,
                              self.q, self.wv, self.ws_proj, stream=m)
        with torch.cuda.stream(m):
            self.U.zero_()
        for l in range(L):
            if record:
                e["score"][l][0].record(m)
            lsa.lsa_index_score(B, L, N, w.D, w.r, w.H, w.dI, self.wdt, None, None, None, None, inp["bias"],
                                self.kdt, inp["K"], inp["kscale"], l, self.q, self.wv, None, None,
                                self.mask, self.logit, None, self.ws_score, status=self.status, stream=m)
            if record:
                e["score"][l][1].record(m)
            lsa.lsa_select_union(B, self.Nw, self.mask[l], self.U, self.new[l], stream=m)
            lsa.lsa_compact(B, N, self.new[l], self.cap, self.idx_new[l], self.cnt_new[l], self.status, stream=m)
            ready = torch.cuda.Event()
            ready.record(m)
            sd.wait_event(ready)
            if record:
                e["gather"][l][0].record(sd)
            lsa.lsa_gather_cold(B, N, w.row_bytes, self.cold, self.idx_new[l], self.cnt_new[l], self.cap,
                                self.hot[l], self.status, stream=sd)
            if record:
                e["gather"][l][1].record(sd)
        lsa.lsa_compact(B, N, self.U, N, self.idx_U, self.cnt_U, self.status, stream=m)
        lsa.lsa_topk(B, L, N, w.k, self.idx_U, N, self.cnt_U, self.logit, self.topk, self.topk_cnt, self.ws_topk,
                     stream=m)
        if record:
            e["select"][1].record(m)
        done = torch.cuda.Event()
        done.record(sd)
        m.wait_event(done)
        if record:
            self.timing.append(e)

    def kernel_times_ms(self):
        """Per step, in ms: the score launches (summed); the gather launches (summed); the
        main stream from the projection through the top-k."""
        score = [sum(a.elapsed_time(b) for a, b in e["score"]) for e in self.timing]
        gather = [sum(a.elapsed_time(b) for a, b in e["gather"]) for e in self.timing]
        select = [e["select"][0].elapsed_time(e["select"][1]) for e in self.timing]
        return score, gather, select


# ----------------------------------------------------------------------------- measurements

def host_link_gbs(device, nbytes=1 << 30, reps=5) -> float:
    """Pinned host -> device copy bandwidth (the host link's measured peak here)."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    best = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del src, dst
    return best


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = tempfile.mktemp(suffix=".csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def source_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def score_source_sha() -> str:
    return source_sha(SCORE_SRC)


def profile_fields(path, files):
    """The key: value lines of a committed ncu summary, or None when it is missing or was
    taken on another version of the kernel source (its source_sha256 field)."""
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    return kv if kv.get("source_sha256") == source_sha(files) else None


def traffic_per_launch():
    """DRAM bytes per score launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    kv = profile_fields(PROFILE_TRAFFIC, SCORE_SRC)
    try:
        return int(kv["dram_bytes_read_per_launch"]) + int(kv["dram_bytes_write_per_launch"])
    except (KeyError, ValueError, TypeError):
        return None


def gather_link_traffic(payload_bytes):
    """Host-link bytes a gather of payload_bytes moves, from the committed ncu summary's
    ratio of PCIe read bytes to payload bytes (None if missing or on other source)."""
    kv = profile_fields(PROFILE_GATHER, GATHER_SRC)
    try:
        return int(round(float(kv["pcie_read_bytes_per_payload_byte"]) * payload_bytes))
    except (KeyError, ValueError, TypeError):
        return None


# ----------------------------------------------------------------------------- oracle

def oracle_sample_step(w: W.ScoreWorkload, raw_inputs, seqs):
    """The oracle's indexer step on sequences `seqs` (all layers, all entries)."""
    from oracle import lsa_oracle as O
    from oracle import step as OS
    units = 0
    for b in seqs:
        zs, marks = [], []
        for l in range(w.L):
            h, Wd, Wu, Ww, K, ks, bias = raw_inputs(l, b)
            q, wv = OS.project(h, Wd, Wu, Ww, w.H, w.dI, w.wdtype)
            z, _, mark = OS.score_layer(q, wv, bias, K, ks, w.kdtype)
            zs.append(z)
            marks.append(mark)
            units += len(z)
        OS.select(marks, zs, w.k)
    return units


def raw_from_device(inp, w, seqs, n_entries):
    """Host copies (storage bytes) of the inputs of the sampled sequences."""
    def raw(t):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()
    cache = {}
    Wd = [raw(inp["Wd"][l]) for l in range(w.L)]
    Wu = [raw(inp["Wu"][l]) for l in range(w.L)]
    Ww = [raw(inp["Ww"][l]) for l in range(w.L)]
    bias = raw(inp["bias"])
    for l in range(w.L):
        for b in seqs:
            ks = raw(inp["kscale"][l, b, :n_entries]) if inp["kscale"] is not None else None
            cache[l, b] = (raw(inp["h"][l, b]), Wd[l], Wu[l], Ww[l], raw(inp["K"][l, b, :n_entries]), ks,
                           float(bias[l]))
    return lambda l, b: cache[l, b]


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp, w, seqs=(0, 1)):
    raw_inputs = raw_from_device(inp, w, seqs, w.N)
    t0 = time.perf_counter()
    units = oracle_sample_step(w, raw_inputs, seqs)
    dt = time.perf_counter() - t0
    return {"value": units / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"sequences {list(seqs)} of {w.B}, all {w.L} layers, all {w.N} entries "
                      f"({units} entry-layer scorings, then union, compaction and top-k) in {dt:.1f} s"}


# ----------------------------------------------------------------------------- arms

def reference_arm(args):
    rank, world, _ = dist_setup()
    if rank != 0:
        return 0
    w = W.WORKLOADS[args.workload]
    n_entries = min(w.N, 1 << 17)
    seqs = (0,)
    wsample = W.scaled(w, B=1, N=n_entries)
    bias, direction = W.load_params(w.name)
    h = W.hidden_states(wsample).transpose(0, 1).contiguous()
    Wd, Wu, Ww = W.all_layer_weights(w)
    kdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[w.kdtype]
    K = torch.empty(w.L, 1, n_entries, w.dI, dtype=kdt)
    ks = torch.empty(w.L, 1, n_entries, dtype=torch.float32) if w.kdtype == "e4m3" else None
    for l in range(w.L):
        k, s = W.keys(w, 0, l, direction[0, l].double(), 0, n_entries)
        K[l, 0] = k
        if ks is not None:
            ks[l, 0] = s
    inp = dict(h=h, Wd=Wd, Wu=Wu, Ww=Ww, bias=bias, K=K, kscale=ks)
    raw_inputs = raw_from_device(inp, wsample, seqs, n_entries)
    for _ in range(args.warmup):
        oracle_sample_step(wsample, raw_inputs, seqs)
    t0 = time.perf_counter()
    units = 0
    for _ in range(args.steps):
        units += oracle_sample_step(wsample, raw_inputs, seqs)
    dt = time.perf_counter() - t0
    value = units / dt
    sample = (f"sequence 0 of {w.B}, all {w.L} layers, first {n_entries} of {w.N} entries per step "
              f"({units // max(args.steps, 1)} entry-layer scorings, then union, compaction and top-k)")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "layers": w.L, "N": w.N, "H_I": w.H, "d_I": w.dI,
                       "top_k": w.k, "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def hot_pool_measure(lsa, trig, device, triggers=8, rho=0.9):
    """Residency across triggers on the benchmark workload: `triggers` consecutive
    triggers whose hidden states drift (h_t = rho h_{t-1} + sqrt(1 - rho^2) eps_t).  Each
    trigger projects, scores all layers, unions them, compacts the union and ranks it on
    the main stream, while lsa_hot_pool_update on the side stream moves only the rows of
    the union not yet resident.  The first trigger fills an empty pool; the figures
    are the mean over the later ones (device time, CUDA events around each trigger)."""
    w, inp = trig.w, trig.inp
    B, L, N = w.B, w.L, w.N
    slots = N               # a sequence's union can reach most of N here; no update may fail
    hs = [W.drifted_hidden_states(w, t, rho, device).transpose(0, 1).contiguous() for t in range(1, triggers + 1)]
    hot = torch.empty(B, slots, w.row_bytes, dtype=torch.uint8, device=device)
    state = lsa.workspace(lsa.lsa_hot_pool_state_bytes(B, N, slots), device)
    ws = lsa.workspace(lsa.lsa_hot_pool_workspace_bytes(B, N, slots), device)
    moved = torch.zeros(B, dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    m, sd = trig.main, trig.side
    lsa.lsa_hot_pool_reset(B, N, slots, state, stream=m)
    torch.cuda.synchronize()
    ms, moved_rows, fetch_rows = [], [], []
    for t, h in enumerate(hs, start=1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(m)
        lsa.lsa_index_project(B, L, w.D, w.r, w.H, w.dI, trig.wdt, h, inp["Wd"], inp["Wu"], inp["Ww"], -1,
                              trig.q, trig.wv, trig.ws_proj, stream=m)
        lsa.lsa_index_score(B, L, N, w.D, w.r, w.H, w.dI, trig.wdt, None, None, None, None, inp["bias"],
                            trig.kdt, inp["K"], inp["kscale"], -1, trig.q, trig.wv, None, None,
                            trig.mask, trig.logit, None, trig.ws_score, status=status, stream=m)
        lsa.lsa_select_fetch(B, L, N, trig.mask, trig.U, None, trig.cap, trig.idx_new, trig.cnt_new,
                             trig.idx_U, trig.cnt_U, trig.ws_sel, logit=trig.logit, key_U=trig.key_U,
                             status=status, stream=m)
        ready = torch.cuda.Event()
        ready.record(m)
        sd.wait_event(ready)
        lsa.lsa_hot_pool_update(B, N, slots, w.row_bytes, t, trig.U, trig.cold, hot, state, moved, status, ws,
                                stream=sd)
        lsa.lsa_topk_keyed(B, w.k, trig.idx_U, N, trig.cnt_U, trig.key_U, trig.topk, trig.topk_cnt, stream=m)
        done = torch.cuda.Event()
        done.record(sd)
        m.wait_event(done)
        e1.record(m)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
        moved_rows.append(int(moved.sum().item()))
        fetch_rows.append(int(trig.cnt_U.sum().item()))
    st = int(status.item())
    later = slice(1, None)
    mean = lambda xs: statistics.mean(xs[later])
    return {"workload": f"{w.name}, {triggers} triggers, hidden-state drift rho={rho} between triggers",
            "slots_per_sequence": slots, "status": st,
            "value": B * L * N / (mean(ms) * 1e-3), "unit": UNIT, "ms_per_trigger": mean(ms),
            "first_trigger_ms": ms[0], "fetch_rows_per_trigger": mean(fetch_rows),
            "moved_rows_per_trigger": mean(moved_rows), "first_trigger_moved_rows": moved_rows[0],
            "host_link_bytes_per_trigger": mean(moved_rows) * w.row_bytes}


def fine_measure(lsa, trig, device, steps=5):
    """The native indexer's fine selection inside the fetched subset (lsa_fine_score over
    each sequence's union fetch list, then lsa_topk with one layer of those scores) after
    a trigger: per-token query and head weights from their own streams, layer 0's keys
    standing in for the indexer's own.  Roofline: per candidate the key row and its scale,
    its list index and its score write (dI + 12 bytes) against the measured HBM peak."""
    w = trig.w
    B, N = w.B, w.N
    qf, wf = W.fine_query(w, device)
    K0 = trig.inp["K"][0]
    ks0 = trig.inp["kscale"][0] if trig.inp["kscale"] is not None else None
    kdt = trig.kdt
    score = torch.empty(B, N, dtype=torch.float32, device=device)
    topk = torch.empty(B, w.k, dtype=torch.int32, device=device)
    tcnt = torch.empty(B, dtype=torch.int32, device=device)
    ws = lsa.workspace(lsa.lsa_fine_score_workspace_bytes(B, w.H, w.dI, kdt), device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    m = trig.main

    def one():
        lsa.lsa_fine_score(B, N, w.H, w.dI, lsa.LSA_BF16, qf, wf, kdt, K0, ks0, trig.idx_U, trig.cap, trig.cnt_U,
                           score, ws, status=st, stream=m)
        lsa.lsa_topk(B, 1, N, w.k, trig.idx_U, trig.cap, trig.cnt_U, score, topk, tcnt, trig.ws_topk, stream=m)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    score_ms = 0.0
    total_ms = 0.0
    for _ in range(steps):
        e[0].record(m)
        lsa.lsa_fine_score(B, N, w.H, w.dI, lsa.LSA_BF16, qf, wf, kdt, K0, ks0, trig.idx_U, trig.cap, trig.cnt_U,
                           score, ws, status=st, stream=m)
        e[1].record(m)
        lsa.lsa_topk(B, 1, N, w.k, trig.idx_U, trig.cap, trig.cnt_U, score, topk, tcnt, trig.ws_topk, stream=m)
        e[2].record(m)
        torch.cuda.synchronize()
        score_ms += e[0].elapsed_time(e[1])
        total_ms += e[0].elapsed_time(e[2])
    score_ms /= steps
    total_ms /= steps
    cands = int(trig.cnt_U.clamp(max=trig.cap).sum().item())
    per = w.dI * K0.element_size() + (4 if ks0 is not None else 0) + 8
    hbm_peak, peak_kind = measured_peaks()
    achieved = cands * per / (score_ms * 1e-3) / 1e9
    return {"workload": f"{w.name}: native-indexer fine top-{w.k} inside each sequence's union fetch list",
            "candidates_per_step": cands, "status": int(st.item()), "score_ms": score_ms, "fine_topk_ms": total_ms,
            "value": cands / (total_ms * 1e-3), "unit": "fetched entries scored+ranked/s",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "bytes_per_candidate": per, "kernel": "score_tc (gathered)",
                         "peak_kind": peak_kind}}


def vote_measure(lsa, device, steps=5):
    """Cross-layer vote labels + loss on the L=24 x P=64 x N=131072 workload: logits from the
    generator, loss scores from the 512K workload's scorer (sequence 0, layer 0), one query
    per position.  Returns the secondary bench object (device time of the lsa_vote_labels
    call, HBM roofline on the 4 bytes per logit it must read)."""
    v = W.VOTE_WORKLOADS["vote_labels_l24_p64_n131072"]
    w2 = W.scaled(W.WORKLOADS["lsa_step_512k_b8_bf16"], B=1, L=1)
    logits = torch.empty(v.L, v.P, v.N, dtype=torch.float32, device=device)
    for p in range(v.P):
        bs = W.vote_boost_set(v, p, device)
        for l in range(v.L):
            logits[l, p] = W.vote_logits(v, l, p, device, boost_set=bs)
    bias, direction = W.load_params(w2.name)
    Wd, Wu, Ww = (t[:1].contiguous() for t in W.all_layer_weights(W.WORKLOADS["lsa_step_512k_b8_bf16"], device))
    K = W.keys(w2, 0, 0, direction[0, 0].double(), 0, w2.N, device)[0].reshape(1, 1, w2.N, w2.dI).contiguous()
    hp = W.position_hidden(v, w2, device)
    scores = torch.empty(v.P, v.N, dtype=torch.float32, device=device)
    Nw2 = (w2.N + 31) // 32
    mask = torch.empty(1, 1, Nw2, dtype=torch.int32, device=device)
    ws = lsa.workspace(lsa.lsa_index_score_workspace_bytes(1, 1, w2.N, w2.D, w2.r, w2.H, w2.dI, 1, 1), device)
    b1 = bias[:1].to(device)
    for p in range(v.P):
        lsa.lsa_index_score(1, 1, w2.N, w2.D, w2.r, w2.H, w2.dI, 1, hp[p:p + 1].reshape(1, 1, w2.D), Wd, Wu, Ww, b1,
                            1, K, None, -1, None, None, None, None, mask, None, scores[p:p + 1], ws)
    Nw = (v.N + 31) // 32
    golden = torch.empty(v.P, Nw, dtype=torch.int32, device=device)
    loss = torch.zeros(2, dtype=torch.float64, device=device)
    vws = lsa.workspace(lsa.lsa_vote_labels_workspace_bytes(v.L, v.P, v.N), device)
    run = lambda: lsa.lsa_vote_labels(v.L, v.P, v.N, logits, v.top_p, v.theta, golden, None, scores, v.gamma,
                                      loss, vws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    nbytes = logits.numel() * 4
    hbm_peak, _ = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    out = {"workload": v.name, "ms": ms, "logits_per_s": logits.numel() / (ms * 1e-3),
           "loss": [float(x) for x in loss.cpu()],
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                        "frac": achieved / hbm_peak, "bytes_per_launch": nbytes}}
    out["train_step"] = train_measure(lsa, device, hp, Wd, Wu, Ww, K, float(b1[0].item()), golden, v.gamma,
                                      [float(x) for x in loss.cpu()], steps)
    del logits, K, scores
    return out


def train_measure(lsa, device, hp, Wd, Wu, Ww, K, bias, golden, gamma, vote_loss, steps=5):
    """One indexer training step (lsa_index_train_step) on the vote workload's P = 64
    positions against sequence 0's N = 131,072 layer-0 keys of the 512K workload, with
    the vote's golden bits as labels: projection, fused forward + backward on the tensor
    cores, projection gradients.  The loss it reports must equal the vote call's loss
    (same scorer, same labels).  Roofline: the forward and backward key products,
    4 P H dI N flops, against the measured dense bf16 peak."""
    P, D = hp.shape
    r, HD = Wu.shape[1], Wu.shape[2]
    H = Ww.shape[2]
    dI = HD // H
    N = K.shape[2]
    loss = torch.zeros(2, dtype=torch.float64, device=device)
    dbias = torch.zeros(1, dtype=torch.float64, device=device)
    dWd = torch.empty(D, r, device=device)
    dWu = torch.empty(r, HD, device=device)
    dWw = torch.empty(D, H, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    ws = lsa.workspace(lsa.lsa_index_train_step_workspace_bytes(P, N, D, r, H, dI), device)
    Kf = K.reshape(N, dI)
    run = lambda: lsa.lsa_index_train_step(P, N, D, r, H, dI, 1, hp, Wd[0], Wu[0], Ww[0], bias, 1, Kf, None, golden,
                                           gamma, None, None, None, loss, dWd, dWu, dWw, dbias, ws, status=st)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    flops = 4.0 * P * H * dI * N
    peak = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))).get("bf16_tflops") \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 1590.0
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": f"train_step_l0_p{P}_n{N} (H={H}, dI={dI}, D={D}, r={r}, vote labels)", "ms": ms,
            "status": int(st.item()), "loss": [float(x) for x in loss.cpu()], "vote_loss": vote_loss,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "flops_per_step": flops,
                         "peak_kind": "measured dense bf16 (burst)"}}


def our_arm(args):
    import lookahead_sparse_kv_score_b200 as lsa
    rank, world, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_pg(world, local, "nccl")
    lsa.lib()
    w = W.WORKLOADS[args.workload]
    if args.batch is not None:
        w = W.scaled(w, B=args.batch)
    args.e2e_steps = max(1, args.e2e_steps)

    inp = device_inputs(w, device)
    cold = cold_pool(w, device)
    trig = Trigger(lsa, w, inp, cold, device)
    trig.schedule = args.schedule
    torch.cuda.synchronize()

    for _ in range(max(args.warmup, 0)):
        trig.run()
    torch.cuda.synchronize()
    trig.status.zero_()
    launches0 = lsa.kernel_launches()
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(dist, device)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(trig.main)
    for _ in range(args.steps):
        trig.run(record=True)
    t_end.record(trig.main)
    torch.cuda.synchronize()
    barrier(dist, device)
    clk = clocks.stop()
    launches = lsa.kernel_launches() - launches0
    ms_local = t_start.elapsed_time(t_end)
    status = int(trig.status.item())
    if status != 0:
        raise SystemExit(f"device status {status} ({lsa.status_string(status)}) during the timed region")

    units, ms, value = whole_job(w.B * w.L * w.N * args.steps, ms_local, dist, device)
    score_ms, gather_ms, select_ms = trig.kernel_times_ms()
    _, sel_ms, sel_value = whole_job(w.B * w.L * w.N * args.steps, sum(select_ms), dist, device)
    score_avg = statistics.mean(score_ms)
    gather_avg = statistics.mean(gather_ms)
    fetched_rows = int(trig.cnt_new.sum().item())          # rows moved by the last step
    # algorithmic bytes of one scoring launch (all layers): the keys and their scales
    key_bytes = w.L * w.B * w.N * (w.dI * trig.inp["K"].element_size() + (4 if w.kdtype == "e4m3" else 0))
    hbm_peak, peak_kind = measured_peaks()
    achieved = key_bytes / (score_avg * 1e-3) / 1e9
    link = host_link_gbs(device)
    gather_gbs = fetched_rows * w.row_bytes / (gather_ms[-1] * 1e-3) / 1e9

    # the two fetch schedules side by side (device time per trigger, same run)
    def time_schedule(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(trig.main)
        for _ in range(reps):
            fn()
        b.record(trig.main)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps
    overlap = {"batched_ms": time_schedule(trig.run_batched), "per_layer_ms": time_schedule(trig.run_per_layer),
               "timed": args.schedule,
               "batched": "all layers scored in one launch, the fused selection and the top-k, then the gathers "
                          "on the side stream",
               "per_layer": "layer l scored alone, its new rows unioned, compacted and gathered on the side stream "
                            "while layer l+1 is scored; the union's list and the top-k after the last layer"}
    if int(trig.status.item()) != 0:
        raise SystemExit(f"device status {int(trig.status.item())} in the schedule comparison")
    fine = fine_measure(lsa, trig, device) if rank == 0 else None

    # end to end: inputs from pinned host memory every step, result read back
    h_host = inp["h"].cpu().pin_memory()
    K_host = inp["K"].cpu().pin_memory()
    ks_host = inp["kscale"].cpu().pin_memory() if inp["kscale"] is not None else None
    topk_host = torch.empty_like(trig.topk, device="cpu").pin_memory()
    cnt_host = torch.empty_like(trig.topk_cnt, device="cpu").pin_memory()
    h2d = h_host.numel() * h_host.element_size() + K_host.numel() * K_host.element_size() + \
        (ks_host.numel() * 4 if ks_host is not None else 0)
    d2h = topk_host.numel() * 4 + cnt_host.numel() * 4

    def e2e_step():
        with torch.cuda.stream(trig.main):
            inp["h"].copy_(h_host, non_blocking=True)
            inp["K"].copy_(K_host, non_blocking=True)
            if ks_host is not None:
                inp["kscale"].copy_(ks_host, non_blocking=True)
        trig.run()
        with torch.cuda.stream(trig.main):
            topk_host.copy_(trig.topk, non_blocking=True)
            cnt_host.copy_(trig.topk_cnt, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(trig.main)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(trig.main)
    torch.cuda.synchronize()
    _, e2e_ms, e2e_value = whole_job(w.B * w.L * w.N * args.e2e_steps, e0.elapsed_time(e1), dist, device)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(inp, w)
    hot_pool = None
    if rank == 0 and not args.no_hot_pool:
        hot_pool = hot_pool_measure(lsa, trig, device)
    vote = None
    if rank == 0 and not args.no_vote:
        del trig, cold
        torch.cuda.empty_cache()
        vote = vote_measure(lsa, device)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.kdtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "layers": w.L, "N": w.N, "D": w.D, "r": w.r, "H_I": w.H,
                       "d_I": w.dI, "top_k": w.k, "row_bytes": w.row_bytes,
                       "l2": "inputs larger than L2 (keys %.2f GB)" % (key_bytes / 1e9),
                       "parallelism": f"replica per GPU x{world}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": traffic_per_launch(),
                         "kernel": ("score_tc (lsa_index_score, one launch per layer; achieved = all layers' "
                                    "bytes over the sum of the three launch times)" if args.schedule == "per_layer"
                                    else "score_tc (lsa_index_score, all layers in one launch)"),
                         "note": "the scoring launch, the kernel the metric's roofline is about; the step's "
                                 "longest kernel is the host-link gather, reported in roofline_gather",
                         "bytes_per_launch": key_bytes, "launch_ms": score_avg, "peak_kind": peak_kind},
            "cpu_baseline": base,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.e2e_steps},
            "clocks": clk,
            "gpu_launches": launches,
            "roofline_gather": {"bound": "host_link", "achieved": gather_gbs, "peak": link, "unit": "GB/s",
                                "frac": gather_gbs / link,
                                "traffic": gather_link_traffic(fetched_rows * w.row_bytes),
                                "traffic_kind": "PCIe read bytes per step (ncu ratio to payload bytes)",
                                "kernel": "gather_cold (zero-copy reads of pinned host rows)",
                                "bytes_per_step": fetched_rows * w.row_bytes, "rows_per_step": fetched_rows,
                                "ms_per_step": gather_avg,
                                "peak_kind": "measured here: pinned host->device cudaMemcpy, 1 GiB"},
            "select_path": {"value": sel_value, "unit": UNIT, "ms_per_step": sel_ms / args.steps,
                            "covers": "projection, scoring, union, compaction and top-k on the main stream of "
                                      "each timed step (per_layer: the layers' gathers run beside the later "
                                      "layers' scoring on the side stream; batched: they follow the top-k)"},
            "gather_overlap": overlap,
            "fine_select": fine,
            "hot_pool": hot_pool,
            "vote_labels": vote,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def select_only_arm(args):
    """Profiling mode: the main-stream part of the step on the benchmark workload (no cold
    pool, no gathers), K timed steps; prints a reduced JSON line.  Not the benchmark."""
    import lookahead_sparse_kv_score_b200 as lsa
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    lsa.lib()
    w = W.WORKLOADS[args.workload]
    if args.batch is not None:
        w = W.scaled(w, B=args.batch)
    inp = device_inputs(w, device)
    trig = Trigger(lsa, w, inp, None, device)
    for _ in range(max(args.warmup, 0)):
        trig.select_only()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(trig.main)
    for _ in range(args.steps):
        trig.select_only()
    b.record(trig.main)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / max(args.steps, 1)
    print(json.dumps({"mode": "select_only", "workload": w.name, "B": w.B, "steps": args.steps,
                      "ms_per_step": ms, "status": int(trig.status.item())}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_arm(args)
    if args.select_only:
        return select_only_arm(args)
    return our_arm(args)


if __name__ == "__main__":
    sys.exit(main())
