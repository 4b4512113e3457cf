"""Batch-256 SSM-layer decode throughput of the ReplaySSM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--layer mamba2|gdn]
                    [--impl rssm|reference]

One *step* is one full window of the layer: L = 16 decode calls for every
sequence of the batch (256 sequences per GPU), the last of which folds the
window into the fp32 checkpoint; so a step decodes 256 x 16 tokens per GPU
and every timed step moves the same bytes.  The timed region starts with the
checkpoint, the ring buffers and a pool of 32 seeded synthetic tokens already
resident in HBM; the 1 GiB (Mamba-2) / 512 MiB (GDN) checkpoint is far larger
than the 126 MB L2, so no L2 flush is needed between steps.

Multi-GPU: each rank decodes its own independent batch of 256 sequences
(replicas; the decode path has no exchange step), value = all ranks' tokens
divided by the slowest rank's device time.

Reported beside the headline: the conventional per-token update kernel on the
same layer and inputs (in-run baseline), the end-to-end rate through the C ABI
with host-resident inputs and outputs, the roofline of the replay kernel, and
the fp64 CPU oracle timed on this host.  ``--impl reference`` times only the
oracle (rank 0) and prints its own line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

if __name__ != "__mp_main__":   # the CPU-baseline workers (spawned) need numpy and the oracle only
    import torch
    import seeded_inputs as si  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0     # B200 HBM3e, nominal
POOL = 32


# ------------------------------------------------------------------ helpers
def dist_setup(ngpus, backend="nccl"):
    """One process per GPU (torch.distributed.run sets RANK / LOCAL_RANK /
    WORLD_SIZE).  Replicas only: the process group carries the start/stop
    barriers and the max-over-ranks of the timings, never decode data."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != ngpus:
        raise SystemExit(f"--gpus {ngpus} but WORLD_SIZE={world}: launch N>1 with torch.distributed.run")
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def job_throughput(world, tokens_per_step, steps, elapsed_max):
    """Whole-job tokens/s: every rank decodes its own batch; the slowest rank's
    device time bounds the job."""
    return world * tokens_per_step * steps / elapsed_max


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML in a thread."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, dev_index, period=0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # no NVML: report it rather than guess
            self.err = str(e)

    @staticmethod
    def _handle(pynvml, dev_index):
        try:
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[dev_index]) if vis and vis.split(",")[0].isdigit() else dev_index
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self._reason_fn(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, files):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
    except Exception:
        return None
    return rec["bytes_per_launch"] if rec.get("source_hash") == source_hash(files) else None


# -------------------------------------------------------------- workloads
class Mamba2Work:
    name = "mamba2"
    keys = ("x", "B", "C", "dt")
    kernel_files = ["hybrid_ssm_decode_replayssm_b200/csrc/mamba2.cu",
                    "hybrid_ssm_decode_replayssm_b200/csrc/m2_common.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/umma.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_device.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_internal.h"]

    def __init__(self, dev, seed, batch=None, read_fmt=0, window=None):
        self.shape = s = (si.MAMBA2_SERVING if batch is None else si.MAMBA2_SERVING.with_(batch=batch))
        if window is not None:
            self.shape = s = s.with_(window=window, max_draft=min(s.max_draft, window))
        self.seed, self.dev, self.read_fmt = seed, dev, read_fmt
        A, D = si.mamba2_params(s, seed)
        self.A, self.D = A.to(dev), D.to(dev)
        self.h0 = si.mamba2_checkpoint(s, seed).to(dev)
        self.host_pool = [si.mamba2_tokens(s, t, seed) for t in range(POOL)]
        self.pool = [[tok[k].to(dev) for k in self.keys] for tok in self.host_pool]
        if dev.type == "cuda":
            from hybrid_ssm_decode_replayssm_b200 import rssm
            self.desc = rssm.make_desc(rssm.RSSM_MAMBA2, s.batch, s.nheads, s.headdim, s.dstate,
                                       ngroups=s.ngroups, window=s.window, max_draft=s.max_draft,
                                       in_dtype=rssm.RSSM_BF16, read_fmt=read_fmt)
        self.out_shape = (s.batch, s.nheads, s.headdim)
        self.tokens_per_call = s.batch
        self.workload = (f"Mamba-2 decode layer: batch {s.batch}, {s.nheads} heads, headdim {s.headdim}, "
                         f"dstate {s.dstate}, {s.ngroups} groups, bf16 x/B/C/dt, fp32 checkpoint, L={s.window}")

    def layer(self):
        from hybrid_ssm_decode_replayssm_b200 import rssm
        return rssm.ReplayLayer(self.desc, self.h0.clone(), self.A, self.D)

    def drafts(self, rnd, k):
        return [t.to(self.dev) for t in (si.mamba2_drafts(self.shape, rnd, k, self.seed)[n] for n in self.keys)]

    rc_kernel_files = ["hybrid_ssm_decode_replayssm_b200/csrc/m2_rc_decode.cu",
                       "hybrid_ssm_decode_replayssm_b200/csrc/m2_common.cuh",
                       "hybrid_ssm_decode_replayssm_b200/csrc/rssm_device.cuh",
                       "hybrid_ssm_decode_replayssm_b200/csrc/rssm_internal.h"]

    def bytes_per_call(self, pos):
        """Algorithmic bytes of the decode call at window position pos (1..L):
        the state read (fp32 checkpoint, or the read copy's codes and scales),
        token inputs, the ring append, the window entries before it, the output;
        at pos = L the fold writes the checkpoint (a read-copy layer also reads
        the fp32 checkpoint then, and writes the new copy)."""
        s = self.shape
        B, H, P, N, G, L = s.batch, s.nheads, s.headdim, s.dstate, s.ngroups, s.window
        e = 2
        ck = B * H * P * N * 4
        inp = B * H * P * e + 2 * B * G * N * e + B * H * e
        entry = B * H * P * e + B * G * N * e + B * H * 4
        out = B * H * P * 4
        if self.read_fmt == 0:
            read, fold = ck, ck
        else:
            rc = B * H * P * N + B * H * P * 4 if self.read_fmt == 1 else B * H * P * N // 2 + B * H * P * N // 16
            read, fold = rc, 2 * ck + rc
        return read + inp + entry + (pos - 1) * entry + out + (fold if pos == L else 0)

    def conventional_bytes(self):
        s = self.shape
        B, H, P, N, G = s.batch, s.nheads, s.headdim, s.dstate, s.ngroups
        return 2 * B * H * P * N * 4 + B * H * P * 2 + 2 * B * G * N * 2 + B * H * 2 + B * H * P * 4


class GDNWork:
    name = "gdn"
    keys = ("q", "k", "v", "alpha", "beta")
    kernel_files = ["hybrid_ssm_decode_replayssm_b200/csrc/dr_decode.cu",
                    "hybrid_ssm_decode_replayssm_b200/csrc/umma.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_device.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_internal.h"]

    def __init__(self, dev, seed, batch=None, read_fmt=0, window=None):
        self.shape = s = si.GDN_SERVING if batch is None else si.GDN_SERVING.with_(batch=batch)
        if window is not None:
            self.shape = s = s.with_(window=window, max_draft=min(s.max_draft, window))
        self.seed, self.dev, self.read_fmt = seed, dev, read_fmt
        self.h0 = si.gdn_checkpoint(s, seed).to(dev)
        self.host_pool = [si.gdn_tokens(s, t, seed) for t in range(POOL)]
        self.pool = [[tok[k].to(dev) for k in self.keys] for tok in self.host_pool]
        if dev.type == "cuda":
            from hybrid_ssm_decode_replayssm_b200 import rssm
            self.desc = rssm.make_desc(rssm.RSSM_GDN, s.batch, s.nheads, s.dv, s.dk, window=s.window,
                                       max_draft=s.max_draft, in_dtype=rssm.RSSM_BF16, read_fmt=read_fmt)
        self.out_shape = (s.batch, s.nheads, s.dv)
        self.tokens_per_call = s.batch
        self.workload = (f"Gated DeltaNet decode layer: batch {s.batch}, {s.nheads} heads, d_k = d_v = {s.dk}, "
                         f"bf16 q/k/v, fp32 alpha/beta, fp32 checkpoint, L={s.window}")

    def layer(self):
        from hybrid_ssm_decode_replayssm_b200 import rssm
        return rssm.ReplayLayer(self.desc, self.h0.clone())

    def drafts(self, rnd, k):
        return [t.to(self.dev) for t in (si.gdn_drafts(self.shape, rnd, k, self.seed)[n] for n in self.keys)]

    def bytes_per_call(self, pos):
        """Algorithmic bytes of the decode call at window position pos (1..L)."""
        s = self.shape
        BH, dk, dv, L = s.batch * s.nheads, s.dk, s.dv, s.window
        ck = BH * dv * dk * 4
        inputs = BH * (2 * dk + dv) * 2 + BH * 8                     # q, k, v, alpha, beta
        append = BH * (dk + dv) * 2 + BH * 8 + BH * dv * 4            # k, v, g, beta rows; new w
        entry = BH * dk * 2 + BH * dv * 4 + BH * 8                    # k, w, g, beta per window entry
        out = BH * dv * 4
        fold = ck + (L - 1) * BH * dv * 2 if pos == L else 0          # state write; v rows re-read
        return ck + inputs + append + (pos - 1) * entry + out + fold

    def conventional_bytes(self):
        s = self.shape
        BH = s.batch * s.nheads
        return 2 * BH * s.dv * s.dk * 4 + BH * (2 * s.dk + s.dv) * 2 + BH * 8 + BH * s.dv * 4


class KDAWork(GDNWork):
    """Kimi Delta Attention layer (per-channel gates) of the GDN serving shape."""
    name = "kda"
    kernel_files = ["hybrid_ssm_decode_replayssm_b200/csrc/kda_decode.cu",
                    "hybrid_ssm_decode_replayssm_b200/csrc/kda.cu",
                    "hybrid_ssm_decode_replayssm_b200/csrc/umma.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_device.cuh",
                    "hybrid_ssm_decode_replayssm_b200/csrc/rssm_internal.h"]

    def __init__(self, dev, seed, batch=None, read_fmt=0, window=None):
        self.shape = s = si.KDA_SERVING if batch is None else si.KDA_SERVING.with_(batch=batch)
        if window is not None:
            self.shape = s = s.with_(window=window)
        self.seed, self.dev, self.read_fmt = seed, dev, read_fmt
        self.h0 = si.kda_checkpoint(s, seed).to(dev)
        self.host_pool = [si.kda_tokens(s, t, seed) for t in range(POOL)]
        self.pool = [[tok[k].to(dev) for k in self.keys] for tok in self.host_pool]
        if dev.type == "cuda":
            from hybrid_ssm_decode_replayssm_b200 import rssm
            self.desc = rssm.make_desc(rssm.RSSM_KDA, s.batch, s.nheads, s.dv, s.dk, window=s.window,
                                       max_draft=0, in_dtype=rssm.RSSM_BF16)
        self.out_shape = (s.batch, s.nheads, s.dv)
        self.tokens_per_call = s.batch
        self.workload = (f"KDA decode layer: batch {s.batch}, {s.nheads} heads, d_k = d_v = {s.dk}, "
                         f"bf16 q/k/v, fp32 per-channel alpha, fp32 beta, fp32 checkpoint, L={s.window}")

    def bytes_per_call(self, pos):
        """Algorithmic bytes of the decode call at window position pos (1..L)."""
        s = self.shape
        BH, dk, dv, L = s.batch * s.nheads, s.dk, s.dv, s.window
        ck = BH * dv * dk * 4
        inputs = BH * (2 * dk + dv) * 2 + BH * dk * 4 + BH * 4       # q, k, v, alpha per channel, beta
        append = BH * (dk + dv) * 2 + BH * dk * 4 + BH * 4 + BH * dv * 4   # k, v, g, beta; new w
        entry = BH * dk * 2 + BH * dk * 4 + BH * dv * 4               # k, g, w per window entry
        out = BH * dv * 4
        fold = ck if pos == L else 0
        return ck + inputs + append + (pos - 1) * entry + out + fold

    def conventional_bytes(self):
        s = self.shape
        BH = s.batch * s.nheads
        return 2 * BH * s.dv * s.dk * 4 + BH * (2 * s.dk + s.dv) * 2 + BH * s.dk * 4 + BH * 4 + BH * s.dv * 4


WORKLOADS = {"mamba2": Mamba2Work, "gdn": GDNWork, "kda": KDAWork}


# ------------------------------------------------------------------ timing
def time_replay(work, layer, steps, warmup, L, out, dev, world, sampler_dev):
    """Device-time `steps` windows of L decode calls (the headline), then the same
    number of windows again with an event pair around every launch (the
    per-launch durations of the roofline)."""
    from hybrid_ssm_decode_replayssm_b200 import rssm
    stream = torch.cuda.current_stream()
    t = 0
    for _ in range(warmup * L):
        layer.decode_step(work.pool[t % POOL], out)
        t += 1
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = rssm.lib().rssm_launch_count()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(sampler_dev) as clk:
        start.record(stream)
        for _ in range(steps * L):
            layer.decode_step(work.pool[t % POOL], out)
            t += 1
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    launches = rssm.lib().rssm_launch_count() - launches0
    elapsed = start.elapsed_time(stop) / 1e3

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps * L)]
    first_pos = t % L
    for i in range(steps * L):
        ev[i][0].record(stream)
        layer.decode_step(work.pool[t % POOL], out)
        ev[i][1].record(stream)
        t += 1
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) / 1e3 for a, b in ev]
    positions = [((first_pos + i) % L) + 1 for i in range(steps * L)]
    return elapsed, per, positions, launches, clk.summary()


def time_conventional(work, layer, steps, warmup, L, out, world):
    state = work.h0.clone()
    t = 0
    for _ in range(warmup * L):
        layer.conventional_step(state, state, work.pool[t % POOL], out)
        t += 1
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    start.record()
    for _ in range(steps * L):
        layer.conventional_step(state, state, work.pool[t % POOL], out)
        t += 1
    stop.record()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(stop) / 1e3


def time_e2e(work, layer, steps, warmup, L, dev, world):
    """Inputs copied host->device from pinned memory and outputs copied back every
    call, pipelined on separate copy streams, through the C-ABI decode call."""
    host_in = [[t.pin_memory() for t in (tok[k] for k in work.keys)] for tok in work.host_pool]
    nslot = 4
    dev_in = [[torch.empty_like(t, device=dev) for t in host_in[0]] for _ in range(nslot)]
    dev_out = [torch.empty(work.out_shape, device=dev) for _ in range(nslot)]
    host_out = [torch.empty(work.out_shape).pin_memory() for _ in range(nslot)]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp = torch.cuda.current_stream()
    ev_in = [torch.cuda.Event() for _ in range(nslot)]
    ev_done = [torch.cuda.Event() for _ in range(nslot)]
    ev_out = [torch.cuda.Event() for _ in range(nslot)]
    for e in ev_out:
        e.record(s_d2h)
    in_bytes = sum(t.numel() * t.element_size() for t in host_in[0])
    out_bytes = dev_out[0].numel() * 4

    def run(ncalls, t0):
        for i in range(ncalls):
            slot, t = i % nslot, t0 + i
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(ev_done[slot])          # slot's inputs no longer read
                for d, h in zip(dev_in[slot], host_in[t % POOL]):
                    d.copy_(h, non_blocking=True)
                ev_in[slot].record(s_h2d)
            comp.wait_event(ev_in[slot])
            comp.wait_event(ev_out[slot])                # slot's previous output copied out
            layer.decode_step(dev_in[slot], dev_out[slot], stream=comp)
            ev_done[slot].record(comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_done[slot])
                host_out[slot].copy_(dev_out[slot], non_blocking=True)
                ev_out[slot].record(s_d2h)
        return t0 + ncalls

    t = run(warmup * L, 0)
    torch.cuda.synchronize()
    barrier(world)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    run(steps * L, t)
    comp.wait_stream(s_d2h)
    comp.wait_stream(s_h2d)
    stop.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(stop) / 1e3, in_bytes * L, out_bytes * L


def _cpu_oracle_worker(kind, state0, toks, params, go, conn):
    """(A spawned process.)  Run the fp64 oracle, as it stands, on one block of
    sequences for every token in `toks`, BLAS at one thread; report the time."""
    from threadpoolctl import threadpool_limits
    if kind == "mamba2":
        from oracle import mamba2 as om
        step = lambda S, t: om.step(S, t["x"], t["B"], t["C"], t["dt"], params["A"], params["D"])
    elif kind == "gdn":
        from oracle import gdn as og
        step = lambda S, t: og.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    else:
        from oracle import kda as ok
        step = lambda S, t: ok.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    S = np.asarray(state0, np.float64)
    toks = [{k: np.asarray(v, np.float64) for k, v in t.items()} for t in toks]
    with threadpool_limits(1):
        conn.send("ready")
        go.wait()
        t0 = time.perf_counter()
        for t in toks:
            S, _ = step(S, t)
        conn.send(time.perf_counter() - t0)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(work, seed, steps=None, cores=None):
    """The fp64 oracle as it stands, on this host's cores: the batch is split into
    one block of sequences per core, each block runs in its own (spawned) process
    with BLAS at one thread, all start together, and the rate is the whole
    batch's tokens over the wall time until the last block is done.  Sample:
    every sequence of the batch for one window (L decode tokens)."""
    import multiprocessing as mp
    steps = steps or work.shape.window
    cores = cores or host_cores()
    B = work.shape.batch
    nproc = max(1, min(cores, B))
    blocks = np.array_split(np.arange(B), nproc)
    state = work.h0.cpu().numpy()
    toks = [{k: v.float().numpy() for k, v in work.host_pool[t % POOL].items()} for t in range(steps)]
    params = {"A": work.A.double().cpu().numpy(), "D": work.D.double().cpu().numpy()} if work.name == "mamba2" else None
    ctx = mp.get_context("spawn")
    go = ctx.Event()
    procs, conns = [], []
    for blk in blocks:
        parent, child = ctx.Pipe()
        p = ctx.Process(target=_cpu_oracle_worker, daemon=True,
                        args=(work.name, state[blk], [{k: v[blk] for k, v in t.items()} for t in toks], params, go, child))
        p.start()
        procs.append(p)
        conns.append(parent)
    for c in conns:
        assert c.recv() == "ready"
    t0 = time.perf_counter()
    go.set()
    per = [c.recv() for c in conns]
    wall = time.perf_counter() - t0
    for p in procs:
        p.join(60)
    return {"value": B * steps / wall, "unit": "tokens/s", "cores": nproc, "kind": "oracle",
            "sample": (f"all {B} sequences x {steps} decode tokens (one window) of the fp64 numpy recurrence, "
                       f"split over {nproc} processes (one per host core, BLAS 1 thread each)"),
            "seconds": round(wall, 2), "slowest_block_s": round(max(per), 2)}


def time_plain_decode(work, layer, steps, warmup, L):
    """Device time of `steps` windows of L decode calls (no per-launch events)."""
    out = torch.empty(work.out_shape, device=work.dev)
    t = 0
    for _ in range(warmup * L):
        layer.decode_step(work.pool[t % POOL], out)
        t += 1
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps * L):
        layer.decode_step(work.pool[t % POOL], out)
        t += 1
    stop.record()
    torch.cuda.synchronize()
    return start.elapsed_time(stop) / 1e3


def speculative_leg(work, rounds=512, warmup=4, k=4):
    """Verify k drafts, accept a seeded prefix U{0..k} per sequence, roll back the
    rest (a fold happens inside verify when the window cannot take k more).
    Baseline: snapshot verify, k conventional steps each writing a new state copy."""
    B = work.shape.batch
    layer = work.layer()
    drafts = [work.drafts(r, k) for r in range(8)]
    accepts = [si.accept_counts(B, r, k, work.seed) for r in range(rounds + warmup)]
    rejects = [(k - a).to(torch.int32).to(work.dev) for a in accepts]
    out = torch.empty((B, k) + work.out_shape[1:], device=work.dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for r in range(warmup):
        layer.verify(k, drafts[r % 8], out)
        layer.rollback(rejects[r])
    e0, e1 = ev(), ev()
    rb = [(ev(), ev()) for _ in range(rounds)]
    torch.cuda.synchronize()
    e0.record()
    for r in range(rounds):
        layer.verify(k, drafts[r % 8], out)
        rb[r][0].record()
        layer.rollback(rejects[warmup + r])
        rb[r][1].record()
    e1.record()
    torch.cuda.synchronize()
    el = e0.elapsed_time(e1) / 1e3
    rollback_us = statistics.mean(a.elapsed_time(b) for a, b in rb) * 1e3
    accepted = sum(int(a.sum()) for a in accepts[warmup:])
    status = layer.get_status()
    del layer
    # snapshot baseline: k snapshots of the full state per round
    snaps = [work.h0.clone() for _ in range(k + 1)]
    base = work.layer()
    one = torch.empty(work.out_shape, device=work.dev)
    draft_tokens = [[[t[:, j].contiguous() for t in drafts[r]] for j in range(k)] for r in range(8)]
    def snapshot_round(r):
        for j in range(k):
            base.conventional_step(snaps[j], snaps[j + 1], draft_tokens[r % 8][j], one)
    for r in range(warmup):
        snapshot_round(r)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record()
    for r in range(rounds):
        snapshot_round(r)
    e1.record()
    torch.cuda.synchronize()
    el_base = e0.elapsed_time(e1) / 1e3
    del base, snaps
    return {"k": k, "rounds": rounds, "verified_tokens_per_s": round(B * k * rounds / el, 1),
            "accepted_tokens_per_s": round(accepted / el, 1),
            "round_us": round(el / rounds * 1e6, 2), "rollback_us": round(rollback_us, 2),
            "mean_accepted": round(accepted / (B * rounds), 3), "status_bits": status,
            "snapshot_baseline": {"round_us": round(el_base / rounds * 1e6, 2),
                                  "accepted_tokens_per_s": round(accepted / el_base, 1),
                                  "how": f"{k} conventional steps per round, each writing a new full-state snapshot"},
            "speedup_vs_snapshot": round(el_base / el, 3)}


def branch_leg(work, steps=48, warmup=8, keep=0.5):
    """Beam-search-like decode: before every token each sequence continues from a
    seeded parent (itself with probability `keep`, else a uniformly drawn
    sequence), then one decode step.  Replay: rssm_branch on a branching layer
    (windows copied, checkpoint slots shared) + decode.  Baseline: the
    conventional design, which must give every re-parented sequence its own copy
    of the parent's full state (a gather of those rows) before its step."""
    import copy
    from hybrid_ssm_decode_replayssm_b200 import rssm
    B = work.shape.batch
    ar = torch.arange(B, device=work.dev)
    parents = [si.branch_parents(B, t, work.seed, keep).to(work.dev) for t in range(16)]
    moved = [torch.nonzero(p != ar).flatten() for p in parents]
    srcs = [p.long()[m] for p, m in zip(parents, moved)]
    desc = copy.copy(work.desc)
    desc.branching = 1
    ck = torch.zeros((2 * B,) + tuple(work.h0.shape[1:]), dtype=torch.float32, device=work.dev)
    ck[:B] = work.h0
    layer = (rssm.ReplayLayer(desc, ck, work.A, work.D) if work.name == "mamba2"
             else rssm.ReplayLayer(desc, ck))
    out = torch.empty(work.out_shape, device=work.dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for t in range(warmup):
        layer.branch(parents[t % 16])
        layer.decode_step(work.pool[t % POOL], out)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    br = [(ev(), ev()) for _ in range(steps)]
    e0.record()
    for t in range(steps):
        br[t][0].record()
        layer.branch(parents[t % 16])
        br[t][1].record()
        layer.decode_step(work.pool[t % POOL], out)
    e1.record()
    torch.cuda.synchronize()
    el = e0.elapsed_time(e1) / 1e3
    branch_us = statistics.mean(a.elapsed_time(b) for a, b in br) * 1e3
    status = layer.get_status()
    del layer, ck
    torch.cuda.empty_cache()
    base = work.layer()
    state = work.h0.clone()

    def conv_step(t):
        m = moved[t % 16]
        state.index_copy_(0, m, state.index_select(0, srcs[t % 16]))
        base.conventional_step(state, state, work.pool[t % POOL], out)
    for t in range(warmup):
        conv_step(t)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record()
    for t in range(steps):
        conv_step(t)
    e1.record()
    torch.cuda.synchronize()
    el_base = e0.elapsed_time(e1) / 1e3
    del base, state
    torch.cuda.empty_cache()
    frac = statistics.mean(float(m.numel()) / B for m in moved)
    return {"steps": steps, "reparented_fraction": round(frac, 3), "tokens_per_s": round(B * steps / el, 1),
            "step_us": round(el / steps * 1e6, 2), "branch_us": round(branch_us, 2), "status_bits": status,
            "conventional_baseline": {"tokens_per_s": round(B * steps / el_base, 1),
                                      "step_us": round(el_base / steps * 1e6, 2),
                                      "how": "gather the parents' full states into the re-parented rows, "
                                             "then a conventional step"},
            "speedup_vs_conventional": round(el_base / el, 3)}


def _window_layer(base, L, fmt):
    import copy
    work = copy.copy(base)
    work.shape = base.shape.with_(window=L, max_draft=min(base.shape.max_draft, L))
    work.desc = copy.copy(base.desc)
    work.desc.window, work.desc.max_draft, work.desc.read_fmt = L, min(base.shape.max_draft, L), fmt
    work.read_fmt = fmt
    return work


def read_copy_leg(base, windows=(1, 4, 8, 16, 32), steps=6, err_calls=64):
    """Replay decode tokens/s with the fp32 checkpoint read directly and with an
    FP8 / NVFP4 read copy, per window length (checkpoint and tokens of `base`);
    and the read copies' output error against the layer reading its fp32
    checkpoint (which the parity tests hold to the fp64 oracle at ~1e-6): per
    call |y_copy - y_fp32| / rms(y_fp32), max and rms over `err_calls` calls."""
    from hybrid_ssm_decode_replayssm_b200 import rssm
    res, err, gbs = {}, {}, {}
    fmts = (("fp32", rssm.RSSM_READ_FP32), ("fp8_e4m3_row", rssm.RSSM_READ_FP8_E4M3_ROW),
            ("nvfp4", rssm.RSSM_READ_NVFP4))
    for name, fmt in fmts:
        row = {}
        for L in windows:
            work = _window_layer(base, L, fmt)
            layer = work.layer()
            n_windows = max(2, (steps * 16) // L)
            el = time_plain_decode(work, layer, n_windows, 2, L)
            row[f"L{L}"] = round(work.shape.batch * L * n_windows / el, 1)
            if work.name == "mamba2":   # HBM bytes per second (algorithmic bytes of the window's calls)
                gbs.setdefault(name, {})[f"L{L}"] = round(
                    sum(work.bytes_per_call(p) for p in range(1, L + 1)) * n_windows / el / 1e9, 1)
            del layer
            torch.cuda.empty_cache()
        res[name] = row
    for name, fmt in fmts[1:]:
        row = {}
        for L in windows:
            ref_l = _window_layer(base, L, rssm.RSSM_READ_FP32).layer()
            rc_l = _window_layer(base, L, fmt).layer()
            y_ref = torch.empty(base.out_shape, device=base.dev)
            y_rc = torch.empty_like(y_ref)
            emax, esq = 0.0, 0.0
            for t in range(err_calls):
                ref_l.decode_step(base.pool[t % POOL], y_ref)
                rc_l.decode_step(base.pool[t % POOL], y_rc)
                rms = float(y_ref.square().mean().sqrt())
                d = (y_rc - y_ref).abs() / rms
                emax = max(emax, float(d.max()))
                esq += float(d.square().mean())
            row[f"L{L}"] = {"max": float(f"{emax:.3e}"), "rms": float(f"{(esq / err_calls) ** 0.5:.3e}")}
            del ref_l, rc_l
            torch.cuda.empty_cache()
        err[name] = row
    res["error_vs_fp32_reads"] = err
    if gbs:
        res["hbm_gbs"] = gbs
    return res


def quantized_state_leg(base, calls=96, warmup=16):
    """The conventional step on a state stored in FP8 / NVFP4 and rounded again
    every token (the design a read copy replaces): tokens/s and GB/s of state
    and token bytes, same layer shape and tokens as `base`."""
    import copy
    from hybrid_ssm_decode_replayssm_b200 import rssm
    res = {}
    s = base.shape
    rows, cols = (s.batch * s.nheads * (s.headdim if base.name == "mamba2" else s.dv),
                  s.dstate if base.name == "mamba2" else s.dk)
    for name, fmt in (("fp8_e4m3_row", rssm.RSSM_READ_FP8_E4M3_ROW), ("nvfp4", rssm.RSSM_READ_NVFP4)):
        work = copy.copy(base)
        work.desc = copy.copy(base.desc)
        work.desc.read_fmt = fmt
        layer = work.layer()
        codes, scales = layer.quantized_state_buffers()
        rc_codes, rc_scales = layer.read_copy_views()
        codes.copy_(rc_codes)
        scales.copy_(rc_scales)
        out = torch.empty(work.out_shape, device=work.dev)
        for t in range(warmup):
            layer.conventional_step_quantized(codes, scales, codes, scales, work.pool[t % POOL], out)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record()
        for t in range(calls):
            layer.conventional_step_quantized(codes, scales, codes, scales, work.pool[t % POOL], out)
        stop.record()
        torch.cuda.synchronize()
        el = start.elapsed_time(stop) / 1e3
        state = codes.numel() + scales.numel() * scales.element_size()
        tok_bytes = work.conventional_bytes() - 2 * rows * cols * 4    # inputs and outputs
        res[name] = {"tokens_per_s": round(s.batch * calls / el, 1),
                     "hbm_gbs": round((2 * state + tok_bytes) * calls / el / 1e9, 1)}
        del layer, codes, scales
        torch.cuda.empty_cache()
    return res


def graph_leg(m2, gw, steps=48, warmup=16):
    """A decode step of three layers (two Mamba-2 and one GDN layer of the serving
    shapes) launched eagerly and replayed from one captured CUDA graph."""
    layers = [m2.layer(), m2.layer(), gw.layer()]
    works = [m2, m2, gw]
    outs = [torch.empty(w.out_shape, device=w.dev) for w in works]
    ins = [[t.clone() for t in w.pool[0]] for w in works]

    def step():
        for layer, i, o in zip(layers, ins, outs):
            layer.decode_step(i, o)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step()
    stop.record()
    torch.cuda.synchronize()
    eager = start.elapsed_time(stop) / 1e3 / steps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps):
        g.replay()
    stop.record()
    torch.cuda.synchronize()
    graphed = start.elapsed_time(stop) / 1e3 / steps
    del g, layers
    torch.cuda.empty_cache()
    return {"layers": "2 x " + m2.workload.split(":")[0] + " + 1 x " + gw.workload.split(":")[0] + " (serving shapes)",
            "eager_us_per_step": round(eager * 1e6, 1), "graph_us_per_step": round(graphed * 1e6, 1),
            "graph_tokens_per_s": round(m2.shape.batch / graphed, 1)}


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--layer", default="mamba2", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="rssm", choices=["rssm", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch (profiling captures only; the metric is quoted at 256)")
    ap.add_argument("--read-fmt", default="fp32", choices=["fp32", "fp8", "nvfp4"],
                    help="read format of the timed layer (profiling captures only; the metric is quoted on fp32 reads)")
    ap.add_argument("--legs", default="replay,conventional,e2e,gdn,kda,speculative,read_copy,quantized_state,graph,branch",
                    help="comma list of timed legs (profiling captures run 'replay' alone)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    if args.impl == "reference":
        # The oracle runs on the host cores: no GPU and no process group; under
        # torchrun rank 0 alone runs it and the other ranks exit without work.
        rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
        if world != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torch.distributed.run")
        local, dev = 0, torch.device("cpu")
        if rank != 0:
            return
    else:
        rank, world, local = dist_setup(args.gpus)
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
    seed = args.seed + rank
    legs = set(args.legs.split(","))
    work = WORKLOADS[args.layer](dev, seed, args.batch, read_fmt={"fp32": 0, "fp8": 1, "nvfp4": 2}[args.read_fmt])
    L = work.shape.window
    tokens_per_step = work.tokens_per_call * L
    cfg = {"workload": work.workload, "global_batch": work.shape.batch * world,
           "tokens_per_step": tokens_per_step * world,
           "step": f"one window: {L} decode calls per sequence, the last folding the window",
           "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
           "l2": "no flush: the fp32 checkpoint (>= 512 MiB) is larger than L2 and streamed every call"}

    if args.impl == "reference":
        if rank == 0:
            cb = cpu_baseline(work, seed)
            line = {"impl": "reference", "metric": "SSM-layer decode tokens/s at batch 256",
                    "value": cb["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                    "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "config": cfg,
                    "cpu_baseline": cb,
                    "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        return

    layer = work.layer()
    out = torch.empty(work.out_shape, device=dev)
    elapsed, per, positions, launches, clocks = time_replay(work, layer, args.steps, args.warmup, L,
                                                            out, dev, world, local)
    elapsed = max_over_ranks(elapsed, world, dev)
    value = job_throughput(world, tokens_per_step, args.steps, elapsed)

    alg_bytes = sum(work.bytes_per_call(p) for p in positions)    # per-launch pass
    kern_time = sum(per)
    peak, peak_kind = measured_peak()
    achieved = alg_bytes / kern_time / 1e9
    if work.read_fmt == 0:
        traffic = ncu_traffic(f"{work.name}_decode", work.kernel_files)
    else:
        traffic = ncu_traffic(f"{work.name}_rc{work.read_fmt}_decode", getattr(work, "rc_kernel_files", work.kernel_files))
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "frac_of_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                "peak_source": f"{peak_kind} copy bandwidth",
                "kernel": f"{work.name} replay decode (append + output, fold every {L}th call)",
                "bytes_per_launch_avg": alg_bytes / len(per),
                "launch_us_avg": round(kern_time / len(per) * 1e6, 2),
                "launch_us_fold": round(statistics.mean(p for p, q in zip(per, positions) if q == L) * 1e6, 2),
                "launch_us_nofold": round(statistics.mean(p for p, q in zip(per, positions) if q != L) * 1e6, 2)}

    conv = None
    if "conventional" in legs:
        conv_el = time_conventional(work, layer, args.steps, args.warmup, L, out, world)
        conv_el = max_over_ranks(conv_el, world, dev)
        conv_value = world * tokens_per_step * args.steps / conv_el
        conv = {"value": round(conv_value, 1), "unit": "tokens/s",
                "hbm_gbs": round(work.conventional_bytes() * L * args.steps / conv_el / 1e9 * world, 1),
                "replay_speedup": round(value / conv_value, 3)}

    e2e = None
    if "e2e" in legs:
        e2e_layer = work.layer()
        e2e_el, h2d, d2h = time_e2e(work, e2e_layer, args.steps, args.warmup, L, dev, world)
        e2e_el = max_over_ranks(e2e_el, world, dev)
        e2e = {"value": round(world * tokens_per_step * args.steps / e2e_el, 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "how": "rssm_decode_step per call with pinned-host inputs copied in and outputs "
                      "copied out, pipelined on copy streams"}

    extras = {}
    if "e2e" in legs:
        del e2e_layer
    gw = None
    if world == 1 and args.layer == "mamba2" and legs & {"gdn", "speculative", "read_copy", "quantized_state", "graph", "branch"}:
        gw = GDNWork(dev, seed, args.batch)
    def layer_leg(w):
        """Replay decode of another layer type at its serving shape, with its
        conventional kernel timed beside it."""
        wl = w.layer()
        wout = torch.empty(w.out_shape, device=dev)
        w_steps = max(20, args.steps // 3)
        w_el, w_per, w_pos, _, _ = time_replay(w, wl, w_steps, args.warmup, L, wout, dev, 1, local)
        w_bytes = sum(w.bytes_per_call(p) for p in w_pos)
        wc_el = time_conventional(w, wl, w_steps, args.warmup, L, wout, 1)
        res = {"workload": w.workload, "value": round(w.tokens_per_call * L * w_steps / w_el, 1),
               "unit": "tokens/s", "hbm_gbs": round(w_bytes / w_el / 1e9, 1),
               "roofline_frac": round(w_bytes / sum(w_per) / 1e9 / measured_peak()[0], 4),
               "frac_of_8tbs": round(w_bytes / sum(w_per) / 1e9 / NOMINAL_HBM_GBS, 4),
               "launch_us_fold": round(statistics.mean(p for p, q in zip(w_per, w_pos) if q == L) * 1e6, 2),
               "launch_us_nofold": round(statistics.mean(p for p, q in zip(w_per, w_pos) if q != L) * 1e6, 2),
               "conventional_tokens_per_s": round(w.tokens_per_call * L * w_steps / wc_el, 1),
               "replay_speedup": round(wc_el / w_el, 3), "status_bits": wl.get_status()}
        del wl
        torch.cuda.empty_cache()
        return res

    if world == 1 and "gdn" in legs and gw is not None:
        extras["gdn"] = layer_leg(gw)
    if world == 1 and "kda" in legs and args.layer == "mamba2":
        extras["kda"] = layer_leg(KDAWork(dev, seed, args.batch))
        torch.cuda.empty_cache()
    if world == 1 and "speculative" in legs:
        extras["speculative"] = {"mamba2": speculative_leg(work)}
        torch.cuda.empty_cache()
        if gw is not None:
            extras["speculative"]["gdn"] = speculative_leg(gw)
            torch.cuda.empty_cache()
    if world == 1 and "branch" in legs:
        extras["branch"] = {"how": "beam-search-like: each sequence re-parented with probability 1/2 before "
                                   "every token", work.name: branch_leg(work)}
        if gw is not None:
            extras["branch"]["gdn"] = branch_leg(gw)
    if world == 1 and "read_copy" in legs:
        extras["read_copy"] = {work.name: read_copy_leg(work)}
        if gw is not None:
            extras["read_copy"]["gdn"] = read_copy_leg(gw)
    if world == 1 and "graph" in legs and gw is not None:
        extras["multi_layer_graph"] = graph_leg(work, gw)
    if world == 1 and "quantized_state" in legs:
        extras["quantized_state_baseline"] = {
            "how": "conventional step on a state stored in the format and rounded again every token",
            work.name: quantized_state_leg(work)}
        if gw is not None:
            extras["quantized_state_baseline"]["gdn"] = quantized_state_leg(gw)
    del gw
    torch.cuda.empty_cache()

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(work, seed)

    if rank == 0:
        # the comparisons come last (a reader that keeps only the end of the line sees them)
        tail, layers = {}, {}
        for k in ("gdn", "kda"):
            if k in extras:
                tail[k] = extras.pop(k)
                layers[k] = tail[k].pop("workload")
        if layers:
            extras = {"other_layers": layers, **extras}
        summary = {}
        if "speculative" in extras:
            summary["speculative_accepted_tokens_per_s"] = {
                k: {"replay": v["accepted_tokens_per_s"], "snapshot": v["snapshot_baseline"]["accepted_tokens_per_s"],
                    "speedup": v["speedup_vs_snapshot"]} for k, v in extras["speculative"].items()}
        if "read_copy" in extras:
            summary["read_copy_L16"] = {
                k: {"tokens_per_s": {f: v[f]["L16"] for f in ("fp32", "fp8_e4m3_row", "nvfp4")},
                    "error_vs_fp32_reads_max": {f: v["error_vs_fp32_reads"][f]["L16"]["max"]
                                                for f in ("fp8_e4m3_row", "nvfp4")}}
                for k, v in extras["read_copy"].items()}
        line = {"metric": "SSM-layer decode tokens/s at batch 256", "value": round(value, 1),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded; bf16 inputs, fp32 checkpoint)", "config": cfg,
                "hbm_gbs": round(alg_bytes / elapsed / 1e9 * world, 1),   # same calls, headline pass
                "clocks": clocks, "gpu_launches": int(launches),
                **extras,
                "cpu_baseline": cb, "e2e": e2e, "roofline": roofline,
                "conventional": conv, **tail, **summary}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
