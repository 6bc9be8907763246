#!/usr/bin/env python
"""Benchmark of the DMS decode step on B200: retained-KV HBM GB/s and decode steps/s.

One step = for every layer cache: dms_append (one token per sequence, slot
reuse, page pops), dms_stats, dms_decode_attention (split-K over the
retained pages with the combine inside the same kernel). The prompt is
bulk-appended beforehand (untimed). Inputs are seeded synthetic tensors with
the shapes of the named workload (learned_kv_cache_decode_b200.workloads).

Several layer caches with distinct pools are cycled inside every step so the
retained K/V read per step is several times the 126 MB L2: timed reads come
from HBM, not from L2.

  python bench.py [--gpus N --steps K --warmup W --workload NAME --layers L]
  python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

Under torchrun each rank runs its own replica on its own GPU (streams are
independent; there is no data-path collective); rank 0 prints one JSON line
with the whole-job value and the max time over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from learned_kv_cache_decode_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "retained-KV HBM GB/s and decode steps/sec (per layer, 1 B200) vs roofline"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen-r1-7b-32k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--layers", type=int, default=0, help="layer caches per step (0: enough to exceed 8x L2)")
    ap.add_argument("--attn-kernel", default="auto", choices=["auto", "mma", "simt"])
    ap.add_argument("--window", type=int, default=0,
                    help="override the workload's delayed-eviction window w (1 = immediate eviction)")
    ap.add_argument("--step", default="fused", choices=["fused", "separate"],
                    help="fused: one dms_decode_step launch per layer; separate: dms_append + dms_decode_attention")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--per-workload", dest="per_workload", action="store_true", default=True,
                    help="also measure the other workloads (and a dense run) into a per_workload block (default)")
    ap.add_argument("--no-per-workload", dest="per_workload", action="store_false")
    ap.add_argument("--depth", default="",
                    help="CR_FIRST,CR_LAST: compression growing with depth, each layer cache with its "
                         "own alpha rate (workloads.depth_layers); per-layer dms_stats at every step; "
                         "no e2e pass")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# inputs

def host_prompt(wl, seqs, ctx):
    """Prompt K, V (bf16 bits or f32), alpha for the given sequences, concatenated in call order."""
    Ks, Vs, As = [], [], []
    for b, s in zip(seqs, ctx):
        K, V = W.kv(wl, b, 0, int(s))
        Ks.append(K)
        Vs.append(V)
        As.append(W.alpha(wl, b, 0, int(s)))
    return np.concatenate(Ks), np.concatenate(Vs), np.concatenate(As)


def host_decode(wl, seqs, ctx, steps):
    """Decode-token inputs for `steps` steps: K, V [steps, B, Hkv, d], alpha [steps, B, Hkv], Q [steps, B, Hq, d]."""
    Ks, Vs, As = [], [], []
    for b, s in zip(seqs, ctx):
        K, V = W.kv(wl, b, int(s), steps)
        Ks.append(K)
        Vs.append(V)
        As.append(W.alpha(wl, b, int(s), steps))
    K = np.stack(Ks, axis=1)
    V = np.stack(Vs, axis=1)
    A = np.stack(As, axis=1)
    Q = np.stack([W.query(wl, 1_000_000 * (seqs[0] // wl.batch) + t)[[b % wl.batch for b in seqs]]
                  for t in range(steps)])
    return K, V, A, Q


def to_torch(x, device):
    import torch
    if x.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device) if device is not None else t


# ---------------------------------------------------------------------------
# clocks (NVML reads only; nothing is changed)

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period: float = 0.005):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml unavailable" if not self.ok else "no samples"}
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit and k != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "source": "nvml, 5 ms poll"}


# ---------------------------------------------------------------------------
# helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_fingerprint(path: str) -> str:
    """sha256 of a C++/CUDA source with its comments and whitespace removed: it
    changes with the code, not with the comments."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return hashlib.sha256(re.sub(r"\s+", "", text).encode()).hexdigest()


def profile_traffic(workload: str, kernel: str, entry: str = "dms_decode_attention"):
    """Per-launch DRAM bytes of the timed kernel from the committed ncu summary,
    valid only while the kernel code is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", f"{entry}_{kernel}_{workload}.md")
    src = os.path.join(ROOT, "learned_kv_cache_decode_b200", "csrc", "dms_attention.cu")
    try:
        text = open(path).read()
        sha = code_fingerprint(src)
        m_sha = re.search(r"code_sha256:\s*([0-9a-f]{64})", text)
        m_tr = re.search(r"traffic_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
        if m_sha and m_tr and m_sha.group(1) == sha:
            return float(m_tr.group(1))
    except OSError:
        pass
    return None


def rank_sequences(rank: int, batch: int) -> list[int]:
    """Global sequence ids of one rank: every rank owns a full batch of its own (weak scaling)."""
    return [rank * batch + b for b in range(batch)]


def reduce_over_ranks(t_ms: float, nbytes: float, world: int, device) -> tuple[float, float]:
    """(max over ranks of the timed region, sum over ranks of the bytes); identity at world == 1."""
    if world <= 1:
        return t_ms, nbytes
    import torch
    import torch.distributed as dist
    v = torch.tensor([t_ms], dtype=torch.float64, device=device)
    dist.all_reduce(v, op=dist.ReduceOp.MAX)
    b = torch.tensor([nbytes], dtype=torch.float64, device=device)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(v.item()), float(b.item())


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle as it stands

def oracle_sample(wl, seqs, steps_done, prompt, dec, n_items=None):
    """Oracle inputs (float64) for the streams of `seqs` at their current last position."""
    items, nbytes = [], 0
    ctx = W.contexts(wl)
    K_p, V_p, A_p, offs = prompt
    Kd, Vd, Ad, Qd = dec
    for k, b in enumerate(seqs):
        s0, s1 = offs[k], offs[k + 1]
        T = int(ctx[b % wl.batch]) + steps_done
        Kfull = np.concatenate([K_p[s0:s1], Kd[:steps_done, k]])
        Vfull = np.concatenate([V_p[s0:s1], Vd[:steps_done, k]])
        Afull = np.concatenate([A_p[s0:s1], Ad[:steps_done, k]])
        q = W.to_f64(Qd[max(steps_done - 1, 0), k])
        g = wl.group
        for h in range(wl.num_kv_heads):
            a = Afull[:, h]
            vis = int(np.count_nonzero((a == 0) | (np.arange(T) > T - 1 - wl.window)))
            nbytes += vis * wl.head_dim * 2 * wl.elem_bytes
            items.append((q[h * g:(h + 1) * g], W.to_f64(Kfull[:, h]), W.to_f64(Vfull[:, h]), a))
            if n_items and len(items) >= n_items:
                return items, nbytes
    return items, nbytes


def time_oracle(items, window, scale, target_s):
    import oracle
    reps, t_total, threads = 0, 0.0, 1
    while t_total < target_s or reps == 0:
        t0 = time.perf_counter()
        _, threads = oracle.attention_batch(items, window, scale)
        t_total += time.perf_counter() - t0
        reps += 1
    return reps, t_total, threads


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    seqs = [0]
    ctx = W.contexts(wl)[seqs]
    K_p, V_p, A_p = host_prompt(wl, seqs, ctx)
    offs = np.concatenate([[0], np.cumsum(ctx)])
    dec = host_decode(wl, seqs, ctx, 1)
    items, nbytes = oracle_sample(wl, seqs, 1, (K_p, V_p, A_p, offs), dec)
    scale = 1.0 / math.sqrt(wl.head_dim)
    import oracle
    for _ in range(args.warmup):
        oracle.attention_batch(items, wl.window, scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _, threads = oracle.attention_batch(items, wl.window, scale)
    dt = time.perf_counter() - t0
    value = nbytes * args.steps / dt / 1e9
    sample = (f"{len(items)} streams (sequence 0, every KV head) of one decode step at the prompt's end; "
              f"fp64 definition-form oracle, OpenMP over streams")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "q_heads": wl.num_q_heads,
                   "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "window": wl.window,
                   "context": wl.context if wl.ctx_range is None else list(wl.ctx_range)},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm

NOMINAL_HBM_GBS = 8000.0   # the B200's nominal HBM3e bandwidth (about 8 TB/s), for the second fraction


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def time_oracle_one_core(items, window, scale, target_s):
    """The oracle's single-stream routine called stream after stream (one core)."""
    import oracle
    reps, t_total = 0, 0.0
    while t_total < target_s or reps == 0:
        t0 = time.perf_counter()
        for q, K, V, a in items:
            oracle.attention(q, K, V, a, window, scale)
        t_total += time.perf_counter() - t0
        reps += 1
    return reps, t_total


def measure(wl, args, world, rank, local, dev, *, steps, warmup, layers=0, depth=None, want_e2e=True,
            want_cpu=False, fused=True, cpu_seconds=None):
    """Prefill L layer caches of workload `wl`, then time decode steps. Returns the
    figures of one workload (and, with want_e2e / want_cpu, its e2e and CPU passes)."""
    import torch
    import torch.distributed as dist
    from learned_kv_cache_decode_b200 import DmsCache

    # this rank's sequences (weak scaling: every rank runs a full batch of its own sequences)
    seqs = rank_sequences(rank, wl.batch)
    ctx_all = W.contexts(wl)
    ctx = np.array([ctx_all[b % wl.batch] for b in seqs])
    B, hkv, hq, d = wl.batch, wl.num_kv_heads, wl.num_q_heads, wl.head_dim
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    burst_steps = 5
    # timed, per-launch, burst and e2e passes
    n_dec = warmup + steps * (3 if want_e2e else 2) + burst_steps
    mps = int((ctx.max() + n_dec) // 16 + 2)
    scale = 1.0 / math.sqrt(d)

    # prompt inputs (host, then device), shared by all layer caches
    K_p, V_p, A_p = host_prompt(wl, seqs, ctx)
    offs = np.concatenate([[0], np.cumsum(ctx)]).astype(np.int64)
    dK, dV, dA = to_torch(K_p, dev), to_torch(V_p, dev), torch.from_numpy(A_p).to(dev)
    d_cu = torch.from_numpy(offs.astype(np.int32)).to(dev)
    ids = torch.arange(B, dtype=torch.int32, device=dev)   # cache-local sequence ids

    def new_layer(max_pages, alpha):
        c = DmsCache(B, hkv, d, wl.window, max_pages, mps, dtype=tdt, attn_kernel=args.attn_kernel)
        c.append(ids, dK, dV, alpha, cu_tokens=d_cu)
        return c

    A_first = None
    if depth:
        # One alpha stream per layer (compression growing with depth); worst-case pools.
        L = layers or 8
        layer_wls = W.depth_layers(wl, L, depth[0], depth[-1])
        pool = B * hkv * mps
        caches = []
        for lw in layer_wls:
            a_l = np.concatenate([W.alpha(lw, b, 0, int(c_)) for b, c_ in zip(seqs, ctx)])
            A_first = a_l if A_first is None else A_first
            caches.append(new_layer(pool, torch.from_numpy(a_l).to(dev)))
    else:
        # Probe cache (worst-case pool) to learn the retained counts, then size every
        # layer pool to what the prompt keeps plus room for every decode token.
        probe = new_layer(B * hkv * mps, dA)
        st0 = probe.stats()
        torch.cuda.synchronize()
        retained = st0["retained"].cpu().numpy().astype(np.int64)
        retained0 = int(retained.sum())
        probe.close()
        del probe
        pool = int(((retained + 15) // 16).sum()) + B * hkv * (n_dec // 16 + 2)
        layer_bytes = retained0 * d * 2 * wl.elem_bytes
        L = layers or max(1, min(32, math.ceil(8 * L2_BYTES / max(layer_bytes, 1))))
        caches = [new_layer(pool, dA) for _ in range(L)]
    torch.cuda.synchronize()
    del dK, dV, dA
    torch.cuda.empty_cache()
    for c in caches:
        if c.status() != 0:
            raise RuntimeError(f"prefill failed: status {c.status()}")

    # decode-step inputs: device-resident for the timed pass, pinned host for the e2e pass
    Kd, Vd, Ad, Qd = host_decode(wl, seqs, ctx, n_dec)
    if depth:   # [L, steps, B, Hkv]: every layer its own decisions
        Ad = np.stack([np.stack([W.alpha(lw, b, int(c_), n_dec) for b, c_ in zip(seqs, ctx)], axis=1)
                       for lw in layer_wls])
    t_K, t_V, t_A, t_Q = (to_torch(x, dev) for x in (Kd, Vd, Ad, Qd))
    outs = [torch.empty((B, hq, d), dtype=tdt, device=dev) for _ in range(L)]
    # (seen, retained) totals after every step: of layer 0 (every layer holds the same
    # tokens), or of every layer with --depth
    totals = torch.zeros((n_dec, L if depth else 1, 2), dtype=torch.int64, device=dev)

    lib = caches[0].lib
    hs = [c._h for c in caches]
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    row_kv = B * hkv * d * wl.elem_bytes
    row_q = B * hq * d * wl.elem_bytes
    pK, pV, pA, pQ = t_K.data_ptr(), t_V.data_ptr(), t_A.data_ptr(), t_Q.data_ptr()
    pT = totals.data_ptr()
    pids = ids.data_ptr()
    ev_pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(steps * L)]
    t_pl = warmup + steps   # first step of the per-launch pass
    odt = 0 if tdt == torch.bfloat16 else 1

    def alpha_ptr(t, l):
        return pA + ((l * n_dec if depth else 0) + t) * B * hkv

    def step(t, timed):
        for l in range(L):
            h = hs[l]
            rc = 0
            if not fused:
                rc |= lib.dms_append(h, sp, B, pids, None, B, pK + t * row_kv, pV + t * row_kv, alpha_ptr(t, l))
            if timed:
                e0, e1 = ev_pairs[(t - t_pl) * L + l]
                e0.record(stream)
            if fused:
                rc |= lib.dms_decode_step(h, sp, B, pids, pK + t * row_kv, pV + t * row_kv, alpha_ptr(t, l),
                                          pQ + t * row_q, hq, scale, outs[l].data_ptr(), odt)
            else:
                rc |= lib.dms_decode_attention(h, sp, B, pids, pQ + t * row_q, hq, scale, outs[l].data_ptr(), odt)
            if timed:
                e1.record(stream)
            if depth:   # every layer its own retained set
                rc |= lib.dms_stats(h, sp, None, None, None, pT + (t * L + l) * 16)
            elif l == 0:   # every layer holds the same tokens: one stats call gives the bytes of all
                rc |= lib.dms_stats(h, sp, None, None, None, pT + t * 16)
            if rc:
                raise RuntimeError(f"library call failed ({rc})")

    for t in range(warmup):
        step(t, False)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches0 = sum(c.launches() for c in caches)
    ev_start, ev_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev_start.record(stream)
        for t in range(warmup, warmup + steps):
            step(t, False)
        ev_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_ms = ev_start.elapsed_time(ev_end)
    launches = sum(c.launches() for c in caches) - launches0

    # Per-launch pass: the next `steps` steps again, with an event pair around
    # every attention launch. The events serialise each launch behind the one
    # before it, so these durations include the launch latency that the
    # timed region overlaps; they are the conservative per-kernel figure.
    for t in range(t_pl, t_pl + steps):
        step(t, True)
    torch.cuda.synchronize()
    tot = totals.cpu().numpy()                                         # [steps, 1 or L, 2]
    per_layer = tot if depth else np.repeat(tot, L, axis=1)            # [steps, L, 2]
    timed_tot = per_layer[warmup:warmup + steps].sum(axis=1)           # [steps, 2] over layers
    bytes_launch = per_layer[warmup:warmup + steps, :, 1].astype(np.float64) * d * 2 * wl.elem_bytes
    total_bytes = float(bytes_launch.sum())
    same = [c.stats()["totals"].cpu().numpy().tolist() for c in caches]
    if not depth and any(x != same[0] for x in same):
        raise RuntimeError(f"layer caches diverged: {same}")
    attn_ms = np.array([a.elapsed_time(b) for a, b in ev_pairs])
    bytes_pl = per_layer[t_pl:t_pl + steps, :, 1].astype(np.float64) * d * 2 * wl.elem_bytes
    status = [c.status() for c in caches]
    if any(status):
        raise RuntimeError(f"device status {status}")

    # max over ranks of the timed region; whole-job bytes
    t_max_ms, bytes_all = reduce_over_ranks(t_ms, total_bytes, world, dev)
    value = bytes_all / (t_max_ms * 1e-3) / 1e9
    achieved_iso = float(bytes_pl.mean()) / (float(attn_ms.mean()) * 1e-3) / 1e9

    # Burst: `burst_steps` more steps between one event pair, no event between
    # launches, so each launch's set-up overlaps the launch before it
    # (programmatic dependent launch). Separate mode times the attention
    # launches alone. Reported beside the per-launch figure, not instead of it.
    t_b = t_pl + steps
    e_b0, e_b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if fused:
        e_b0.record(stream)
        for t in range(t_b, t_b + burst_steps):
            step(t, False)
        e_b1.record(stream)
    else:
        for t in range(t_b, t_b + burst_steps):   # keep the decode going: append outside the events
            for l in range(L):
                lib.dms_append(hs[l], sp, B, pids, None, B, pK + t * row_kv, pV + t * row_kv, alpha_ptr(t, l))
            lib.dms_stats(hs[0], sp, None, None, None, pT + t * 16)
        e_b0.record(stream)
        for t in range(t_b, t_b + burst_steps):
            for l in range(L):
                lib.dms_decode_attention(hs[l], sp, B, pids, pQ + t * row_q, hq, scale, outs[l].data_ptr(), odt)
        e_b1.record(stream)
    torch.cuda.synchronize()
    burst_ms = e_b0.elapsed_time(e_b1) / (burst_steps * L)
    b_tot = totals.cpu().numpy()[t_b:t_b + burst_steps]   # [steps, 1 or L, 2]
    achieved_burst = float(b_tot[:, :, 1].astype(np.float64).mean()) * d * 2 * wl.elem_bytes / (burst_ms * 1e-3) / 1e9
    # Roofline of the dominant kernel. Fused: the timed region holds the step
    # launches, back to back as a decode loop issues them, plus one small
    # dms_stats launch per step, so its average launch duration is this rank's
    # region time over its step launches (the stats launches count against
    # it). Separate: the attention launches alone, back to back between one
    # event pair (the burst). The per-launch event pairs are reported beside
    # it: an event between two launches makes each start only once the one
    # before has finished, which removes the overlap of consecutive launches.
    if fused:
        launch_ms = t_ms / (steps * L)
        achieved = float(bytes_launch.mean()) / (launch_ms * 1e-3) / 1e9
    else:
        launch_ms = burst_ms
        achieved = achieved_burst
    peak, peak_kind = peaks()

    res = {
        "wl": wl, "L": L, "B": B, "hq": hq, "hkv": hkv, "d": d, "ctx": ctx, "value": value, "t_max_ms": t_max_ms,
        "steps": steps, "total_bytes": total_bytes, "launches": launches, "clocks": clk.summary(),
        "timed_tot": timed_tot, "per_layer": per_layer, "warmup": warmup,
        "bytes_launch": float(bytes_launch.mean()) if fused else float(bytes_pl.mean()),
        "launch_ms": launch_ms, "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
        "attn_ms": attn_ms, "achieved_iso": achieved_iso, "burst_ms": burst_ms, "achieved_burst": achieved_burst,
    }

    # ---- end-to-end pass through the public API with pinned host buffers. Per
    # step and per layer: one host-to-device copy of each input a model step
    # feeds that layer (its new K and V rows, alpha and Q; every layer gets its
    # own copy of the bytes) and one device-to-host copy of every layer's
    # output. The copies run on their own stream, double-buffered, so step
    # t+1's inputs and step t-1's outputs move while step t computes; events
    # order every reuse.
    if want_e2e and not depth:
        rep = lambda x: np.ascontiguousarray(np.broadcast_to(x[:, None], (x.shape[0], L) + x.shape[1:]))
        hK, hV, hA, hQ = (to_torch(rep(x), None).pin_memory() for x in (Kd, Vd, Ad, Qd))   # [steps, L, ...]
        h_out = [torch.empty((L, B, hq, d), dtype=tdt).pin_memory() for _ in range(2)]
        d_out = [torch.empty((L, B, hq, d), dtype=tdt, device=dev) for _ in range(2)]
        stage = [(torch.empty((L, B, hkv, d), dtype=tdt, device=dev),
                  torch.empty((L, B, hkv, d), dtype=tdt, device=dev),
                  torch.empty((L, B, hkv), dtype=torch.uint8, device=dev),
                  torch.empty((L, B, hq, d), dtype=tdt, device=dev))
                 for _ in range(2)]
        copy_s = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        t0_e2e = t_b + burst_steps
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

        def h2d(t):
            p = t % 2
            k_, v_, a_, q_ = stage[p]
            with torch.cuda.stream(copy_s):
                if t - 2 >= t0_e2e:
                    copy_s.wait_event(comp_done[p])   # step t-2 has finished reading this staging set
                k_.copy_(hK[t], non_blocking=True)
                v_.copy_(hV[t], non_blocking=True)
                a_.copy_(hA[t], non_blocking=True)
                q_.copy_(hQ[t], non_blocking=True)
                h2d_done[p].record(copy_s)

        e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_a.record(stream)
        copy_s.wait_stream(stream)
        h2d(t0_e2e)
        for t in range(t0_e2e, t0_e2e + steps):
            p = t % 2
            k_, v_, a_, q_ = stage[p]
            if t + 1 < t0_e2e + steps:
                h2d(t + 1)
            stream.wait_event(h2d_done[p])
            if t - 2 >= t0_e2e:
                stream.wait_event(d2h_done[p])    # step t-2's outputs have left this buffer
            for l in range(L):
                if fused:
                    caches[l].decode_step(ids, k_[l], v_[l], a_[l], q_[l], scale=scale, out=d_out[p][l])
                else:
                    caches[l].append(ids, k_[l], v_[l], a_[l])
                    caches[l].decode_attention(ids, q_[l], scale=scale, out=d_out[p][l])
                if l == 0:
                    lib.dms_stats(hs[l], sp, None, None, None, pT + t * 16)
            comp_done[p].record(stream)
            with torch.cuda.stream(copy_s):
                copy_s.wait_event(comp_done[p])
                h_out[p].copy_(d_out[p], non_blocking=True)
                d2h_done[p].record(copy_s)
        stream.wait_stream(copy_s)
        e_b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e_a.elapsed_time(e_b)
        tot2 = totals.cpu().numpy()[t0_e2e:t0_e2e + steps, 0]   # layer 0 stands for all (no --depth)
        e2e_bytes = float(tot2[:, 1].astype(np.float64).sum()) * L * d * 2 * wl.elem_bytes
        e2e_ms, e2e_bytes = reduce_over_ranks(e2e_ms, e2e_bytes, world, dev)
        h2d_b = L * (2 * row_kv + B * hkv + row_q)
        d2h_b = L * B * hq * d * wl.elem_bytes
        res["e2e"] = {"value": e2e_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d_b,
                      "d2h_bytes_per_step": d2h_b, "ms_per_step": e2e_ms / steps,
                      "copies": "per layer: new K, V rows, alpha and Q in, output out; own stream, "
                                "double-buffered (step t+1 in, step t-1 out while step t computes)"}

    # ---- CPU baseline: the oracle on a bounded sample of the same step (rank 0, N = 1)
    if want_cpu:
        sample_seqs = list(range(min(B, 2)))
        A_s, Ad_s = (A_first, Ad[0]) if depth else (A_p, Ad)   # --depth: layer 0's decisions
        items, nbytes = oracle_sample(wl, [seqs[i] for i in sample_seqs], warmup + steps,
                                      (K_p, V_p, A_s, offs),
                                      (Kd[:, sample_seqs], Vd[:, sample_seqs], Ad_s[:, sample_seqs],
                                       Qd[:, sample_seqs]))
        cpu_s = args.cpu_seconds if cpu_seconds is None else cpu_seconds
        reps, t_cpu, threads = time_oracle(items, wl.window, scale, cpu_s)
        reps1, t_cpu1 = time_oracle_one_core(items, wl.window, scale, cpu_s / 2)
        # per decode step of the whole workload (every stream of every layer), from the sample's rate
        step_bytes = total_bytes / steps
        res["cpu"] = {
            "value": nbytes * reps / t_cpu / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "one_core": {"value": nbytes * reps1 / t_cpu1 / 1e9, "unit": "GB/s", "cores": 1,
                         "ms_per_step": step_bytes / (nbytes * reps1 / t_cpu1) * 1e3},
            "ms_per_step": step_bytes / (nbytes * reps / t_cpu) * 1e3,
            "sample": f"{len(items)} streams (sequences {sample_seqs}, every KV head) at the last timed step, "
                      f"repeated {reps}x on {threads} threads ({t_cpu:.1f} s) and {reps1}x on one core "
                      f"({t_cpu1:.1f} s); fp64 definition-form oracle; ms_per_step scales the sample's rate "
                      f"to every stream of every layer of one step"}

    for c in caches:
        c.close()
    del caches
    torch.cuda.empty_cache()
    return res


def brief(res):
    """The per-workload figures of one measurement."""
    wl = res["wl"]
    peak = res["peak"]
    return {
        "value": res["value"], "unit": "GB/s", "ms_per_step": res["t_max_ms"] / res["steps"],
        "layers": res["L"], "steps": res["steps"],
        "bytes_per_launch": res["bytes_launch"], "launch_ms": res["launch_ms"],
        "frac": res["achieved"] / peak, "frac_nominal": res["achieved"] / NOMINAL_HBM_GBS,
        "launch_ms_isolated": float(res["attn_ms"].mean()),
        "frac_isolated": res["achieved_iso"] / peak, "frac_isolated_nominal": res["achieved_iso"] / NOMINAL_HBM_GBS,
        "compression_ratio": float(res["timed_tot"][-1, 0] / res["timed_tot"][-1, 1]),
        "decode_steps_per_s_per_layer": res["steps"] * res["L"] / (res["t_max_ms"] * 1e-3),
        "context": int(res["ctx"].max()) if wl.ctx_range is None else list(wl.ctx_range),
        "clocks_sm_mhz": res["clocks"].get("sm_mhz"),
    }


def per_workload_runs(args, world, rank, local, dev, main_wl):
    """The other workloads, each measured with fewer steps, no e2e and a short
    oracle sample (all host cores and one core); the long run at both ends of its
    decode loop; a dense (all kept) run of the 32K workload for context; the tiny
    workload as a correctness-only note."""
    import dataclasses
    steps = min(args.steps, 20)
    runs = {}
    lr = W.WORKLOADS["longrun-2k-30k"]
    jobs = [
        ("llama3.2-1b", W.WORKLOADS["llama3.2-1b"]),
        ("qwen-r1-32b-chains", W.WORKLOADS["qwen-r1-32b-chains"]),
        ("longrun-2k-30k@2k", lr),
        # the state after its 30K decode steps: the prompt and every decode token appended at
        # once (a bulk append equals token-by-token appends), then timed
        ("longrun-2k-30k@32k", dataclasses.replace(lr, context=lr.context + lr.decode_steps)),
        ("qwen-r1-7b-32k-dense", dataclasses.replace(W.WORKLOADS["qwen-r1-7b-32k"], alpha_mode="bernoulli",
                                                     alpha_args=(0.0,))),
    ]
    if main_wl.name != "qwen-r1-7b-32k":
        jobs.insert(0, ("qwen-r1-7b-32k", W.WORKLOADS["qwen-r1-7b-32k"]))
    for name, wl in jobs:
        if wl.name == main_wl.name and wl == main_wl:
            continue
        t0 = time.perf_counter()
        r = measure(wl, args, world, rank, local, dev, steps=steps, warmup=3, want_e2e=False,
                    want_cpu=not args.no_cpu_baseline, fused=args.step == "fused", cpu_seconds=3.0)
        runs[name] = brief(r)
        if "cpu" in r:   # a short oracle sample of the same step: all host cores and one core
            runs[name]["oracle_ms_per_step"] = r["cpu"]["ms_per_step"]
            runs[name]["oracle_ms_per_step_one_core"] = r["cpu"]["one_core"]["ms_per_step"]
            runs[name]["oracle_cores"] = r["cpu"]["cores"]
        runs[name]["wall_s"] = time.perf_counter() - t0
    runs["tiny"] = {"note": "correctness only: one fp32 stream of about 280 retained tokens (0.15 MB per step), "
                            "checked every step against the oracle in tests/test_gpu_configs.py"}
    return runs


def main():
    args = parse_args()
    wl = W.WORKLOADS[args.workload]
    if args.window:
        import dataclasses
        wl = dataclasses.replace(wl, window=args.window)
    depth = [float(x) for x in args.depth.split(",")] if args.depth else None
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    fused = args.step == "fused"
    res = measure(wl, args, world, rank, local, dev, steps=args.steps, warmup=args.warmup, layers=args.layers,
                  depth=depth, want_e2e=not (args.no_e2e or depth),
                  want_cpu=rank == 0 and world == 1 and not args.no_cpu_baseline, fused=fused)
    per = None
    if args.per_workload and not depth and not args.window and world == 1:
        per = per_workload_runs(args, world, rank, local, dev, wl)

    if rank == 0:
        L, B, hq, hkv, d = res["L"], res["B"], res["hq"], res["hkv"], res["d"]
        steps = args.steps
        peak, achieved = res["peak"], res["achieved"]
        kernel = {"auto": "mma" if wl.dtype == "bf16" else "simt"}.get(args.attn_kernel, args.attn_kernel)
        attn_ms, timed_tot, per_layer = res["attn_ms"], res["timed_tot"], res["per_layer"]
        launch_timing = ("timed region (CUDA events at its two ends) over its step launches; "
                         "isolated: an event pair around every launch, in a second pass over the next steps"
                         if fused else
                         "attention launches back to back between one event pair (the burst); "
                         "isolated: an event pair around every launch, in a second pass over the next steps")
        line = {
            "metric": METRIC, "value": res["value"], "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": res["t_max_ms"] / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {
                "workload": wl.name, "batch_per_gpu": B, "q_heads": hq, "kv_heads": hkv, "head_dim": d,
                "window": wl.window,
                "context": int(res["ctx"].max()) if wl.ctx_range is None else list(wl.ctx_range),
                "layers": L, "attn_kernel": kernel, "parallelism": f"replicas x{world}",
                "l2": f"inputs larger than L2: {L} layer pools, {res['total_bytes'] / steps / 2**20:.0f} MiB "
                      f"retained K/V read per step vs 126 MiB L2",
                "step": ("per layer: dms_decode_step (append 1 token/seq + attention, one launch)" if fused else
                         "per layer: dms_append (1 token/seq) + dms_decode_attention") +
                        ("; one dms_stats per layer per step" if depth else "; one dms_stats per step"),
            },
            "decode_steps_per_s_per_layer": steps * L / (res["t_max_ms"] * 1e-3),
            "retained_bytes_per_step": res["total_bytes"] / steps,
            "compression_ratio": float(timed_tot[-1, 0] / timed_tot[-1, 1]),
            **({"depth": {"cr_schedule": depth, "layer_cr": [
                float(x) for x in per_layer[args.warmup + steps - 1, :, 0] /
                per_layer[args.warmup + steps - 1, :, 1]]}} if depth else {}),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": res["peak_kind"],
                         "frac_nominal": achieved / NOMINAL_HBM_GBS, "peak_nominal": NOMINAL_HBM_GBS,
                         "traffic": profile_traffic(wl.name, kernel,
                                                    "dms_decode_step" if fused else "dms_decode_attention"),
                         "kernel": f"dms_decode_step ({kernel}, append fused)" if fused else
                                   f"dms_decode_attention ({kernel})",
                         "bytes_per_launch": res["bytes_launch"],
                         "launch_ms": res["launch_ms"], "launch_timing": launch_timing,
                         "launch_ms_isolated": float(attn_ms.mean()),
                         "launch_ms_isolated_p10": float(np.percentile(attn_ms, 10)),
                         "launch_ms_isolated_p90": float(np.percentile(attn_ms, 90)),
                         "achieved_isolated": res["achieved_iso"], "frac_isolated": res["achieved_iso"] / peak,
                         "frac_isolated_nominal": res["achieved_iso"] / NOMINAL_HBM_GBS,
                         "launch_ms_burst": res["burst_ms"], "achieved_burst": res["achieved_burst"],
                         "frac_burst": res["achieved_burst"] / peak},
            "gpu_launches": res["launches"],
            "clocks": res["clocks"],
        }
        if "e2e" in res:
            line["e2e"] = res["e2e"]
        if "cpu" in res:
            line["cpu_baseline"] = res["cpu"]
        if per is not None:
            line["per_workload"] = per
        print(json.dumps(line), flush=True)

    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
