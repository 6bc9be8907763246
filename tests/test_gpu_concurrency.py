"""Decode steps of two caches on two unordered CUDA streams at the same time (GPU).

The fused decode step runs on a persistent grid of one CTA per SM. Two such
launches on two streams can each hold part of the SMs while the rest of their
CTAs wait to be scheduled. No CTA of a launch waits on another CTA of it: the
step reads one copy of the per-stream counts and writes the other (a state
parity the host flips), and the window ring keeps w + 1 entries, so the entry
of the token that leaves and the entry the new token writes are different
words. So both launches finish whatever share of the device each gets.

Both streams wait on one event, recorded behind a sleeping kernel on a third
stream, while every step of both caches is queued; the event releases both at
the same moment, so the queued launches run back to back on the two streams at
once. Which stream's launch takes the SMs first is the hardware's choice, so a
run in which one stream finished before the other began proves nothing: the
test takes up to three attempts, each checked in full, and fails if none of
them overlapped.
Outputs of every step and sequence are checked against the fp64 oracle, the
bookkeeping of both caches bit for bit against the slot-pool simulator.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_kv_cache_decode_b200 import _native
from learned_kv_cache_decode_b200 import workloads as W
from harness import Run, compare, to_device

pytestmark = pytest.mark.gpu


def wl(name, batch, hq, hkv, d, dtype, w, ctx_range, steps, p, seed):
    return W.Workload(name, batch, hq, hkv, d, dtype, w, 0, ctx_range, steps, "bernoulli", (p,), seed)


def stage(run, steps):
    """Decode inputs of `steps` steps on the device, the simulator advanced step by
    step, and the position count of every sequence after each step."""
    B = run.wl.batch
    seqs = list(range(B))
    dev, seen = [], []
    for t in range(steps):
        K, V, A, Q = run.decode_inputs(t, seqs)
        dev.append((to_device(K, run.wl), to_device(V, run.wl), torch.from_numpy(A).cuda(), to_device(Q, run.wl), Q))
        rc, _ = run.sim.append(seqs, [1] * B, A)
        assert rc == 0, rc
        run.seen += 1
        seen.append(run.seen.copy())
    return dev, seen


def oracle_at(run, b, T, q):
    K, V = W.kv(run.wl, b, 0, T)
    A = run.alpha_of(b, 0, T, K)
    return oracle.decode_gqa(W.to_f64(q), W.to_f64(K), W.to_f64(V), A, run.wl.window, run.scale)


STEPS = 24      # decode steps per attempt
ATTEMPTS = 3    # attempts to see the two streams overlap (each checked in full)

CASES = [
    (wl("concurrent-a-g7-d128", 6, 28, 4, 128, "bf16", 32, (300, 2500), STEPS * ATTEMPTS, 0.7, 61),
     wl("concurrent-b-g2-d64", 8, 16, 8, 64, "bf16", 16, (100, 1800), STEPS * ATTEMPTS, 0.6, 62)),
    (wl("concurrent-c-g7-d128", 5, 28, 4, 128, "bf16", 8, (40, 1200), STEPS * ATTEMPTS, 0.8, 63),
     wl("concurrent-d-g7-d128", 5, 28, 4, 128, "bf16", 8, (40, 1200), STEPS * ATTEMPTS, 0.8, 64)),
]


def attempt(runs, streams, fused):
    """Queue STEPS steps of both caches behind one gate, release both streams at
    once, check every output and the bookkeeping; return the streams' time spans."""
    staged = [stage(run, STEPS) for run in runs]
    outs = [torch.empty((STEPS, run.wl.batch, run.wl.num_q_heads, run.wl.head_dim), dtype=torch.bfloat16,
                        device="cuda") for run in runs]
    ids = [torch.arange(run.wl.batch, dtype=torch.int32, device="cuda") for run in runs]
    torch.cuda.synchronize()
    begin = [torch.cuda.Event(enable_timing=True) for _ in runs]
    end = [torch.cuda.Event(enable_timing=True) for _ in runs]
    gate = torch.cuda.Stream()
    t0 = torch.cuda.Event(enable_timing=True)
    go = torch.cuda.Event()
    with torch.cuda.stream(gate):
        t0.record(gate)
        torch.cuda._sleep(50_000_000)   # holds both streams while they are filled
        go.record(gate)
    for s in streams:
        s.wait_event(go)
    for r, s in enumerate(streams):
        with torch.cuda.stream(s):
            begin[r].record(s)
    for t in range(STEPS):
        for r, (run, s) in enumerate(zip(runs, streams)):
            K, V, A, Q, _ = staged[r][0][t]
            with torch.cuda.stream(s):
                if fused:
                    run.cache.decode_step(ids[r], K, V, A, Q, scale=run.scale, out=outs[r][t])
                else:
                    run.cache.append(ids[r], K, V, A)
                    run.cache.decode_attention(ids[r], Q, scale=run.scale, out=outs[r][t])
    for r, s in enumerate(streams):
        with torch.cuda.stream(s):
            end[r].record(s)
    torch.cuda.synchronize()
    for run in runs:
        assert run.cache.status() == _native.DMS_OK
        run.check_metadata()
    for r, run in enumerate(runs):
        dev, seen = staged[r]
        for t in range(STEPS):
            Q = dev[t][4]
            for b in range(run.wl.batch):
                compare(outs[r][t, b], oracle_at(run, b, int(seen[t][b]), Q[b]))
    return [(t0.elapsed_time(b), t0.elapsed_time(e)) for b, e in zip(begin, end)]


@pytest.mark.parametrize("fused", [True, False], ids=["fused_step", "two_launches"])
@pytest.mark.parametrize("pair", CASES, ids=["different_shapes", "same_shape"])
def test_two_caches_step_on_two_unordered_streams_at_once(pair, fused):
    runs = [Run(case) for case in pair]
    streams = [torch.cuda.Stream() for _ in runs]
    try:
        for run in runs:
            run.prefill(chunk=333)
            run.check_metadata()
        seen = []
        for _ in range(ATTEMPTS):
            spans = attempt(runs, streams, fused)
            seen.append(spans)
            if spans[0][0] < spans[1][1] and spans[1][0] < spans[0][1]:
                break
        else:
            pytest.fail(f"the two streams never overlapped in {ATTEMPTS} attempts: {seen}")
    finally:
        for run in runs:
            run.close()
