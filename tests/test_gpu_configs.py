"""The five decode workloads at full size, CUDA path vs the CPU oracle (GPU).

Metadata (page tables, counters, free stack, retained sets of every
stream) is compared bit for bit after the prefill and at checkpoints;
attention outputs are compared on sampled (step, sequence) pairs and for
every sequence at the last step, all query heads, against the fp64 oracle in
definition form.
"""
import numpy as np
import pytest
import torch

from learned_kv_cache_decode_b200 import workloads as W
from learned_kv_cache_decode_b200 import _native
from harness import Run, compare

pytestmark = pytest.mark.gpu


def _run_config(name, check_steps, check_seqs, steps=None, chunk=4096, metadata_every=None, fused=False):
    """Sampled sequences at the steps in check_steps, and every sequence at the last step."""
    wl = W.WORKLOADS[name]
    run = Run(wl, steps=steps)
    try:
        run.prefill(chunk=chunk)
        run.check_metadata()
        n = run.steps
        for step in range(n):
            out, Q = run.decode_step(step, fused=fused)
            if step == n - 1:
                torch.cuda.synchronize()
                ref = run.oracle_all(Q)
                for b in range(wl.batch):
                    compare(out[b], ref[b])
            elif step in check_steps:
                torch.cuda.synchronize()
                for b in check_seqs:
                    compare(out[b], run.oracle_out(b, Q[b]))
            if metadata_every and (step + 1) % metadata_every == 0:
                run.check_metadata()
        run.check_metadata()
        assert run.cache.status() == _native.DMS_OK
        return run
    finally:
        run.close()


def test_tiny_every_step_every_head():
    wl = W.WORKLOADS["tiny"]
    run = Run(wl)
    try:
        run.prefill(chunk=512)
        run.check_metadata()
        for step in range(wl.decode_steps):
            out, Q = run.decode_step(step)
            torch.cuda.synchronize()
            compare(out[0], run.oracle_out(0, Q[0]), max_abs=1e-4, mean_abs=1e-5)
        run.check_metadata()
    finally:
        run.close()


def test_llama32_1b_shape():
    _run_config("llama3.2-1b", check_steps={0, 128, 255}, check_seqs=range(8), metadata_every=64)


def test_qwen_r1_7b_32k():
    _run_config("qwen-r1-7b-32k", check_steps={0, 255}, check_seqs=[0, 7, 15], metadata_every=128)


def test_qwen_r1_32b_chains():
    _run_config("qwen-r1-32b-chains", check_steps={0, 255}, check_seqs=[0, 21, 63], metadata_every=128)


@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
def test_longrun_2k_30k(fused):
    """2K prompt then 30K decode steps; slot reuse, page-table growth and sequence
    restarts (page returns and re-pops) checked against the oracle every 1K steps,
    through dms_append + dms_decode_attention or through dms_decode_step."""
    wl = W.WORKLOADS["longrun-2k-30k"]
    run = Run(wl)
    try:
        run.prefill(chunk=2048)
        run.check_metadata()
        for step in range(wl.decode_steps):
            if step > 0 and step % 5000 == 0:
                # one sequence finishes and a new one starts in its place
                b = (step // 5000) % wl.batch
                run.cache.reset_seq(b)
                assert run.sim.reset_seq(b) == 0
                run.seen[b] = 0
                run._blk.pop(b, None)
                run.ctx[b] = 1024
                run.prefill(chunk=1024, seqs=[b])
            out, Q = run.decode_step(step, fused=fused)
            if (step + 1) % 1000 == 0:
                torch.cuda.synchronize()
                run.check_metadata()
                for b in (step % wl.batch, (step * 7 + 3) % wl.batch):
                    compare(out[b], run.oracle_out(b, Q[b]))
        st = run.cache.stats()
        tot = st["totals"].cpu().numpy()
        assert 6.0 < tot[0] / tot[1] < 9.0, tot      # CR about 8 with p = 0.875
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


def test_qwen_r1_7b_32k_fused_step():
    """The same workload through dms_decode_step (append and attention in one launch)."""
    _run_config("qwen-r1-7b-32k", check_steps={0, 255}, check_seqs=[0, 7, 15], metadata_every=128, fused=True)


def test_qwen_r1_32b_chains_fused_step():
    _run_config("qwen-r1-32b-chains", check_steps={0, 255}, check_seqs=[0, 21, 63], metadata_every=128,
                fused=True)
