"""dms_decode_attention_noalloc against dms_decode_attention (GPU).

The allocation-free entry point serves callers that may not allocate device
memory while they decode (a framework whose caching allocator owns the
device memory, a runtime that lends the library its K/V pages). It takes
the caller's pool, page table and retained counts and keeps its split-K
scratch in a static device array. Here the caller's buffers are built from
a dms_cache (its page table and counts from dms_snapshot, its rows from
dms_gather_kv), and two calls in a row must agree with the cache's own
entry point within the bf16 (or f32) tolerance of the parity tests.

This file is named so that pytest collects it last: if it fails, a run that
stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from learned_kv_cache_decode_b200 import _native, decode_attention_noalloc
from learned_kv_cache_decode_b200 import workloads as W
from harness import MAX_ABS, MEAN_ABS, Run, to_device

pytestmark = pytest.mark.gpu


def caller_buffers(run):
    """The cache's K/V, page table and counts copied into caller-owned tensors."""
    cache, wl = run.cache, run.wl
    snap = cache.snapshot()
    mp, mps, d = cache.cfg.max_pages, cache.cfg.max_pages_per_stream, wl.head_dim
    pool = torch.zeros((mp, 2, 16, d), dtype=cache.cfg.dtype, device="cuda")
    for st in range(cache.streams):
        n = int(snap["n"][st])
        if n == 0:
            continue
        K, V = cache.gather_kv(st // wl.num_kv_heads, st % wl.num_kv_heads, n)
        slots = torch.arange(n, device="cuda")
        pages = torch.from_numpy(snap["page_table"][st, : (n + 15) // 16].astype(np.int64)).cuda()[slots // 16]
        pool[pages, 0, slots % 16] = K
        pool[pages, 1, slots % 16] = V
    table = torch.from_numpy(snap["page_table"]).cuda()
    retained = torch.from_numpy(snap["n"]).cuda()
    return pool, table, retained


def check_close(got, ref, f32):
    diff = (got.float() - ref.float()).abs()
    max_abs, mean_abs = (1e-4, 1e-5) if f32 else (MAX_ABS, MEAN_ABS)
    assert float(diff.max()) <= max_abs and float(diff.mean()) <= mean_abs, (float(diff.max()), float(diff.mean()))


CASES = [
    W.Workload("noalloc-bf16-g7-d128", 3, 21, 3, 128, "bf16", 32, 0, (40, 900), 2, "bernoulli", (0.6,), 41),
    W.Workload("noalloc-f32-g4-d64", 2, 8, 2, 64, "f32", 16, 0, (1, 500), 2, "bernoulli", (0.5,), 42),
]


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_cache_entry_point_twice(wl):
    run = Run(wl, check_sim=False)
    try:
        run.prefill(chunk=333)
        ids = torch.arange(wl.batch, dtype=torch.int32, device="cuda")
        f32 = wl.dtype == "f32"
        for step in range(2):   # two calls in a row, each after one more decode token
            out_ref, Q = run.decode_step(step)
            torch.cuda.synchronize()
            pool, table, retained = caller_buffers(run)
            out = torch.empty_like(out_ref)
            got = decode_attention_noalloc(pool, table, retained, wl.num_kv_heads, ids, to_device(Q, wl),
                                           scale=run.scale, out=out)
            torch.cuda.synchronize()
            check_close(got, out_ref, f32)
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


def test_noalloc_rejects_more_streams_than_its_scratch_holds():
    hkv, d = 8, 128
    n_seqs = _native.DMS_NOALLOC_MAX_STREAMS // hkv + 1
    pool = torch.zeros((4, 2, 16, d), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((n_seqs * hkv, 1), dtype=torch.int32, device="cuda")
    retained = torch.zeros(n_seqs * hkv, dtype=torch.int32, device="cuda")
    ids = torch.arange(n_seqs, dtype=torch.int32, device="cuda")
    Q = torch.zeros((n_seqs, hkv, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_native.DmsError) as e:
        decode_attention_noalloc(pool, table, retained, hkv, ids, Q)
    assert e.value.code == _native.DMS_ERR_INVALID
