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
import math

import numpy as np
import pytest
import torch

import oracle
from learned_kv_cache_decode_b200 import _native, decode_attention_noalloc
from learned_kv_cache_decode_b200 import workloads as W
from harness import MAX_ABS, MEAN_ABS, Run, compare, to_device

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


def wl(name, batch, hq, hkv, d, dtype, w, ctx_range, steps, p, seed):
    return W.Workload(name, batch, hq, hkv, d, dtype, w, 0, ctx_range, steps, "bernoulli", (p,), seed)


@pytest.mark.parametrize("case", [
    wl("noalloc-subset-bf16-g7-d128", 5, 28, 4, 128, "bf16", 16, (1, 1500), 2, 0.7, 43),
    wl("noalloc-subset-f32-g4-d64", 4, 8, 2, 64, "f32", 8, (30, 600), 2, 0.5, 44),
], ids=["bf16-g7-d128", "f32-g4-d64"])
def test_noalloc_permuted_subset_against_the_oracle(case):
    """A call on a permuted subset of the sequences: its call streams are not the
    cache's stream ids. Two calls in a row, every output against the fp64 oracle."""
    run = Run(case, check_sim=False)
    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
    try:
        run.prefill(chunk=257)
        seqs = [3, 0, 2] if case.batch > 4 else [2, 0]
        for step in range(2):
            run.decode_step(step)   # one more token everywhere (the cache's own path)
            torch.cuda.synchronize()
            pool, table, retained = caller_buffers(run)
            Q = W.query(case, 100 + step)[seqs]
            ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
            out = torch.empty((len(seqs), case.num_q_heads, case.head_dim), dtype=pool.dtype, device="cuda")
            got = decode_attention_noalloc(pool, table, retained, case.num_kv_heads, ids, to_device(Q, case),
                                           scale=run.scale, out=out)
            torch.cuda.synchronize()
            for j, b in enumerate(seqs):
                compare(got[j], run.oracle_out(b, Q[j]), **tol)
    finally:
        run.close()


def test_plans_with_different_stream_counts_share_one_kernel():
    """Caches of 8 and 512 streams and an allocation-free call of 4 streams use the
    same attention kernel with plans of different shared-memory sizes. The kernel's
    shared-memory limit is one attribute of the function for the whole process, so
    no plan's set-up may lower it under another plan: after the small call's set-up,
    both caches still decode (two launches and the fused step), against the oracle."""
    small = Run(wl("shared-fn-small", 2, 8, 4, 128, "bf16", 16, (100, 400), 3, 0.6, 73))
    big = Run(wl("shared-fn-big", 128, 8, 4, 128, "bf16", 16, (10, 70), 3, 0.6, 74))
    try:
        small.prefill(chunk=97)
        big.prefill(chunk=64)
        for step, fused in ((0, False), (1, False), (2, True)):
            out_s, Qs = small.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            for b in range(2):
                compare(out_s[b], small.oracle_out(b, Qs[b]))
            pool, table, retained = caller_buffers(small)   # the noalloc plan of 4 streams comes last
            got = decode_attention_noalloc(pool, table, retained, 4, torch.tensor([1], dtype=torch.int32,
                                           device="cuda"), to_device(Qs[[1]], small.wl), scale=small.scale)
            torch.cuda.synchronize()
            compare(got[0], small.oracle_out(1, Qs[1]))
            out_b, Qb = big.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            for b in range(0, 128, 9):
                compare(out_b[b], big.oracle_out(b, Qb[b]))
        for run in (small, big):
            run.check_metadata()
            assert run.cache.status() == _native.DMS_OK
    finally:
        small.close()
        big.close()


def test_noalloc_clamps_retained_counts_to_the_page_table():
    """Caller-owned counts outside [0, 16 * max_pages_per_stream] are clamped: a
    count past the page table's reach attends exactly the rows the table can
    address, a negative one gives zeros. The other streams are unaffected."""
    d, g, mps, mp = 64, 4, 3, 8
    gen = torch.Generator().manual_seed(75)
    pool = torch.randn((mp, 2, 16, d), generator=gen).to(torch.bfloat16)
    table = torch.tensor([[5, 2, 7], [1, 0, 3], [4, 6, 0]], dtype=torch.int32)
    retained = torch.tensor([16 * mps + 37, -50, 21], dtype=torch.int32)
    Q = torch.randn((3, g, d), generator=gen).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    got = decode_attention_noalloc(pool.cuda(), table.cuda(), retained.cuda(), 1,
                                   torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda"), Q.cuda(),
                                   scale=scale)
    torch.cuda.synchronize()
    f64 = pool.double().numpy()
    for st, n in ((0, 16 * mps), (2, 21)):   # stream 0 clamped to its three pages
        rows = [(int(table[st, l // 16]), l % 16) for l in range(n)]
        K = np.stack([f64[p, 0, r] for p, r in rows])
        V = np.stack([f64[p, 1, r] for p, r in rows])
        ref = oracle.attention(Q[st].double().numpy(), K, V, np.zeros(n, dtype=np.uint8), n + 1, scale)
        compare(got[st], ref)
    assert torch.count_nonzero(got[1]) == 0
