"""CUDA path vs the CPU oracle on small seeded cases (GPU).

Each case spans several pages and split-K pieces, ragged last pages and
sequences of very different lengths. Metadata (page tables, counters, free
stack, retained sets) must match the oracle's simulator bit for bit;
outputs must be within max abs 2e-2 / mean abs 2e-3 of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_kv_cache_decode_b200 import alpha_from_logit
from learned_kv_cache_decode_b200 import workloads as W
from learned_kv_cache_decode_b200 import _native
from harness import Run, compare, to_device

pytestmark = pytest.mark.gpu


def wl(name, batch, hq, hkv, d, dtype, w, ctx_range, steps, p, seed):
    return W.Workload(name, batch, hq, hkv, d, dtype, w, 0, ctx_range, steps, "bernoulli", (p,), seed)


CASES = [
    wl("f32-g4-d64", 2, 8, 2, 64, "f32", 16, (1, 300), 5, 0.5, 11),
    wl("f32-g7-d128", 2, 14, 2, 128, "f32", 16, (30, 400), 4, 0.5, 12),
    wl("bf16-g7-d128", 3, 14, 2, 128, "bf16", 16, (1, 700), 5, 0.6, 13),
    wl("bf16-g4-d64", 3, 8, 2, 64, "bf16", 64, (100, 900), 5, 0.7, 14),
    wl("bf16-g5-d128-w1", 2, 10, 2, 128, "bf16", 1, (0, 200), 4, 0.5, 15),
    wl("bf16-g8-d64", 2, 16, 2, 64, "bf16", 32, (17, 500), 4, 0.9, 16),
    wl("bf16-g1-d128", 3, 3, 3, 128, "bf16", 8, (5, 90), 4, 0.3, 17),
    wl("bf16-g2-d64-dense", 2, 4, 2, 64, "bf16", 16, (40, 600), 4, 0.0, 18),
    wl("bf16-g4-d128-window", 2, 8, 2, 128, "bf16", 48, (40, 600), 4, 1.0, 19),
    wl("bf16-g7-d128-wide-window", 2, 14, 2, 128, "bf16", 4096, (100, 700), 4, 0.5, 20),
]


def kernels_for(w):
    return ["simt"] if w.dtype == "f32" else ["mma", "simt"]


@pytest.mark.parametrize("case", CASES, ids=[c.name for c in CASES])
def test_small_cases(case):
    for kern in kernels_for(case):
        run = Run(case, attn_kernel=kern)
        try:
            run.prefill(chunk=97)    # several bulk calls per sequence, odd sizes
            run.check_metadata()
            for step in range(case.decode_steps):
                out, Q = run.decode_step(step)
                torch.cuda.synchronize()
                for b in range(case.batch):
                    ref = run.oracle_out(b, Q[b])
                    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
                    compare(out[b], ref, **tol)
            run.check_metadata()
            assert run.cache.status() == _native.DMS_OK
        finally:
            run.close()


def test_kv_rows_are_copied_bit_exactly():
    case = wl("gather", 2, 8, 2, 128, "bf16", 16, (200, 300), 3, 0.5, 21)
    run = Run(case)
    try:
        run.prefill(chunk=64)
        for step in range(3):
            run.decode_step(step)
        for b in range(case.batch):
            T = int(run.seen[b])
            K, V = W.kv(case, b, 0, T)
            for h in range(case.num_kv_heads):
                pos = run.sim.retained(b * case.num_kv_heads + h)
                gk, gv = run.cache.gather_kv(b, h, len(pos))
                gk = gk.view(torch.int16).cpu().numpy().view(np.uint16)
                gv = gv.view(torch.int16).cpu().numpy().view(np.uint16)
                np.testing.assert_array_equal(gk, K[pos, h])
                np.testing.assert_array_equal(gv, V[pos, h])
    finally:
        run.close()


def test_stats_match_oracle_counts():
    case = wl("stats", 4, 8, 2, 64, "bf16", 16, (10, 500), 2, 0.6, 22)
    run = Run(case)
    try:
        run.prefill()
        run.decode_step(0)
        st = run.cache.stats()
        o = run.sim.snapshot()
        np.testing.assert_array_equal(st["retained"].cpu().numpy(), o["n"])
        np.testing.assert_array_equal(st["seen"].cpu().numpy(), o["pos"])
        tot = st["totals"].cpu().numpy()
        assert tot[0] == o["pos"].sum() and tot[1] == o["n"].sum()
        for h in range(case.num_kv_heads):
            ref = o["pos"][h::case.num_kv_heads].sum() / o["n"][h::case.num_kv_heads].sum()
            assert abs(float(st["head_cr"][h]) - ref) <= 1e-6 * ref
    finally:
        run.close()


@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
def test_stats_host_matches_oracle_counts(fused):
    """dms_stats_host: host per-stream counts and the overall CR (fp64) equal to the
    simulator's, after decode steps of either path (a fused step flips the state parity
    the host copies from)."""
    case = wl("stats-host", 4, 8, 2, 64, "bf16", 16, (10, 500), 3, 0.6, 23)
    run = Run(case)
    try:
        run.prefill()
        for step in range(3):
            run.decode_step(step, fused=fused)
            st = run.cache.stats_host()
            o = run.sim.snapshot()
            np.testing.assert_array_equal(st["retained"], o["n"])
            np.testing.assert_array_equal(st["seen"], o["pos"])
            assert st["cr_overall"] == float(o["pos"].sum()) / float(o["n"].sum())
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


def test_depth_wise_compression_per_layer():
    """Layer caches whose compression grows with depth (W.depth_layers, CR 2 -> 16 over 4
    layers) stepped through the fused path in turn: every output against the oracle, and
    each layer's dms_stats (per-stream counts, per-head and overall CR) equal to the
    oracle's counts; the measured ratios grow layer over layer."""
    base = wl("depth", 3, 14, 2, 128, "bf16", 16, (300, 900), 6, 0.5, 43)
    runs = [Run(x) for x in W.depth_layers(base, 4, 2.0, 16.0)]
    try:
        for run in runs:
            run.prefill(chunk=257)
        for step in range(base.decode_steps):
            for run in runs:
                out, Q = run.decode_step(step, fused=True)
                torch.cuda.synchronize()
                for b in range(base.batch):
                    compare(out[b], run.oracle_out(b, Q[b]))
        crs = []
        for run in runs:
            st = run.cache.stats()
            o = run.sim.snapshot()
            np.testing.assert_array_equal(st["retained"].cpu().numpy(), o["n"])
            np.testing.assert_array_equal(st["seen"].cpu().numpy(), o["pos"])
            tot = st["totals"].cpu().numpy()
            assert tot[0] == o["pos"].sum() and tot[1] == o["n"].sum()
            for h in range(base.num_kv_heads):
                ref = o["pos"][h::base.num_kv_heads].sum() / o["n"][h::base.num_kv_heads].sum()
                assert abs(float(st["head_cr"][h]) - ref) <= 1e-6 * ref
            crs.append(tot[0] / tot[1])
            assert run.cache.status() == _native.DMS_OK
        assert crs == sorted(crs) and crs[-1] > 3 * crs[0], crs
    finally:
        for run in runs:
            run.close()


def test_empty_and_partial_batches():
    """Sequences never appended give zeros; decode over a subset, in any order."""
    case = wl("subset", 5, 8, 2, 64, "bf16", 16, (0, 300), 3, 0.5, 23)
    run = Run(case)
    try:
        run.prefill(seqs=[0, 2, 4])
        ids = torch.tensor([1, 3], dtype=torch.int32, device="cuda")
        q = torch.randn(2, 8, 64, device="cuda").to(torch.bfloat16)
        out = run.cache.decode_attention(ids, q)
        assert torch.count_nonzero(out) == 0
        for step in range(3):
            out, Q = run.decode_step(step, seqs=[4, 0])
            torch.cuda.synchronize()
            for k, b in enumerate([4, 0]):
                compare(out[k], run.oracle_out(b, Q[k]))
        run.check_metadata()
    finally:
        run.close()


def test_f32_output_of_bf16_cache():
    case = wl("outf32", 2, 8, 2, 128, "bf16", 16, (100, 400), 2, 0.5, 24)
    run = Run(case)
    try:
        run.prefill()
        for step in range(2):
            out, Q = run.decode_step(step, out_dtype=torch.float32)
            torch.cuda.synchronize()
            assert out.dtype == torch.float32
            for b in range(case.batch):
                compare(out[b], run.oracle_out(b, Q[b]), max_abs=5e-3, mean_abs=5e-4)
    finally:
        run.close()


def test_sequence_reset_returns_pages_in_order():
    case = wl("reset", 3, 8, 2, 64, "bf16", 16, (50, 300), 2, 0.5, 25)
    run = Run(case)
    try:
        run.prefill()
        run.decode_step(0)
        run.cache.reset_seq(1)
        assert run.sim.reset_seq(1) == 0
        run.seen[1] = 0
        run._blk.pop(1, None)
        run.check_metadata()
        run.ctx[1] = 120
        run.prefill(chunk=50, seqs=[1])
        run.check_metadata()
        out, Q = run.decode_step(1)
        torch.cuda.synchronize()
        for b in range(case.batch):
            compare(out[b], run.oracle_out(b, Q[b]))
        run.check_metadata()
    finally:
        run.close()


def test_pool_exhaustion_latches_and_poisons():
    case = wl("exhaust", 1, 4, 1, 64, "bf16", 16, (64, 64), 0, 0.0, 26)
    run = Run(case, max_pages=4, check_sim=False)
    try:
        run.prefill()                   # 64 tokens, all kept: exactly 4 pages
        assert run.cache.status() == _native.DMS_OK
        run.decode_step(0)              # needs a 5th page
        assert run.cache.status() == _native.DMS_ERR_POOL_EXHAUSTED
        with pytest.raises(_native.DmsError) as e:
            run.decode_step(1)
        assert e.value.code == _native.DMS_ERR_POISONED
        run.cache.reset()
        assert run.cache.status() == _native.DMS_OK
        snap = run.cache.snapshot()
        assert snap["free_count"] == 4 and snap["n"].sum() == 0
    finally:
        run.close()


def test_bulk_pool_exhaustion_and_bad_seq():
    case = wl("bulk-exhaust", 2, 4, 1, 64, "bf16", 16, (100, 100), 0, 0.0, 27)
    run = Run(case, max_pages=8, check_sim=False)
    try:
        run.prefill()                   # 2 x 100 tokens need 14 pages > 8
        assert run.cache.status() == _native.DMS_ERR_POOL_EXHAUSTED
        run.cache.reset()
        ids = torch.tensor([5], dtype=torch.int32, device="cuda")   # max_seqs is 2
        k = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device="cuda")
        run.cache.append(ids, k, k, torch.zeros(1, 1, dtype=torch.uint8, device="cuda"))
        assert run.cache.status() == _native.DMS_ERR_BAD_SEQ
    finally:
        run.close()


def test_host_argument_checks():
    case = wl("args", 1, 4, 1, 64, "bf16", 16, (10, 10), 0, 0.5, 28)
    run = Run(case, check_sim=False)
    try:
        ids = torch.tensor([0], dtype=torch.int32, device="cuda")
        q = torch.zeros(1, 12, 64, dtype=torch.bfloat16, device="cuda")   # g = 12 > 8
        with pytest.raises(_native.DmsError) as e:
            run.cache.decode_attention(ids, q)
        assert e.value.code == _native.DMS_ERR_INVALID
        k = torch.zeros(2, 1, 64, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(_native.DmsError):   # 2 rows for 1 sequence without cu_tokens
            run.cache.append(ids, k, k, torch.zeros(2, 1, dtype=torch.uint8, device="cuda"))
    finally:
        run.close()
    from learned_kv_cache_decode_b200 import DmsCache
    for bad in (dict(head_dim=96), dict(window=0), dict(max_pages=0)):
        args = dict(max_seqs=1, num_kv_heads=1, head_dim=64, window=4, max_pages=4, max_pages_per_stream=4)
        args.update(bad)
        with pytest.raises(_native.DmsError):
            DmsCache(**args)


# ---------------------------------------------------------------------------
# dms_decode_step: append and attention fused into one launch


@pytest.mark.parametrize("case", CASES, ids=[c.name for c in CASES])
def test_small_cases_fused_step(case):
    """The fused step against the oracle: metadata bit for bit, outputs within tolerance."""
    for kern in kernels_for(case):
        run = Run(case, attn_kernel=kern)
        try:
            run.prefill(chunk=97)
            run.check_metadata()
            for step in range(case.decode_steps):
                out, Q = run.decode_step(step, fused=True)
                torch.cuda.synchronize()
                for b in range(case.batch):
                    ref = run.oracle_out(b, Q[b])
                    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
                    compare(out[b], ref, **tol)
                run.check_metadata()
            assert run.cache.status() == _native.DMS_OK
        finally:
            run.close()


def test_fused_step_equals_two_launches():
    """Same inputs through dms_decode_step and through dms_append + dms_decode_attention:
    identical bookkeeping and pool rows, outputs equal to fp32 rounding order."""
    case = wl("fused-vs-two", 4, 28, 4, 128, "bf16", 24, (1, 800), 40, 0.7, 31)
    a, b = Run(case), Run(case, check_sim=False)
    try:
        a.prefill(chunk=200)
        b.prefill(chunk=200)
        for step in range(case.decode_steps):
            oa, _ = a.decode_step(step)
            ob, _ = b.decode_step(step, fused=True)
            torch.cuda.synchronize()
            diff = (oa.float() - ob.float()).abs()
            assert float(diff.max()) <= 1e-2 and float(diff.mean()) <= 1e-3
        sa, sb = a.cache.snapshot(), b.cache.snapshot()
        for k in ("n", "pos", "n_pages", "page_table", "free_list"):
            np.testing.assert_array_equal(sa[k], sb[k], err_msg=k)
        assert sa["free_count"] == sb["free_count"]
        for st in range(case.streams):
            n = int(sa["n"][st])
            if n:
                ka, va = a.cache.gather_kv(st // case.num_kv_heads, st % case.num_kv_heads, n)
                kb, vb = b.cache.gather_kv(st // case.num_kv_heads, st % case.num_kv_heads, n)
                assert torch.equal(ka, kb) and torch.equal(va, vb)
        assert a.cache.status() == _native.DMS_OK and b.cache.status() == _native.DMS_OK
    finally:
        a.close()
        b.close()


def test_fused_step_pool_exhaustion_matches_two_launches():
    """A pool too small for this step's page pops: both paths latch POOL_EXHAUSTED and
    leave the same bookkeeping (streams that needed a page unchanged, the others appended)."""
    case = wl("fused-exhaust", 3, 6, 2, 64, "bf16", 8, (30, 30), 4, 0.0, 32)
    ctx = W.contexts(case)
    need = int(sum(-(-int(c) // 16) for c in ctx)) * case.num_kv_heads   # prompt pages, all kept
    snaps, status = [], []
    for fused in (False, True):
        run = Run(case, max_pages=need + 1, check_sim=False)
        try:
            run.prefill(chunk=64)
            for step in range(3):   # streams reach 32 tokens: every stream needs a page at once
                run.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            status.append(run.cache.status())
            snaps.append(run.cache.snapshot())
        finally:
            run.close()
    assert status == [_native.DMS_ERR_POOL_EXHAUSTED] * 2
    for k in ("n", "pos", "n_pages", "free_list"):
        np.testing.assert_array_equal(snaps[0][k], snaps[1][k], err_msg=k)
    assert snaps[0]["free_count"] == snaps[1]["free_count"]


def test_fused_step_bad_seq_latches():
    case = wl("fused-badseq", 2, 4, 1, 64, "bf16", 8, (20, 40), 1, 0.5, 33)
    run = Run(case, check_sim=False)
    try:
        run.prefill(chunk=64)
        d = lambda x: torch.zeros(x, dtype=torch.bfloat16, device="cuda")
        ids = torch.tensor([0, 7], dtype=torch.int32, device="cuda")   # 7 >= max_seqs
        run.cache.decode_step(ids, d((2, 1, 64)), d((2, 1, 64)), torch.zeros((2, 1), dtype=torch.uint8,
                              device="cuda"), d((2, 4, 64)))
        torch.cuda.synchronize()
        assert run.cache.status() == _native.DMS_ERR_BAD_SEQ
    finally:
        run.close()


SCHEDULE_CASES = [
    wl("schedule-bf16-g7-d128", 6, 14, 2, 128, "bf16", 8, (1, 500), 0, 0.6, 34),
    wl("schedule-bf16-g4-d64-w1", 6, 8, 2, 64, "bf16", 1, (10, 300), 0, 0.5, 35),
    wl("schedule-f32-g4-d64", 5, 8, 2, 64, "f32", 24, (1, 400), 0, 0.5, 36),
]


@pytest.mark.parametrize("case", SCHEDULE_CASES, ids=[c.name for c in SCHEDULE_CASES])
@pytest.mark.parametrize("caches", [1, 2], ids=["one_cache", "two_caches_interleaved"])
def test_fused_step_schedule_follows_every_change(case, caches):
    """A fused step leaves the next one its schedule (counts, positions, leaving slots,
    page lists). Drive it through every way that schedule can stop matching: the same
    streams again, a permuted order, a prefix subset, a superset, a two-launch step in
    between, a sequence restart, and back. Metadata bit for bit and every output against
    the oracle, at every step.

    With two caches stepped in turn on one stream, the kernel before each fused step is
    the other cache's, so the step plans from the schedule and issues its first copies
    before its dependency wait, and checks the guess against the seq ids after it (a
    changed stream list takes the fallback: drain, reset the stage barriers, re-plan)."""
    B = case.batch
    perm = [3, 1, 0, 4, 2] + list(range(5, B))
    plan = ([("fused", list(range(B)))] * 4 + [("fused", perm)] * 2 + [("fused", perm[:3])] +
            [("fused", perm)] * 2 + [("two", list(range(B)))] + [("fused", list(range(B)))] * 3 +
            [("reset", 2)] + [("fused", list(range(B)))] * 3 + [("fused", list(range(B))[::-1])] * 2)
    runs = [Run(case, steps=len(plan)) for _ in range(caches)]
    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
    try:
        for run in runs:
            run.prefill(chunk=97)
            run.check_metadata()
        for step, (kind, arg) in enumerate(plan):
            for run in runs:
                if kind == "reset":
                    run.cache.reset_seq(arg)
                    assert run.sim.reset_seq(arg) == 0
                    run.seen[arg] = 0
                    run._blk.pop(arg, None)
                    run.prefill(chunk=97, seqs=[arg])
                    continue
                out, Q = run.decode_step(step, seqs=arg, fused=kind == "fused")
                torch.cuda.synchronize()
                for j, b in enumerate(arg):
                    try:
                        compare(out[j], run.oracle_out(b, Q[j]), **tol)
                    except AssertionError as e:
                        raise AssertionError(f"step {step} ({kind} {arg}), sequence {b}: {e}") from None
            for run in runs:
                run.check_metadata()
        for run in runs:
            assert run.cache.status() == _native.DMS_OK
    finally:
        for run in runs:
            run.close()


SWEEP_WINDOWS = [1, 2, 16, 32, 64, 128, 256]


@pytest.mark.parametrize("w", SWEEP_WINDOWS)
@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
def test_window_sweep(w, fused):
    """The delayed-eviction window swept from immediate eviction (w = 1: a marked token is
    attended by its own step's query only, the plainest reading of the paper's
    immediate-eviction ablation, section 5.3 and Fig. 5) to
    256, on one workload shape, through both decode paths: metadata bit for bit, every
    output against the oracle."""
    case = wl(f"sweep-w{w}", 3, 21, 3, 128, "bf16", w, (300, 900), 6, 0.7, 42)
    run = Run(case)
    try:
        run.prefill(chunk=257)
        run.check_metadata()
        for step in range(case.decode_steps):
            out, Q = run.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            for b in range(case.batch):
                compare(out[b], run.oracle_out(b, Q[b]))
        run.check_metadata()
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


@pytest.mark.parametrize("batch", [256, 257], ids=["1024_streams_fused", "1028_streams_two_launches"])
def test_decode_step_at_the_stream_limit_and_past_it(batch):
    """dms_decode_step at the fused kernel's limit of 1024 streams (256 sequences x 4 KV
    heads) and just past it, where the call issues the two launches instead: metadata bit
    for bit and every sequence's output against the oracle at every step."""
    case = wl(f"limit-{batch}", batch, 8, 4, 64, "bf16", 8, (10, 60), 3, 0.6, 45)
    run = Run(case)
    try:
        run.prefill(chunk=64)
        run.check_metadata()
        for step in range(case.decode_steps):
            before = run.cache.launches()
            out, Q = run.decode_step(step, fused=True)
            launched = run.cache.launches() - before
            assert launched == 1 if batch * case.num_kv_heads <= 1024 else launched >= 2, launched
            torch.cuda.synchronize()
            for b in range(batch):
                compare(out[b], run.oracle_out(b, Q[b]))
            run.check_metadata()
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


def test_fused_step_after_another_caches_stats_kernel():
    """Fused steps on cache A with a dms_stats call on cache B between them. The stats
    kernel lets the next kernel start at once, so A's previous step may still be running
    when the next one starts; the host leaves stats out of its per-stream record, so the
    record still names A and the step does not read A's state before its wait.
    Metadata and every output against the oracle."""
    case = wl("after-stats-bf16-g7-d128", 4, 14, 2, 128, "bf16", 8, (40, 500), 12, 0.6, 40)
    a, b = Run(case), Run(case)
    try:
        a.prefill(chunk=97)
        b.prefill(chunk=97)
        for step in range(case.decode_steps):
            out, Q = a.decode_step(step, fused=True)
            b.cache.stats()
            torch.cuda.synchronize()
            for j in range(case.batch):
                compare(out[j], a.oracle_out(j, Q[j]))
        a.check_metadata()
        assert a.cache.status() == _native.DMS_OK and b.cache.status() == _native.DMS_OK
    finally:
        a.close()
        b.close()


GUESS_CASES = [
    wl("guess-bf16-g7-d128", 6, 14, 2, 128, "bf16", 8, (1, 500), 0, 0.6, 38),
    wl("guess-f32-g4-d64", 5, 8, 2, 64, "f32", 24, (1, 400), 0, 0.5, 39),
]


@pytest.mark.parametrize("case", GUESS_CASES, ids=[c.name for c in GUESS_CASES])
def test_attention_alone_guess_follows_every_change(case):
    """dms_decode_attention on two caches, back to back after all of a step's appends:
    the kernel before each attention launch is the other cache's, so the launch guesses
    its stream list from the previous attention call on its cache, plans from the cache
    state and starts its first copies before its dependency wait, then checks the guess
    against the seq ids. The attention lists change from call to call (the same, a
    permutation, a subset, a superset, twice on the same state); every output against
    the oracle."""
    B = case.batch
    every = list(range(B))
    perm = [3, 1, 0, 4, 2] + list(range(5, B))
    lists = [[every, every], [every], [perm], [perm, perm], [perm[:3]], [every, every[::-1]], [every], [every]]
    runs = [Run(case, steps=len(lists)) for _ in range(2)]
    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
    try:
        for run in runs:
            run.prefill(chunk=97)
        for step, calls in enumerate(lists):
            for run in runs:   # one token for every sequence of both caches first
                K, V, A, _ = run.decode_inputs(step, every)
                run.cache.append(torch.tensor(every, dtype=torch.int32, device="cuda"), to_device(K, case),
                                 to_device(V, case), torch.from_numpy(A).cuda())
                assert run.sim.append(every, [1] * B, A)[0] == 0
                for b in every:
                    run.seen[b] += 1
            for seqs in calls:   # then the attention calls, alternating between the caches
                Qall = W.query(case, step)
                outs = [run.cache.decode_attention(torch.tensor(seqs, dtype=torch.int32, device="cuda"),
                                                   to_device(Qall[seqs], case), scale=run.scale) for run in runs]
                torch.cuda.synchronize()
                for run, out in zip(runs, outs):
                    for j, b in enumerate(seqs):
                        compare(out[j], run.oracle_out(b, Qall[b]), **tol)
        for run in runs:
            run.check_metadata()
            assert run.cache.status() == _native.DMS_OK
    finally:
        for run in runs:
            run.close()


def test_decode_step_captured_in_a_cuda_graph_replays_step_after_step():
    """dms_decode_step captured into a CUDA graph (issued as dms_append +
    dms_decode_attention under capture), replayed once per decode step with the
    step's inputs copied into the captured buffers: metadata bit for bit and every
    output against the oracle."""
    case = wl("graph-bf16-g7-d128", 3, 21, 3, 128, "bf16", 16, (40, 600), 6, 0.6, 37)
    run = Run(case)
    try:
        run.prefill(chunk=97)
        seqs = list(range(case.batch))
        K, V, A, Q = run.decode_inputs(0, seqs)
        ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
        dK, dV, dQ = to_device(K, case), to_device(V, case), to_device(Q, case)
        dA = torch.from_numpy(A).cuda()
        out = torch.empty_like(dQ)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run.cache.decode_step(ids, dK, dV, dA, dQ, scale=run.scale, out=out)
        # capture only records the launches: the cache is unchanged so far
        run.check_metadata()
        for step in range(case.decode_steps):
            K, V, A, Q = run.decode_inputs(step, seqs)
            dK.copy_(to_device(K, case))
            dV.copy_(to_device(V, case))
            dA.copy_(torch.from_numpy(A))
            dQ.copy_(to_device(Q, case))
            g.replay()
            torch.cuda.synchronize()
            rc, _ = run.sim.append(seqs, [1] * len(seqs), A)
            assert rc == 0
            for b in seqs:
                run.seen[b] += 1
            for b in seqs:
                compare(out[b], run.oracle_out(b, Q[b]))
            run.check_metadata()
        assert run.cache.status() == _native.DMS_OK
        del g
    finally:
        run.close()


def test_attention_of_two_caches_captured_in_a_graph_between_eager_calls():
    """dms_decode_attention on two caches captured into one CUDA graph, replayed once
    per step after eager appends, with eager attention calls on the same stream between
    replays. Launches into a capturing stream are neither recorded nor started early, so
    the eager calls' early starts see only what really ran. Every output against the
    oracle."""
    case = wl("graph-two-caches", 4, 14, 2, 128, "bf16", 8, (40, 500), 6, 0.6, 41)
    runs = [Run(case), Run(case)]
    B = case.batch
    every = list(range(B))
    ids = torch.tensor(every, dtype=torch.int32, device="cuda")
    try:
        for run in runs:
            run.prefill(chunk=97)
        dQ = [torch.empty((B, case.num_q_heads, case.head_dim), dtype=torch.bfloat16, device="cuda")
              for _ in runs]
        outs = [torch.empty_like(q) for q in dQ]
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for run, q, o in zip(runs, dQ, outs):
                run.cache.decode_attention(ids, q, scale=run.scale, out=o)
        for step in range(case.decode_steps):
            Q = W.query(case, step)
            for run, q in zip(runs, dQ):
                K, V, A, _ = run.decode_inputs(step, every)
                run.cache.append(ids, to_device(K, case), to_device(V, case), torch.from_numpy(A).cuda())
                assert run.sim.append(every, [1] * B, A)[0] == 0
                for b in every:
                    run.seen[b] += 1
                q.copy_(to_device(Q, case))
            g.replay()
            eager = [run.cache.decode_attention(ids, to_device(Q, case), scale=run.scale) for run in runs]
            torch.cuda.synchronize()
            for run, o, e in zip(runs, outs, eager):
                for b in every:
                    ref = run.oracle_out(b, Q[b])
                    compare(o[b], ref)
                    compare(e[b], ref)
        for run in runs:
            run.check_metadata()
            assert run.cache.status() == _native.DMS_OK
        del g
    finally:
        for run in runs:
            run.close()


def test_bounded_waits_give_up_latch_timeout_and_reset_recovers():
    """Failure detection without a GPU fault. The library's two bounded waits run on
    conditions that never come true: a flag nothing sets, and an mbarrier phase whose
    bytes never arrive. Each gives up after about a second and latches DMS_ERR_TIMEOUT.
    The cache is then poisoned; dms_cache_reset brings it back, and the same cache (and
    context) decodes correctly again."""
    import oracle
    case = wl("selftest", 2, 8, 2, 64, "bf16", 16, (20, 300), 3, 0.5, 44)
    run = Run(case)
    try:
        run.prefill(chunk=64)
        t = run.cache.selftest_bounded_waits()
        torch.cuda.synchronize()
        assert t.cpu().tolist() == [1, 1]
        assert run.cache.status() == _native.DMS_ERR_TIMEOUT
        with pytest.raises(_native.DmsError) as err:
            run.cache.decode_attention(torch.tensor([0], dtype=torch.int32, device="cuda"),
                                       torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda"))
        assert err.value.code == _native.DMS_ERR_POISONED
        run.cache.reset()
        assert run.cache.status() == _native.DMS_OK
        # a fresh start on the same cache, checked against a fresh oracle simulator
        cfg = run.cache.cfg
        run.sim.close()
        run.sim = oracle.Sim(case.batch, case.num_kv_heads, case.window, cfg.max_pages, cfg.max_pages_per_stream)
        run.seen[:] = 0
        run._blk.clear()
        run.prefill(chunk=64)
        run.check_metadata()
        for step in range(case.decode_steps):
            out, Q = run.decode_step(step, fused=True)
            torch.cuda.synchronize()
            for b in range(case.batch):
                compare(out[b], run.oracle_out(b, Q[b]))
        run.check_metadata()
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


# ---------------------------------------------------------------------------
# alpha read from a designated key channel (dms_append_keyed, dms_decode_step_keyed)

KEYED = [
    (wl("keyed-bf16-g7-d128", 3, 21, 3, 128, "bf16", 16, (1, 700), 6, 0.5, 41), 5),
    (wl("keyed-bf16-g4-d64-w1", 2, 8, 2, 64, "bf16", 1, (20, 300), 5, 0.5, 42), 63),
    (wl("keyed-f32-g4-d64", 2, 8, 2, 64, "f32", 24, (1, 400), 5, 0.5, 43), 0),
]


@pytest.mark.parametrize("case,channel", KEYED, ids=[c.name for c, _ in KEYED])
@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
def test_alpha_from_key_channel(case, channel, fused):
    """The library reads alpha from the sign of key channel `channel` (prefill and every
    decode step); the oracle gets the same bits from oracle.alpha_from_keys. Metadata bit
    for bit, outputs within tolerance."""
    run = Run(case, alpha_channel=channel)
    try:
        run.prefill(chunk=97)
        run.check_metadata()
        for step in range(case.decode_steps):
            out, Q = run.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            for b in range(case.batch):
                tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
                compare(out[b], run.oracle_out(b, Q[b]), **tol)
            run.check_metadata()
        snap = run.sim.snapshot()
        assert 0 < int(snap["n"].sum()) < int(run.seen.sum()) * case.num_kv_heads   # some tokens did leave
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


def test_keyed_entry_points_reject_a_channel_outside_head_dim():
    case = wl("keyed-bad", 1, 2, 1, 64, "bf16", 8, (10, 10), 1, 0.5, 44)
    run = Run(case, check_sim=False)
    try:
        ids = torch.zeros(1, dtype=torch.int32, device="cuda")
        K = torch.zeros((1, 1, 64), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(_native.DmsError) as e:
            run.cache.append(ids, K, K, None, alpha_channel=64)
        assert e.value.code == _native.DMS_ERR_INVALID
        with pytest.raises(_native.DmsError) as e:
            run.cache.decode_step(ids, K, K, None, torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda"),
                                  alpha_channel=-1 + 65)
        assert e.value.code == _native.DMS_ERR_INVALID
    finally:
        run.close()


# ---------------------------------------------------------------------------
# alpha read from a designated query channel (dms_decode_step_qkeyed, dms_alpha_from_logit)

QKEYED = [
    (wl("qkeyed-bf16-g7-d128", 3, 21, 3, 128, "bf16", 16, (1, 700), 6, 0.5, 46), (6, 5)),
    (wl("qkeyed-bf16-g4-d64-w1", 2, 8, 2, 64, "bf16", 1, (20, 300), 5, 0.5, 47), (0, 63)),
    (wl("qkeyed-f32-g4-d64", 2, 8, 2, 64, "f32", 4, (1, 400), 6, 0.5, 48), (3, 0)),
]


@pytest.mark.parametrize("case,pick", QKEYED, ids=[c.name for c, _ in QKEYED])
@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
def test_alpha_from_query_channel(case, pick, fused):
    """Every decode token's alpha comes from channel c of query head j of its KV head's
    group in the step's queries: fused (dms_decode_step_qkeyed) or dms_alpha_from_logit
    (checked bit for bit against oracle.alpha_from_queries) then dms_append. Metadata bit
    for bit, outputs within tolerance of the oracle fed the same bits."""
    run = Run(case, alpha_query=pick)
    tol = dict(max_abs=1e-4, mean_abs=1e-5) if case.dtype == "f32" else {}
    try:
        run.prefill(chunk=97)
        for step in range(case.decode_steps):
            out, Q = run.decode_step(step, fused=fused)
            torch.cuda.synchronize()
            for b in range(case.batch):
                compare(out[b], run.oracle_out(b, Q[b]), **tol)
            run.check_metadata()
        marks = sum(int(a.sum()) for a in run.dec_alpha.values())
        assert 0 < marks < len(run.dec_alpha) * case.num_kv_heads   # both decisions occur
        assert run.cache.status() == _native.DMS_OK
    finally:
        run.close()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_alpha_from_logit_special_values_bit_exact(dtype):
    """dms_alpha_from_logit on keys (one head per KV head) and on queries (a group of
    g), on random logits mixed with +-0, subnormals, +-inf and NaN: bit for bit equal to
    the oracle's sign rule."""
    gen = np.random.default_rng(49)
    rows, hkv, g, d = 257, 3, 4, 64
    X = gen.standard_normal((rows, hkv * g, d)).astype(np.float32)
    special = np.array([0.0, -0.0, 1e-40, -1e-40, np.inf, -np.inf, np.nan, 1.0, -1.0], dtype=np.float32)
    X[:, :, 7] = special[gen.integers(0, len(special), size=(rows, hkv * g))]
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    Xt = torch.from_numpy(X).to(tdt)
    Xh = Xt.numpy() if dtype == "f32" else Xt.view(torch.int16).numpy().view(np.uint16)
    Xd = Xt.cuda()
    for head, ch in ((0, 7), (3, 7), (2, 11)):
        got = alpha_from_logit(Xd, hkv, ch, head).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.alpha_from_queries(Xh, hkv, head, ch))
    K = Xd[:, :hkv].contiguous()   # keys: one head per KV head
    got = alpha_from_logit(K, hkv, 7).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.alpha_from_keys(Xh[:, :hkv], 7))
