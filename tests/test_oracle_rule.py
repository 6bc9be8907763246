"""Pins for the oracle's retention rule and slot-pool simulator (CPU only).

What pins what:
  * hand-derived traces (tests/golden/delayed_eviction_traces.txt) fix the
    window bound and the slot-reuse order;
  * the closed form n_s = (s+1) - #{j <= s-w : alpha_j = 1} and the dense
    invariant (slots [0, n) occupied, ceil(n/16) pages) hold for random runs;
  * brute force over every alpha pattern of length <= 12 compares the
    simulator (ring-free lookup, slot reuse) with the visibility definition;
  * a hand-derived free-stack trace (tests/golden/page_pops.txt) fixes the
    page-pop and reset order;
  * hand-encoded logits (tests/golden/alpha_from_keys.txt) fix the sign rule
    that reads alpha from a designated key channel (zero and NaN keep).
"""
import os
import itertools

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _parse_traces():
    traces, cur = [], None
    for line in open(os.path.join(GOLD, "delayed_eviction_traces.txt")):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, _, rest = line.partition(" ")
        if key == "trace":
            cur = {"name": rest, "visible": {}}
            traces.append(cur)
        elif key == "window":
            cur["w"] = int(rest)
        elif key == "alpha":
            cur["alpha"] = [int(x) for x in rest.split()]
        elif key == "visible":
            s, _, pos = rest.partition(":")
            cur["visible"][int(s)] = [int(x) for x in pos.split()]
        elif key == "slots":
            cur["slots"] = [int(x) for x in rest.split()]
        elif key == "final":
            cur["final"] = [int(x) for x in rest.split()]
    return traces


TRACES = _parse_traces()


@pytest.mark.parametrize("tr", TRACES, ids=[t["name"] for t in TRACES])
def test_golden_visible_sets(tr):
    a, w = tr["alpha"], tr["w"]
    assert len(tr["visible"]) == len(a)
    for s, expect in tr["visible"].items():
        assert oracle.visible_positions(a, s, w) == expect
        got_c = [j for j in range(s + 1) if oracle.lib().dmso_visible(s, j, a[j], w)]
        assert got_c == expect
        assert oracle.retained_count_closed_form(a, s, w) == len(expect)


@pytest.mark.parametrize("tr", TRACES, ids=[t["name"] for t in TRACES])
def test_golden_slots(tr):
    a, w = tr["alpha"], tr["w"]
    sim = oracle.Sim(1, 1, w, max_pages=4, max_pages_per_stream=4)
    logical = []
    for s, bit in enumerate(a):
        rc, phys = sim.append([0], [1], np.array([[bit]], dtype=np.uint8), want_slots=True)
        assert rc == 0
        snap = sim.snapshot()
        page = int(phys[0, 0]) // 16
        logical_page = list(snap["page_table"][0]).index(page)
        logical.append(logical_page * 16 + int(phys[0, 0]) % 16)
        assert sorted(sim.retained(0).tolist()) == tr["visible"][s]
    assert logical == tr["slots"]
    assert sim.retained(0).tolist() == tr["final"]


def test_visible_rule_edges():
    vis = oracle.lib().dmso_visible
    assert vis(5, 6, 0, 3) == 0          # future position
    assert vis(5, -1, 0, 3) == 0
    assert vis(5, 5, 1, 1) == 1          # own token always visible (w >= 1)
    assert vis(5, 4, 1, 1) == 0
    assert vis(5, 3, 1, 3) == 1          # age 2 < 3
    assert vis(5, 2, 1, 3) == 0          # age 3 == w -> gone
    assert vis(10**6, 0, 0, 1) == 1      # kept tokens stay forever


def test_c_and_python_rule_agree():
    rng = np.random.default_rng(7)
    for _ in range(200):
        T = int(rng.integers(1, 60))
        w = int(rng.integers(1, 70))
        a = rng.integers(0, 2, T).tolist()
        s = T - 1
        py = oracle.visible_positions(a, s, w)
        c = [j for j in range(T) if oracle.lib().dmso_visible(s, j, a[j], w)]
        assert py == c


def _run_stream(alpha_seq, w, page_size, check_each_step=True):
    pages = len(alpha_seq) // page_size + 1
    sim = oracle.Sim(1, 1, w, max_pages=pages, max_pages_per_stream=pages, page_size=page_size)
    for s, bit in enumerate(alpha_seq):
        rc, _ = sim.append([0], [1], np.array([[bit]], dtype=np.uint8))
        assert rc == 0
        if check_each_step or s == len(alpha_seq) - 1:
            ret = sim.retained(0).tolist()
            vis = oracle.visible_positions(alpha_seq, s, w)
            assert sorted(ret) == vis, (alpha_seq, w, s)
            assert len(set(ret)) == len(ret)
            assert len(ret) == oracle.retained_count_closed_form(alpha_seq, s, w)
            snap = sim.snapshot()
            assert snap["n_pages"][0] == -(-len(ret) // page_size)
    return sim


@pytest.mark.parametrize("T", [1, 2, 5, 8, 10])
def test_brute_force_all_patterns(T):
    for w in sorted({1, 2, 3, 5, T}):
        for bits in itertools.product((0, 1), repeat=T):
            _run_stream(list(bits), w, page_size=4)


def test_brute_force_length12():
    T = 12
    for w in (1, 3, 5, 12):
        for bits in itertools.product((0, 1), repeat=T):
            _run_stream(list(bits), w, page_size=4, check_each_step=False)


def test_bulk_append_equals_token_by_token():
    rng = np.random.default_rng(3)
    for w in (1, 4, 16, 37):
        a = rng.integers(0, 2, (300, 2)).astype(np.uint8)
        s1 = oracle.Sim(1, 2, w, 64, 64)
        for t in range(300):
            assert s1.append([0], [1], a[t:t + 1])[0] == 0
        s2 = oracle.Sim(1, 2, w, 64, 64)
        assert s2.append([0], [120], a[:120])[0] == 0
        assert s2.append([0], [180], a[120:])[0] == 0
        x, y = s1.snapshot(), s2.snapshot()
        for k in ("n", "pos", "n_pages"):
            np.testing.assert_array_equal(x[k], y[k])
        # page ids differ only in pop order across streams; the retained sets match
        for st in range(2):
            assert s1.retained(st).tolist() == s2.retained(st).tolist()


def test_closed_form_random_long():
    rng = np.random.default_rng(11)
    for w, p in ((256, 0.875), (16, 0.5), (1, 0.3)):
        a = (rng.random(3000) < p).astype(np.uint8)
        sim = _run_stream(a.tolist(), w, page_size=16, check_each_step=False)
        assert sim.snapshot()["n"][0] == oracle.retained_count_closed_form(a, 2999, w)


def test_all_marked_keeps_exactly_w():
    for w in (1, 2, 7, 16):
        sim = _run_stream([1] * 50, w, page_size=16, check_each_step=False)
        assert sorted(sim.retained(0).tolist()) == list(range(50 - w, 50))


def test_window_covers_context_keeps_all():
    rng = np.random.default_rng(5)
    a = rng.integers(0, 2, 40).tolist()
    sim = _run_stream(a, 40, page_size=16, check_each_step=False)
    assert sorted(sim.retained(0).tolist()) == list(range(40))


def test_golden_page_pops():
    sim = oracle.Sim(2, 2, 64, max_pages=16, max_pages_per_stream=8)
    for line in open(os.path.join(GOLD, "page_pops.txt")):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        f = line.split()
        if f[0] == "op":
            kw = dict(x.split("=") for x in f[2:])
            seq = int(kw["seq"])
            if f[1] == "append":
                t = int(kw["tokens"])
                assert sim.append([seq], [t], np.zeros((t, 2), np.uint8))[0] == 0
            else:
                assert sim.reset_seq(seq) == 0
        elif f[0] == "expect":
            st = int(f[1])
            pages = [int(x) for x in line.split(":")[1].split()]
            snap = sim.snapshot()
            assert snap["n_pages"][st] == len(pages)
            assert snap["page_table"][st][:len(pages)].tolist() == pages
        elif f[0] == "free_count":
            assert sim.snapshot()["free_count"] == int(f[1])


def test_pool_exhaustion_and_stream_capacity():
    sim = oracle.Sim(1, 1, 8, max_pages=2, max_pages_per_stream=8)
    assert sim.append([0], [32], np.zeros((32, 1), np.uint8))[0] == 0
    assert sim.append([0], [1], np.zeros((1, 1), np.uint8))[0] == 2   # pool exhausted
    sim2 = oracle.Sim(1, 1, 8, max_pages=8, max_pages_per_stream=1)
    assert sim2.append([0], [16], np.zeros((16, 1), np.uint8))[0] == 0
    assert sim2.append([0], [1], np.zeros((1, 1), np.uint8))[0] == 6


# ---------------------------------------------------------------------------
# alpha read from a designated key channel (the eviction logit)

def _golden_logits():
    rows = []
    for line in open(os.path.join(GOLD, "alpha_from_keys.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        dt, bits, want = line.split()
        rows.append((dt, int(bits, 16), int(want)))
    return rows


def test_golden_alpha_from_keys():
    rows = _golden_logits()
    assert len(rows) >= 10
    for dt, bits, want in rows:
        d = 8
        if dt == "bf16":
            K = np.zeros((1, 2, d), dtype=np.uint16)
            K[0, 1, 5] = bits
        else:
            K = np.zeros((1, 2, d), dtype=np.float32)
            K.view(np.uint32)[0, 1, 5] = bits
        a = oracle.alpha_from_keys(K, 5)
        assert a.shape == (1, 2) and a.dtype == np.uint8
        assert a[0, 1] == want, (dt, hex(bits))
        assert a[0, 0] == 0   # the other head's channel holds +0.0


def test_alpha_from_keys_reads_only_the_designated_channel():
    rng = np.random.default_rng(5)
    K = rng.standard_normal((50, 3, 16)).astype(np.float32)
    for c in (0, 7, 15):
        a = oracle.alpha_from_keys(K, c)
        K2 = K.copy()
        K2[..., [x for x in range(16) if x != c]] *= -1.0   # other channels do not matter
        np.testing.assert_array_equal(oracle.alpha_from_keys(K2, c), a)
        K3 = K.copy()
        K3[..., c] *= -1.0   # flipping the logit flips every non-zero decision
        np.testing.assert_array_equal(oracle.alpha_from_keys(K3, c), 1 - a)


def _golden_queries():
    q, picks = [], []
    for line in open(os.path.join(GOLD, "alpha_from_queries.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, *rest = line.split()
        if key == "q":
            q.append([float(x) for x in rest[1:]])
        elif key == "pick":
            picks.append((int(rest[0]), int(rest[1]), [int(rest[2]), int(rest[3])]))
    return np.array(q, dtype=np.float32), picks


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_golden_alpha_from_queries(dtype):
    """The hand-worked picks fix which query head of each group holds the logit
    (contiguous grouping: an interleaved one gives different bits for some picks)."""
    q, picks = _golden_queries()
    assert q.shape == (6, 4) and len(picks) >= 8
    Q = q[None]                                           # one token [1, Hq, d]
    if dtype == "bf16":
        Q = (Q.view(np.uint32) >> np.uint32(16)).astype(np.uint16)   # exact: every value fits bf16
    for head, ch, want in picks:
        a = oracle.alpha_from_queries(Q, 2, head, ch)
        assert a.shape == (1, 2) and a.dtype == np.uint8
        assert a[0].tolist() == want, (head, ch, a[0].tolist(), want)


def test_alpha_from_queries_is_the_key_rule_on_the_designated_heads():
    """With g = 1 the query rule is the key rule; with g > 1 it reads only the
    designated head of each group, whatever the other heads hold."""
    rng = np.random.default_rng(8)
    X = rng.standard_normal((40, 4, 16)).astype(np.float32)
    np.testing.assert_array_equal(oracle.alpha_from_queries(X, 4, 0, 9), oracle.alpha_from_keys(X, 9))
    Q = rng.standard_normal((40, 12, 16)).astype(np.float32)   # Hkv = 3, g = 4
    a = oracle.alpha_from_queries(Q, 3, 2, 5)
    Q2 = Q.copy()
    for k in range(3):
        for j in (0, 1, 3):
            Q2[:, 4 * k + j] = -Q2[:, 4 * k + j]   # the other heads of each group do not matter
    np.testing.assert_array_equal(oracle.alpha_from_queries(Q2, 3, 2, 5), a)
    Q3 = Q.copy()
    Q3[:, [2, 6, 10], 5] *= -1.0                   # flipping the designated logits flips every decision
    np.testing.assert_array_equal(oracle.alpha_from_queries(Q3, 3, 2, 5), 1 - a)
