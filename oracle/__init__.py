"""CPU oracle for the DMS decode path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package.
The product library never imports it and shares no code with it.

Two parts:

* ``libdms_oracle.so`` (plain C, fp64; see dms_oracle.h): the visibility
  rule, masked attention in definition form, and a sequential simulator of
  the slot-pool allocation policy.
* pure-Python helpers for tiny enumerations: ``visible_positions`` (the rule
  written out) and ``retained_count_closed_form``.

Source of the rule: "Inference-Time Hyper-Scaling with KV Cache
Compression" (paper summary), Key claims and Method, section 3.2: a token
marked for eviction at step t stays attendable until step t + w, and the
eviction decisions act as an additive attention mask. Reading adopted for
the bound: j is visible to the query at step s iff alpha_j == 0 or
s - j < w, so with every token marked the window holds exactly w tokens,
the current one included.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i, d, p = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.dmso_visible.argtypes = [ctypes.c_long, ctypes.c_long, i, i]
        L.dmso_visible.restype = i
        L.dmso_attention.argtypes = [i, i, i, i, p, p, p, p, d, p]
        L.dmso_attention.restype = None
        L.dmso_attention_batch.argtypes = [i, p, i, i, i, p, p, p, p, d, p]
        L.dmso_attention_batch.restype = i
        L.dmso_sim_create.argtypes = [i, i, i, i, i, i]
        L.dmso_sim_create.restype = p
        L.dmso_sim_destroy.argtypes = [p]
        L.dmso_sim_destroy.restype = None
        L.dmso_sim_append.argtypes = [p, i, p, p, p, p]
        L.dmso_sim_append.restype = i
        L.dmso_sim_reset_seq.argtypes = [p, i]
        L.dmso_sim_reset_seq.restype = i
        L.dmso_sim_snapshot.argtypes = [p, p, p, p, p, p, p, p]
        L.dmso_sim_snapshot.restype = None
        L.dmso_sim_retained.argtypes = [p, i, p]
        L.dmso_sim_retained.restype = i
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------------------
# Pure-Python statements of the rule (tiny inputs only)

def visible_positions(alpha_seq, s: int, window: int) -> list[int]:
    """Positions j <= s attendable at step s: alpha_j == 0 or s - j < w."""
    return [j for j in range(s + 1) if alpha_seq[j] == 0 or s - j < window]


def retained_count_closed_form(alpha_seq, s: int, window: int) -> int:
    """n_s = (s + 1) - #{ j <= s - w : alpha_j = 1 }: the tokens seen minus
    those marked at least w steps ago."""
    return (s + 1) - sum(1 for j in range(0, s - window + 1) if alpha_seq[j] == 1)


# ---------------------------------------------------------------------------
# Attention

def alpha_from_keys(K: np.ndarray, channel: int) -> np.ndarray:
    """Eviction decisions read from a designated key channel: uint8 [..., Hkv].

    Method section of the paper summary: one neuron of the K projection per head
    is repurposed to produce the eviction logit. At inference the token is
    marked iff that logit is > 0 (the plainest binarisation of the logit; the
    pages do not state one); zero and NaN keep it. K holds stored
    values: bf16 bits as uint16, or float32.
    """
    x = np.asarray(K)
    logit = (x[..., channel].astype(np.uint32) << np.uint32(16)).view(np.float32) if x.dtype == np.uint16 \
        else x[..., channel].astype(np.float32)
    return (logit > 0).astype(np.uint8)


def alpha_from_queries(Q: np.ndarray, num_kv_heads: int, head: int, channel: int) -> np.ndarray:
    """Eviction decisions read from a designated channel of one query head per KV
    head: uint8 [..., Hkv].

    Method section of the paper summary: the eviction logit may come from a
    neuron of the Q projection instead of the K one. The decision stays one per
    KV head, so one query head of each group is designated: query heads
    k*g .. k*g+g-1 belong to KV head k (contiguous GQA grouping) and ``head``
    picks k*g + head. The sign rule is that of alpha_from_keys. Q holds stored
    values [..., Hq, d]: bf16 bits as uint16, or float32.
    """
    x = np.asarray(Q)
    g = x.shape[-2] // num_kv_heads
    assert 0 <= head < g and g * num_kv_heads == x.shape[-2]
    rows = x[..., [k * g + head for k in range(num_kv_heads)], :]   # [..., Hkv, d]
    return alpha_from_keys(rows, channel)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, alpha_seq: np.ndarray,
              window: int, scale: float) -> np.ndarray:
    """Masked softmax attention of g query heads over one stream, fp64.

    q: [g, d]; K, V: [T, d] for positions 0..T-1 (query at T-1); alpha: [T].
    Returns [g, d] float64.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    a = np.ascontiguousarray(alpha_seq, dtype=np.uint8)
    g, d = q.shape
    T = K.shape[0]
    assert K.shape == (T, d) and V.shape == (T, d) and a.shape == (T,)
    out = np.zeros((g, d), dtype=np.float64)
    lib().dmso_attention(T, window, d, g, _ptr(q), _ptr(K), _ptr(V), _ptr(a),
                         float(scale), _ptr(out))
    return out


def decode_gqa(q: np.ndarray, K: np.ndarray, V: np.ndarray, alpha_seq: np.ndarray,
               window: int, scale: float) -> np.ndarray:
    """One decode step of one sequence with grouped-query attention.

    Query head h reads KV head h // g, g = Hq / Hkv (contiguous grouping, as
    in GQA, which the citation map of "Inference-Time Hyper-Scaling with KV
    Cache Compression" lists under "Builds on"). The eviction decision is per
    KV head, so all g query heads of a group see the same positions.

    q: [Hq, d]; K, V: [T, Hkv, d]; alpha: [T, Hkv]. Returns [Hq, d] float64.
    """
    hq, d = q.shape
    T, hkv, _ = K.shape
    g = hq // hkv
    out = np.empty((hq, d), dtype=np.float64)
    for k in range(hkv):
        out[k * g:(k + 1) * g] = attention(q[k * g:(k + 1) * g], K[:, k], V[:, k],
                                           alpha_seq[:, k], window, scale)
    return out


def attention_batch(items, window: int, scale: float):
    """Run attention for many streams in one call (OpenMP when available).

    items: list of (q [g,d], K [T,d], V [T,d], alpha [T]) float64/uint8 arrays.
    Returns (list of [g, d] outputs, threads used).
    """
    n = len(items)
    keep = []
    Ts = np.zeros(n, dtype=np.int32)
    arrs = {k: (ctypes.c_void_p * max(n, 1))() for k in ("q", "K", "V", "a", "o")}
    outs = []
    g = d = 0
    for i, (q, K, V, a) in enumerate(items):
        q = np.ascontiguousarray(q, dtype=np.float64)
        K = np.ascontiguousarray(K, dtype=np.float64)
        V = np.ascontiguousarray(V, dtype=np.float64)
        a = np.ascontiguousarray(a, dtype=np.uint8)
        g, d = q.shape
        o = np.zeros((g, d), dtype=np.float64)
        keep += [q, K, V, a]
        outs.append(o)
        Ts[i] = K.shape[0]
        arrs["q"][i], arrs["K"][i], arrs["V"][i] = _ptr(q), _ptr(K), _ptr(V)
        arrs["a"][i], arrs["o"][i] = _ptr(a), _ptr(o)
    threads = lib().dmso_attention_batch(
        n, _ptr(Ts), window, d, g, arrs["q"], arrs["K"], arrs["V"], arrs["a"],
        float(scale), arrs["o"])
    return outs, threads


# ---------------------------------------------------------------------------
# Slot-pool simulator

class Sim:
    """Sequential simulator of the slot pool (see dms_oracle.h)."""

    def __init__(self, max_seqs: int, num_kv_heads: int, window: int, max_pages: int,
                 max_pages_per_stream: int, page_size: int = 16):
        self.max_seqs, self.hkv, self.window = max_seqs, num_kv_heads, window
        self.max_pages, self.mps, self.page_size = max_pages, max_pages_per_stream, page_size
        self._h = lib().dmso_sim_create(max_seqs, num_kv_heads, window, page_size,
                                        max_pages, max_pages_per_stream)
        if not self._h:
            raise ValueError("invalid simulator configuration")

    def close(self) -> None:
        if self._h:
            lib().dmso_sim_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def append(self, seq_ids, counts, alpha: np.ndarray, want_slots: bool = False):
        """alpha: uint8 [sum(counts), Hkv] in call order. Returns (status, phys_slots|None)."""
        seq = np.ascontiguousarray(seq_ids, dtype=np.int32)
        cnt = np.ascontiguousarray(counts, dtype=np.int32)
        a = np.ascontiguousarray(alpha, dtype=np.uint8).reshape(-1, self.hkv)
        assert a.shape[0] == int(cnt.sum())
        slots = np.full(a.shape, -1, dtype=np.int32) if want_slots else None
        rc = lib().dmso_sim_append(self._h, len(seq), _ptr(seq), _ptr(cnt), _ptr(a),
                                   _ptr(slots) if want_slots else None)
        return rc, slots

    def reset_seq(self, seq_id: int) -> int:
        return lib().dmso_sim_reset_seq(self._h, seq_id)

    def snapshot(self) -> dict:
        S = self.max_seqs * self.hkv
        out = {
            "page_table": np.empty((S, self.mps), dtype=np.int32),
            "n_pages": np.empty(S, dtype=np.int32),
            "n": np.empty(S, dtype=np.int32),
            "pos": np.empty(S, dtype=np.int32),
            "slot_pos": np.empty(self.max_pages * self.page_size, dtype=np.int32),
            "free_list": np.empty(self.max_pages, dtype=np.int32),
            "free_count": np.empty(1, dtype=np.int32),
        }
        lib().dmso_sim_snapshot(self._h, *(_ptr(out[k]) for k in (
            "page_table", "n_pages", "n", "pos", "slot_pos", "free_list", "free_count")))
        out["free_count"] = int(out["free_count"][0])
        return out

    def retained(self, stream: int) -> np.ndarray:
        buf = np.empty(self.mps * self.page_size, dtype=np.int32)
        n = lib().dmso_sim_retained(self._h, stream, _ptr(buf))
        return buf[:n].copy()


def available() -> bool:
    try:
        lib()
        return True
    except (OSError, FileNotFoundError, ImportError):
        return False


__all__ = ["lib", "visible_positions", "retained_count_closed_form", "alpha_from_keys", "alpha_from_queries",
           "attention", "decode_gqa",
           "attention_batch", "Sim", "available"]
