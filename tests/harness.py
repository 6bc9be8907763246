"""Drive one workload through the CUDA path and through the CPU oracle.

Test infrastructure: imports both the library and the oracle (the two never
import each other). Inputs come from the seeded generators in
learned_kv_cache_decode_b200.workloads.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from learned_kv_cache_decode_b200 import DmsCache, alpha_from_logit
from learned_kv_cache_decode_b200 import workloads as W

MAX_ABS = 2e-2     # tolerance on bf16 inputs, max |gpu - oracle|
MEAN_ABS = 2e-3    # tolerance on bf16 inputs, mean |gpu - oracle|


def torch_dtype(wl: W.Workload) -> torch.dtype:
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def to_device(x: np.ndarray, wl: W.Workload, device="cuda") -> torch.Tensor:
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def pool_pages(wl: W.Workload, ctx: np.ndarray, steps: int, extra: int = 0) -> tuple[int, int]:
    """(max_pages, max_pages_per_stream) large enough for every alpha (no eviction at all)."""
    mps = int((ctx.max() + steps + extra) // 16 + 2)
    return wl.streams * mps, mps


class Run:
    """One workload on one cache plus its oracle simulator, call for call."""

    def __init__(self, wl: W.Workload, attn_kernel: str = "auto", steps: int | None = None,
                 max_pages: int | None = None, check_sim: bool = True, alpha_channel: int | None = None,
                 alpha_query: tuple[int, int] | None = None):
        """alpha_channel: the library reads every token's alpha from the sign of this key
        channel (dms_append_keyed / dms_decode_step_keyed); the oracle gets the same bits
        from oracle.alpha_from_keys.
        alpha_query = (head, channel): the decode tokens' alpha comes from that channel of
        that query head of each group in the step's queries (dms_decode_step_qkeyed, or
        dms_alpha_from_logit then dms_append); the oracle gets the same bits from
        oracle.alpha_from_queries. The prompt's alpha is the workload's."""
        self.wl = wl
        self.alpha_channel = alpha_channel
        self.alpha_query = alpha_query
        self.dec_alpha = {}   # (seq, position) -> alpha row of a decode token taken from the queries
        self.ctx = W.contexts(wl)
        self.steps = wl.decode_steps if steps is None else steps
        mp, mps = pool_pages(wl, self.ctx, self.steps)
        if max_pages is not None:
            mp = max_pages
        self.cache = DmsCache(wl.batch, wl.num_kv_heads, wl.head_dim, wl.window, mp, mps,
                              dtype=torch_dtype(wl), attn_kernel=attn_kernel)
        self.sim = oracle.Sim(wl.batch, wl.num_kv_heads, wl.window, mp, mps) if check_sim else None
        self.seen = np.zeros(wl.batch, dtype=np.int64)   # tokens appended per sequence
        self.scale = 1.0 / math.sqrt(wl.head_dim)
        self._blk = {}   # seq -> (first position, K, V, alpha) of pre-generated decode tokens

    # -- appends ---------------------------------------------------------
    def prefill(self, chunk: int = 4096, seqs=None) -> None:
        """Bulk-append every prompt in chunks of `chunk` tokens per sequence per call."""
        seqs = list(range(self.wl.batch)) if seqs is None else list(seqs)
        while True:
            ids, counts, Ks, Vs, As = [], [], [], [], []
            for b in seqs:
                left = int(self.ctx[b] - self.seen[b])
                if left <= 0:
                    continue
                t = min(chunk, left)
                K, V = W.kv(self.wl, b, int(self.seen[b]), t)
                ids.append(b)
                counts.append(t)
                Ks.append(K)
                Vs.append(V)
                As.append(self.alpha_of(b, int(self.seen[b]), t, K))
            if not ids:
                return
            self.append_bulk(ids, counts, np.concatenate(Ks), np.concatenate(Vs), np.concatenate(As))

    def alpha_of(self, b: int, start: int, count: int, K: np.ndarray | None = None) -> np.ndarray:
        """Eviction bits of positions [start, start+count) of sequence b."""
        if self.alpha_channel is None:
            return W.alpha(self.wl, b, start, count)
        if K is None:
            K, _ = W.kv(self.wl, b, start, count)
        return oracle.alpha_from_keys(K, self.alpha_channel)

    def append_bulk(self, ids, counts, K, V, A) -> None:
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        alpha = None if self.alpha_channel is not None else torch.from_numpy(np.ascontiguousarray(A)).cuda()
        self.cache.append(torch.tensor(ids, dtype=torch.int32, device="cuda"), to_device(K, self.wl),
                          to_device(V, self.wl), alpha, cu_tokens=torch.from_numpy(cu).cuda(),
                          alpha_channel=self.alpha_channel)
        if self.sim is not None:
            rc, _ = self.sim.append(ids, counts, A)
            assert rc == 0, rc
        for b, c in zip(ids, counts):
            self.seen[b] += c

    def _token(self, b: int, block: int = 256):
        pos = int(self.seen[b])
        e = self._blk.get(b)
        if e is None or not (e[0] <= pos < e[0] + len(e[3])):
            K, V = W.kv(self.wl, b, pos, block, threads=1)
            e = (pos, K, V, self.alpha_of(b, pos, block, K))
            self._blk[b] = e
        o = pos - e[0]
        return e[1][o], e[2][o], e[3][o]

    def decode_inputs(self, step: int, seqs):
        """K, V [B, Hkv, d], alpha [B, Hkv] of the next token of each sequence, and Q [B, Hq, d]."""
        toks = [self._token(b) for b in seqs]
        K = np.stack([t[0] for t in toks])
        V = np.stack([t[1] for t in toks])
        A = np.stack([t[2] for t in toks])
        Q = W.query(self.wl, step)[list(seqs)]
        if self.alpha_query is not None:
            A = oracle.alpha_from_queries(Q, self.wl.num_kv_heads, *self.alpha_query)
            for j, b in enumerate(seqs):
                self.dec_alpha[(b, int(self.seen[b]))] = A[j]
        return K, V, A, Q

    def decode_step(self, step: int, seqs=None, out_dtype=None, fused: bool = False):
        """Append one token per sequence and attend: two launches (dms_append then
        dms_decode_attention) or, with `fused`, one dms_decode_step."""
        seqs = list(range(self.wl.batch)) if seqs is None else list(seqs)
        K, V, A, Q = self.decode_inputs(step, seqs)
        ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
        dev_alpha = None if self.alpha_channel is not None else torch.from_numpy(A).cuda()
        if self.alpha_query is not None:
            head, channel = self.alpha_query
            dQ = to_device(Q, self.wl)
            if fused:
                out = self.cache.decode_step(ids, to_device(K, self.wl), to_device(V, self.wl), None, dQ,
                                             scale=self.scale, out_dtype=out_dtype, alpha_channel=channel,
                                             alpha_head=head)
            else:
                a_dev = alpha_from_logit(dQ, self.wl.num_kv_heads, channel, head)
                np.testing.assert_array_equal(a_dev.cpu().numpy(), A)   # the decisions, bit for bit
                self.cache.append(ids, to_device(K, self.wl), to_device(V, self.wl), a_dev)
                out = self.cache.decode_attention(ids, dQ, scale=self.scale, out_dtype=out_dtype)
            if self.sim is not None:
                rc, _ = self.sim.append(seqs, [1] * len(seqs), A)
                assert rc == 0, rc
            for b in seqs:
                self.seen[b] += 1
            return out, Q
        if fused:
            out = self.cache.decode_step(ids, to_device(K, self.wl), to_device(V, self.wl), dev_alpha,
                                         to_device(Q, self.wl), scale=self.scale, out_dtype=out_dtype,
                                         alpha_channel=self.alpha_channel)
            if self.sim is not None:
                rc, _ = self.sim.append(seqs, [1] * len(seqs), A)
                assert rc == 0, rc
            for b in seqs:
                self.seen[b] += 1
            return out, Q
        self.cache.append(ids, to_device(K, self.wl), to_device(V, self.wl), dev_alpha,
                          alpha_channel=self.alpha_channel)
        if self.sim is not None:
            rc, _ = self.sim.append(seqs, [1] * len(seqs), A)
            assert rc == 0, rc
        for b in seqs:
            self.seen[b] += 1
        out = self.cache.decode_attention(ids, to_device(Q, self.wl), scale=self.scale, out_dtype=out_dtype)
        return out, Q

    # -- oracle ----------------------------------------------------------
    def oracle_out(self, b: int, q: np.ndarray) -> np.ndarray:
        """Oracle output [Hq, d] for sequence b at its current last position."""
        T = int(self.seen[b])
        K, V = W.kv(self.wl, b, 0, T)
        A = self.alpha_of(b, 0, T, K)
        if self.dec_alpha:
            A = A.copy()
            for (sb, pos), row in self.dec_alpha.items():
                if sb == b and pos < T:
                    A[pos] = row
        return oracle.decode_gqa(W.to_f64(q), W.to_f64(K), W.to_f64(V), A, self.wl.window, self.scale)

    def oracle_all(self, Q: np.ndarray, seqs=None, group: int = 2) -> np.ndarray:
        """Oracle outputs [len(seqs), Hq, d] of many sequences at their current last
        positions, streams run in parallel by the oracle's batch routine, `group`
        sequences at a time (bounded host memory)."""
        seqs = list(range(self.wl.batch)) if seqs is None else list(seqs)
        hkv, g = self.wl.num_kv_heads, self.wl.group
        out = np.empty((len(seqs), self.wl.num_q_heads, self.wl.head_dim))
        for j0 in range(0, len(seqs), group):
            items = []
            for j in range(j0, min(j0 + group, len(seqs))):
                b = seqs[j]
                T = int(self.seen[b])
                K, V = W.kv(self.wl, b, 0, T)
                A = self.alpha_of(b, 0, T, K)
                if self.dec_alpha:
                    A = A.copy()
                    for (sb, pos), row in self.dec_alpha.items():
                        if sb == b and pos < T:
                            A[pos] = row
                q, K, V = W.to_f64(Q[j]), W.to_f64(K), W.to_f64(V)
                for k in range(hkv):
                    items.append((q[k * g:(k + 1) * g], K[:, k], V[:, k], A[:, k]))
            res, _ = oracle.attention_batch(items, self.wl.window, self.scale)
            for n, j in enumerate(range(j0, min(j0 + group, len(seqs)))):
                out[j] = np.concatenate(res[n * hkv:(n + 1) * hkv])
        return out

    def check_metadata(self) -> None:
        """Page tables, counters, free stack and retained sets bit-exact against the simulator."""
        g, o = self.cache.snapshot(), self.sim.snapshot()
        for k in ("n", "pos", "n_pages"):
            np.testing.assert_array_equal(g[k], o[k], err_msg=k)
        assert g["free_count"] == o["free_count"]
        fc = g["free_count"]
        np.testing.assert_array_equal(g["free_list"][:fc], o["free_list"][:fc])
        for st in range(self.wl.streams):
            np_ = int(o["n_pages"][st])
            np.testing.assert_array_equal(g["page_table"][st, :np_], o["page_table"][st, :np_],
                                          err_msg=f"page table of stream {st}")
            n = int(o["n"][st])
            if n:
                l = np.arange(n)
                phys = o["page_table"][st, l // 16] * 16 + l % 16
                np.testing.assert_array_equal(g["slot_pos"][phys], o["slot_pos"][phys],
                                              err_msg=f"retained positions of stream {st}")

    def close(self) -> None:
        self.cache.close()
        if self.sim is not None:
            self.sim.close()


def compare(got: torch.Tensor, ref: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS) -> tuple[float, float]:
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    mx, mn = float(err.max()), float(err.mean())
    assert np.all(np.isfinite(g)), "non-finite output"
    assert mx <= max_abs and mn <= mean_abs, f"max abs {mx:.3g} (<= {max_abs}), mean abs {mn:.3g} (<= {mean_abs})"
    return mx, mn
