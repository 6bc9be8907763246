"""Seeded synthetic inputs for the DMS decode workloads.

This module holds shapes, value distributions and random draws only. It
contains none of the retention or attention arithmetic, so both the CUDA
path and the CPU oracle can take their inputs from it.

Every block of random numbers comes from its own ``numpy`` PCG64 stream,
keyed by ``SeedSequence([seed, kind, seq, chunk])``. Any side can therefore
regenerate the K/V rows or eviction bits of one sequence at any position
without replaying the rest.

The five workloads are synthetic stand-ins for the models and reasoning
benchmarks measured in "Inference-Time Hyper-Scaling with KV Cache
Compression" (paper summary, Results; Table 1; Figs. 3-4). Only the
attention shapes of those models are kept. No benchmark item, dataset
record or trained weight is used.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import dataclasses

import numpy as np

KV_CHUNK = 1024       # positions per independently seeded K/V block
ALPHA_CHUNK = 4096    # positions per independently seeded alpha block

_KIND_K, _KIND_V, _KIND_Q, _KIND_ALPHA, _KIND_CTX, _KIND_P = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    alpha_mode:
      "bernoulli"  : alpha ~ Bernoulli(p), alpha_args = (p,)
      "ramp"       : p(j) = p0 + (p1 - p0) * min(j, L) / L, alpha_args = (p0, p1, L)
      "per_stream" : p drawn once per (sequence, KV head) ~ U[lo, hi], alpha_args = (lo, hi)
    """

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str            # "bf16" or "f32"
    window: int
    context: int          # prompt length of every sequence (ignored if ctx_range set)
    ctx_range: tuple | None
    decode_steps: int
    alpha_mode: str
    alpha_args: tuple
    seed: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def streams(self) -> int:
        return self.batch * self.num_kv_heads


WORKLOADS: dict[str, Workload] = {
    # 1 sequence, 4 query / 1 KV head, d 64, fp32, prompt 512, w 16, 64 steps.
    "tiny": Workload("tiny", 1, 4, 1, 64, "f32", 16, 512, None, 64,
                     "bernoulli", (0.5,), 1001),
    # Llama-3.2-1B attention shape: 32/8 heads, d 64, batch 8, 4K prompt, CR about 2.
    "llama3.2-1b": Workload("llama3.2-1b", 8, 32, 8, 64, "bf16", 256, 4096, None, 256,
                            "bernoulli", (0.5,), 1002),
    # Qwen-R1-7B shape: 28/4 heads, d 128, batch 16, 32K prompt, p ramps 0.5 -> 0.9375
    # over the first 10K positions (compression grows along the sequence).
    "qwen-r1-7b-32k": Workload("qwen-r1-7b-32k", 16, 28, 4, 128, "bf16", 256, 32768, None, 256,
                               "ramp", (0.5, 0.9375, 10000), 1003),
    # Qwen-R1-32B shape, 64 independent chains, prompts uniform in [8K, 32K],
    # per-(chain, head) eviction rate uniform in [0.8, 0.95].
    "qwen-r1-32b-chains": Workload("qwen-r1-32b-chains", 64, 40, 8, 128, "bf16", 256, 0,
                                   (8192, 32768), 256, "per_stream", (0.8, 0.95), 1004),
    # Long decode loop: 28/4 heads, d 128, batch 32, 2K prompt then 30K steps, CR about 8.
    "longrun-2k-30k": Workload("longrun-2k-30k", 32, 28, 4, 128, "bf16", 256, 2048, None, 30000,
                               "bernoulli", (0.875,), 1005),
}


def depth_layers(wl: Workload, layers: int, cr_first: float, cr_last: float) -> list[Workload]:
    """Per-layer workloads with compression that grows with depth ("Inference-Time
    Hyper-Scaling with KV Cache Compression", paper summary, Method: early layers are
    compressed less, Fig. 6). Layer l draws alpha ~ Bernoulli(p_l), with the long-context
    ratio 1 / (1 - p_l) linear in l from cr_first to cr_last, each layer from its own
    seed. Only alpha is drawn from a layer workload; K, V and queries come from `wl`."""
    out = []
    for l in range(layers):
        cr = cr_first + (cr_last - cr_first) * (l / (layers - 1) if layers > 1 else 0.0)
        out.append(dataclasses.replace(wl, name=f"{wl.name}-layer{l}", alpha_mode="bernoulli",
                                       alpha_args=(1.0 - 1.0 / cr,), seed=wl.seed + 7919 * (l + 1)))
    return out


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float64."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray) -> np.ndarray:
    """Exact float64 view of stored values (bf16 bits as uint16, or float32)."""
    return bf16_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)


def contexts(wl: Workload) -> np.ndarray:
    """Prompt length of each sequence."""
    if wl.ctx_range is None:
        return np.full(wl.batch, wl.context, dtype=np.int64)
    lo, hi = wl.ctx_range
    return _rng(wl.seed, _KIND_CTX).integers(lo, hi, size=wl.batch, endpoint=True).astype(np.int64)


def stream_rates(wl: Workload, seq: int) -> np.ndarray:
    """Per-KV-head eviction probability of one sequence (per_stream mode only)."""
    lo, hi = wl.alpha_args
    return _rng(wl.seed, _KIND_P, seq).uniform(lo, hi, size=wl.num_kv_heads)


def alpha_prob(wl: Workload, seq: int, positions: np.ndarray) -> np.ndarray:
    """Eviction probability p for each position (rows) and KV head (columns)."""
    positions = np.asarray(positions, dtype=np.float64)
    h = wl.num_kv_heads
    if wl.alpha_mode == "bernoulli":
        return np.full((positions.size, h), wl.alpha_args[0])
    if wl.alpha_mode == "ramp":
        p0, p1, length = wl.alpha_args
        p = p0 + (p1 - p0) * np.minimum(positions, length) / length
        return np.repeat(p[:, None], h, axis=1)
    if wl.alpha_mode == "per_stream":
        return np.repeat(stream_rates(wl, seq)[None, :], positions.size, axis=0)
    raise ValueError(wl.alpha_mode)


def alpha(wl: Workload, seq: int, start: int, count: int) -> np.ndarray:
    """Eviction bits for positions [start, start+count) of one sequence: uint8 [count, Hkv]."""
    out = np.empty((count, wl.num_kv_heads), dtype=np.uint8)
    if count == 0:
        return out
    end = start + count
    for c in range(start // ALPHA_CHUNK, (end - 1) // ALPHA_CHUNK + 1):
        c0 = c * ALPHA_CHUNK
        u = _rng(wl.seed, _KIND_ALPHA, seq, c).random((ALPHA_CHUNK, wl.num_kv_heads))
        lo, hi = max(start, c0), min(end, c0 + ALPHA_CHUNK)
        p = alpha_prob(wl, seq, np.arange(lo, hi))
        out[lo - start:hi - start] = (u[lo - c0:hi - c0] < p).astype(np.uint8)
    return out


def _normal_block(wl: Workload, kind: int, seq: int, chunk: int) -> np.ndarray:
    x = _rng(wl.seed, kind, seq, chunk).standard_normal(
        (KV_CHUNK, wl.num_kv_heads, wl.head_dim), dtype=np.float32)
    return bf16_bits(x) if wl.dtype == "bf16" else x


def kv(wl: Workload, seq: int, start: int, count: int, threads: int = 8):
    """K and V rows for positions [start, start+count) of one sequence.

    Returns two arrays [count, Hkv, d]: uint16 bf16 bits for bf16 workloads,
    float32 otherwise.
    """
    dt = np.uint16 if wl.dtype == "bf16" else np.float32
    shape = (count, wl.num_kv_heads, wl.head_dim)
    K, V = np.empty(shape, dtype=dt), np.empty(shape, dtype=dt)
    if count == 0:
        return K, V
    end = start + count
    chunks = list(range(start // KV_CHUNK, (end - 1) // KV_CHUNK + 1))

    def fill(c: int) -> None:
        c0 = c * KV_CHUNK
        lo, hi = max(start, c0), min(end, c0 + KV_CHUNK)
        K[lo - start:hi - start] = _normal_block(wl, _KIND_K, seq, c)[lo - c0:hi - c0]
        V[lo - start:hi - start] = _normal_block(wl, _KIND_V, seq, c)[lo - c0:hi - c0]

    if len(chunks) > 1 and threads > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, chunks))
    else:
        for c in chunks:
            fill(c)
    return K, V


def query(wl: Workload, step: int) -> np.ndarray:
    """Queries of decode step ``step`` for all sequences: [B, Hq, d]."""
    x = _rng(wl.seed, _KIND_Q, step).standard_normal(
        (wl.batch, wl.num_q_heads, wl.head_dim), dtype=np.float32)
    return bf16_bits(x) if wl.dtype == "bf16" else x
