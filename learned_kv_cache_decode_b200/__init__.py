"""learned_kv_cache_decode_b200: the decode hot path of Dynamic Memory
Sparsification (DMS) on NVIDIA B200, behind the C ABI of ``libdms.so``.

DMS ("Inference-Time Hyper-Scaling with KV Cache Compression"): every KV
head takes a learned binary eviction decision per token; a token marked at
step t stays attendable until step t + w, then leaves the cache and its slot
is reused. Decode attention runs over the retained tokens only.

This module is argument marshalling for the C ABI (include/dms.h). PyTorch
provides device memory and the current CUDA stream; every step of the path
runs in the library's kernels.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _native
from ._native import DmsError

__all__ = ["DmsCache", "DmsError", "decode_attention_noalloc", "alpha_from_logit"]

_DTYPES = {torch.bfloat16: _native.DMS_BF16, torch.float32: _native.DMS_F32}
_KERNELS = {"auto": _native.DMS_ATTN_AUTO, "simt": _native.DMS_ATTN_SIMT, "mma": _native.DMS_ATTN_MMA}


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


@dataclass
class CacheConfig:
    max_seqs: int
    num_kv_heads: int
    head_dim: int
    window: int
    max_pages: int
    max_pages_per_stream: int
    dtype: torch.dtype = torch.bfloat16
    attn_kernel: str = "auto"
    page_size: int = 16


class DmsCache:
    """A DMS slot pool on the current CUDA device (wraps ``dms_cache``)."""

    def __init__(self, max_seqs: int, num_kv_heads: int, head_dim: int, window: int, max_pages: int,
                 max_pages_per_stream: int, dtype: torch.dtype = torch.bfloat16, attn_kernel: str = "auto",
                 page_size: int = 16):
        self.lib = _native.load()
        self.cfg = CacheConfig(max_seqs, num_kv_heads, head_dim, window, max_pages, max_pages_per_stream,
                               dtype, attn_kernel, page_size)
        if dtype not in _DTYPES or attn_kernel not in _KERNELS:
            raise ValueError("dtype must be bfloat16 or float32; attn_kernel auto|simt|mma")
        c = _native.DmsConfig(max_seqs, num_kv_heads, head_dim, page_size, window, max_pages,
                              max_pages_per_stream, _DTYPES[dtype], _KERNELS[attn_kernel])
        h = ctypes.c_void_p()
        _native.check(self.lib.dms_cache_create(ctypes.byref(c), ctypes.byref(h)), "dms_cache_create")
        self._h = h
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.streams = max_seqs * num_kv_heads

    # -- lifecycle ---------------------------------------------------------
    def close(self) -> None:
        if getattr(self, "_h", None):
            self.lib.dms_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self) -> None:
        _native.check(self.lib.dms_cache_reset(self._h, _stream()), "dms_cache_reset")

    def reset_seq(self, seq_id: int) -> None:
        _native.check(self.lib.dms_seq_reset(self._h, _stream(), int(seq_id)), "dms_seq_reset")

    # -- hot path ----------------------------------------------------------
    def append(self, seq_ids: torch.Tensor, K: torch.Tensor, V: torch.Tensor, alpha: torch.Tensor | None = None,
               cu_tokens: torch.Tensor | None = None, alpha_channel: int | None = None) -> None:
        """Append tokens. seq_ids int32 [B]; K, V [T, Hkv, d]; alpha uint8 [T, Hkv], or
        alpha_channel: alpha = K[..., alpha_channel] > 0; cu_tokens int32 [B+1] or None
        for one token per sequence."""
        n = int(seq_ids.numel())
        if alpha_channel is not None:
            _native.check(self.lib.dms_append_keyed(self._h, _stream(), n, _ptr(seq_ids), _ptr(cu_tokens),
                                                    int(K.shape[0]), _ptr(K), _ptr(V), int(alpha_channel)),
                          "dms_append_keyed")
            return
        _native.check(self.lib.dms_append(self._h, _stream(), n, _ptr(seq_ids), _ptr(cu_tokens),
                                          int(K.shape[0]), _ptr(K), _ptr(V), _ptr(alpha)), "dms_append")

    def decode_attention(self, seq_ids: torch.Tensor, Q: torch.Tensor, scale: float | None = None,
                         out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None) -> torch.Tensor:
        """GQA decode attention over the retained tokens. Q [B, Hq, d] -> out [B, Hq, d]."""
        b, hq, d = Q.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        if out is None:
            out = torch.empty((b, hq, d), dtype=out_dtype or Q.dtype, device=Q.device)
        _native.check(self.lib.dms_decode_attention(self._h, _stream(), int(seq_ids.numel()), _ptr(seq_ids),
                                                    _ptr(Q), hq, float(scale), _ptr(out),
                                                    _DTYPES[out.dtype]), "dms_decode_attention")
        return out

    def decode_step(self, seq_ids: torch.Tensor, K: torch.Tensor, V: torch.Tensor, alpha: torch.Tensor | None,
                    Q: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None,
                    out_dtype: torch.dtype | None = None, alpha_channel: int | None = None,
                    alpha_head: int | None = None) -> torch.Tensor:
        """One decode step in one launch: append one token per sequence (K, V [B, Hkv, d],
        alpha uint8 [B, Hkv], or alpha_channel: alpha = K[..., alpha_channel] > 0, or with
        alpha_head as well: alpha = Q[:, kv * g + alpha_head, alpha_channel] > 0) and
        attend with Q [B, Hq, d] -> out [B, Hq, d]."""
        b, hq, d = Q.shape
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        if out is None:
            out = torch.empty((b, hq, d), dtype=out_dtype or Q.dtype, device=Q.device)
        if alpha_channel is not None and alpha_head is not None:
            _native.check(self.lib.dms_decode_step_qkeyed(self._h, _stream(), int(seq_ids.numel()), _ptr(seq_ids),
                                                          _ptr(K), _ptr(V), _ptr(Q), hq, int(alpha_head),
                                                          int(alpha_channel), float(scale), _ptr(out),
                                                          _DTYPES[out.dtype]), "dms_decode_step_qkeyed")
            return out
        if alpha_channel is not None:
            _native.check(self.lib.dms_decode_step_keyed(self._h, _stream(), int(seq_ids.numel()), _ptr(seq_ids),
                                                         _ptr(K), _ptr(V), int(alpha_channel), _ptr(Q), hq,
                                                         float(scale), _ptr(out), _DTYPES[out.dtype]),
                          "dms_decode_step_keyed")
            return out
        _native.check(self.lib.dms_decode_step(self._h, _stream(), int(seq_ids.numel()), _ptr(seq_ids), _ptr(K),
                                               _ptr(V), _ptr(alpha), _ptr(Q), hq, float(scale), _ptr(out),
                                               _DTYPES[out.dtype]), "dms_decode_step")
        return out

    # -- inspection --------------------------------------------------------
    def stats(self) -> dict:
        """Device tensors: retained [S], seen [S], head_cr [Hkv], totals [2] (async)."""
        dev = self.device
        r = torch.empty(self.streams, dtype=torch.int32, device=dev)
        s = torch.empty(self.streams, dtype=torch.int32, device=dev)
        cr = torch.empty(self.cfg.num_kv_heads, dtype=torch.float32, device=dev)
        tot = torch.empty(2, dtype=torch.int64, device=dev)
        _native.check(self.lib.dms_stats(self._h, _stream(), _ptr(r), _ptr(s), _ptr(cr), _ptr(tot)), "dms_stats")
        return {"retained": r, "seen": s, "head_cr": cr, "totals": tot}

    def stats_host(self) -> dict:
        """Host copies of the per-stream counts and the overall compression ratio
        (wraps dms_stats_host; syncs the stream)."""
        import numpy as np
        r = np.empty(self.streams, dtype=np.int32)
        s = np.empty(self.streams, dtype=np.int32)
        cr = ctypes.c_double()
        _native.check(self.lib.dms_stats_host(self._h, _stream(), r.ctypes.data, s.ctypes.data, ctypes.byref(cr)),
                      "dms_stats_host")
        return {"retained": r, "seen": s, "cr_overall": cr.value}

    def snapshot(self) -> dict:
        """Host copies of the bookkeeping (syncs the stream)."""
        import numpy as np
        S, mps, mp = self.streams, self.cfg.max_pages_per_stream, self.cfg.max_pages
        out = {
            "page_table": np.empty((S, mps), dtype=np.int32),
            "n_pages": np.empty(S, dtype=np.int32),
            "n": np.empty(S, dtype=np.int32),
            "pos": np.empty(S, dtype=np.int32),
            "slot_pos": np.empty(mp * self.cfg.page_size, dtype=np.int32),
            "free_list": np.empty(mp, dtype=np.int32),
            "free_count": np.empty(1, dtype=np.int32),
        }
        args = [out[k].ctypes.data for k in ("page_table", "n_pages", "n", "pos", "slot_pos", "free_list",
                                             "free_count")]
        _native.check(self.lib.dms_snapshot(self._h, _stream(), *args), "dms_snapshot")
        out["free_count"] = int(out["free_count"][0])
        return out

    def gather_kv(self, seq_id: int, kv_head: int, rows: int):
        """Retained K, V rows of one stream in logical slot order: two [rows, d] tensors."""
        K = torch.empty((rows, self.cfg.head_dim), dtype=self.cfg.dtype, device=self.device)
        V = torch.empty_like(K)
        _native.check(self.lib.dms_gather_kv(self._h, _stream(), int(seq_id), int(kv_head), int(rows),
                                             _ptr(K), _ptr(V)), "dms_gather_kv")
        return K, V

    def selftest_bounded_waits(self) -> torch.Tensor:
        """Run the library's bounded waits on conditions that never come true (about two
        seconds). Each gives up and latches DMS_ERR_TIMEOUT, poisoning the cache until
        reset(). Returns a device int32 [2]: 1 where each wait gave up."""
        t = torch.zeros(2, dtype=torch.int32, device=self.device)
        _native.check(self.lib.dms_selftest_bounded_waits(self._h, _stream(), _ptr(t)), "dms_selftest_bounded_waits")
        return t

    def status(self) -> int:
        """Latched device status (syncs)."""
        return int(self.lib.dms_get_status(self._h, _stream()))

    def launches(self) -> int:
        return int(self.lib.dms_launch_count(self._h))


def decode_attention_noalloc(kv_pool: torch.Tensor, page_table: torch.Tensor, retained: torch.Tensor,
                             num_kv_heads: int, seq_ids: torch.Tensor, Q: torch.Tensor,
                             scale: float | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Decode attention over caller-owned paged K/V; the library allocates nothing
    (wraps ``dms_decode_attention_noalloc``).

    kv_pool [max_pages, 2, 16, d] (K rows then V rows per page), page_table int32
    [max_seqs * num_kv_heads, max_pages_per_stream], retained int32 [max_seqs *
    num_kv_heads], seq_ids int32 [B], Q [B, Hq, d] -> out [B, Hq, d]. ``out`` must be
    passed by a caller that may not allocate.
    """
    lib = _native.load()
    b, hq, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((b, hq, d), dtype=Q.dtype, device=Q.device)
    streams, mps = page_table.shape
    kv = _native.DmsPagedKv(kv_pool.data_ptr(), page_table.data_ptr(), retained.data_ptr(),
                            streams // num_kv_heads, num_kv_heads, d, kv_pool.shape[0], mps,
                            _DTYPES[kv_pool.dtype])
    _native.check(lib.dms_decode_attention_noalloc(_stream(), ctypes.byref(kv), int(seq_ids.numel()),
                                                   _ptr(seq_ids), _ptr(Q), hq, float(scale), _ptr(out),
                                                   _DTYPES[out.dtype]), "dms_decode_attention_noalloc")
    return out


def alpha_from_logit(X: torch.Tensor, num_kv_heads: int, channel: int, head: int = 0,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """Eviction decisions from the sign of a designated projection channel (wraps
    ``dms_alpha_from_logit``). X [rows, num_kv_heads * h, d] holds keys (h = 1) or
    queries (h = g, and ``head`` picks one query head of each KV head's group);
    returns uint8 [rows, num_kv_heads]: 1 iff X[r, k * h + head, channel] > 0."""
    lib = _native.load()
    rows, heads, d = X.shape
    if heads % num_kv_heads:
        raise ValueError("the head count of X must be a multiple of num_kv_heads")
    if out is None:
        out = torch.empty((rows, num_kv_heads), dtype=torch.uint8, device=X.device)
    _native.check(lib.dms_alpha_from_logit(_stream(), _ptr(X), _DTYPES[X.dtype], rows, num_kv_heads,
                                           heads // num_kv_heads, int(head), d, int(channel), _ptr(out)),
                  "dms_alpha_from_logit")
    return out
