"""Scores with a large spread, where the kernel departs most from the oracle (GPU).

The kernel keeps an fp32 online softmax per warp, merges the warps of a CTA,
and combines the pieces of a stream that several CTAs share. With ordinary
N(0, 1) inputs the scores stay within a few units; here they do not:

  * queries scaled by 8 and 16 (exact in bf16: powers of two), so every
    running max moves by tens of units and the rescale factors underflow;
  * one dominant key per stream, aligned with one query head, placed on page
    and piece boundaries (with fewer pages than SMs every page is a piece of
    its own, so pages 15 | 16 and 31 | 32 sit on split-K boundaries), so one
    piece's partial outweighs the others' by e^40 and more in the combine;
  * in the decode step, a dominant key that leaves the window at this very
    step (it must be masked, or the output would be its value row), and a
    dominant new token (merged from the step's inputs).

Every output is compared with the fp64 oracle at the usual tolerances.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from learned_kv_cache_decode_b200 import DmsCache, _native
from learned_kv_cache_decode_b200 import workloads as W
from harness import MAX_ABS, MEAN_ABS, compare

pytestmark = pytest.mark.gpu


def stored(x, dtype):
    """float32 -> the stored values (bf16 bits as uint16, or float32) and a device tensor."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        bits = W.bf16_bits(x)
        return bits, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return x, torch.from_numpy(x).cuda()


def dominant_key(q_row, d, strength=4.0):
    """A key whose score with q_row is about strength * sqrt(d) * |q| * scale above the rest."""
    return strength * math.sqrt(d) * q_row / np.linalg.norm(q_row)


CASES = [  # (dtype, kernel, d, g, w, q scale)
    ("bf16", "mma", 128, 7, 64, 8.0),
    ("bf16", "mma", 128, 7, 64, 16.0),
    ("bf16", "mma", 64, 4, 16, 16.0),
    ("bf16", "simt", 128, 7, 64, 16.0),
    ("f32", "simt", 64, 4, 16, 8.0),
]


@pytest.mark.parametrize("dtype,kernel,d,g,w,qs", CASES,
                         ids=[f"{c[0]}-{c[1]}-d{c[2]}-g{c[3]}-q{int(c[5])}" for c in CASES])
@pytest.mark.parametrize("alpha_mode", ["dense", "mixed"])
def test_dominant_keys_on_piece_boundaries_and_scaled_queries(dtype, kernel, d, g, w, qs, alpha_mode):
    hkv, B = 2, 4
    hq = g * hkv
    T = [48, 40, 33, 80]   # tokens per sequence: several pages, ragged last pages
    where = [[15, 16], [31, 32], [0, 32], [47, 79]]   # dominant keys: page / piece boundaries
    rng = np.random.default_rng(90 + d + g + int(qs))
    scale = 1.0 / math.sqrt(d)
    Q = rng.standard_normal((B, hq, d)).astype(np.float32) * qs
    Qh, Qd = stored(Q, dtype)
    Qf = W.to_f64(Qh)
    mps = 8
    cache = DmsCache(B, hkv, d, w, B * hkv * mps, mps, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                     attn_kernel=kernel)
    try:
        Ks, Vs, As = [], [], []
        for b in range(B):
            K = rng.standard_normal((T[b], hkv, d)).astype(np.float32)
            V = rng.standard_normal((T[b], hkv, d)).astype(np.float32)
            A = (rng.random((T[b], hkv)) < 0.5).astype(np.uint8) if alpha_mode == "mixed" else \
                np.zeros((T[b], hkv), dtype=np.uint8)
            for k in range(hkv):
                for j, p in enumerate(where[b]):
                    K[p, k] = dominant_key(Q[b, k * g + j % g], d)   # head j of the group
                    A[p, k] = 0                                        # kept
            Ks.append(stored(K, dtype)[0])
            Vs.append(stored(V, dtype)[0])
            As.append(A)
        cu = np.concatenate([[0], np.cumsum(T)]).astype(np.int32)
        ids = torch.arange(B, dtype=torch.int32, device="cuda")
        dev = lambda x: stored(W.to_f64(x).astype(np.float32), dtype)[1]
        cache.append(ids, dev(np.concatenate(Ks)), dev(np.concatenate(Vs)),
                     torch.from_numpy(np.concatenate(As)).cuda(), cu_tokens=torch.from_numpy(cu).cuda())
        out = cache.decode_attention(ids, Qd, scale=scale, out_dtype=torch.float32)
        torch.cuda.synchronize()
        tol = dict(max_abs=1e-4, mean_abs=1e-5) if dtype == "f32" else dict(max_abs=MAX_ABS, mean_abs=MEAN_ABS)
        for b in range(B):
            ref = oracle.decode_gqa(Qf[b], W.to_f64(Ks[b]), W.to_f64(Vs[b]), As[b], w, scale)
            compare(out[b], ref, **tol)
        assert cache.status() == _native.DMS_OK
    finally:
        cache.close()


@pytest.mark.parametrize("fused", [False, True], ids=["two_launches", "fused_step"])
@pytest.mark.parametrize("kernel", ["mma", "simt"])
def test_dominant_key_leaving_at_the_step_and_dominant_new_token(fused, kernel):
    """Sequence 0: the token that leaves the window at this step (marked, s - w) is
    dominant; attending it would return its value row. Sequence 1: the new token is
    dominant (in the fused step it enters the final merge from the step's inputs).
    Sequence 2: a dominant key that stays. All against the oracle."""
    d, g, hkv, w, B = 128, 7, 2, 8, 3
    hq = g * hkv
    T = 40
    rng = np.random.default_rng(97)
    scale = 1.0 / math.sqrt(d)
    Q = rng.standard_normal((B, hq, d)).astype(np.float32) * 8.0
    Qh, Qd = stored(Q, "bf16")
    mps = 6
    cache = DmsCache(B, hkv, d, w, B * hkv * mps, mps, attn_kernel=kernel)
    try:
        K = rng.standard_normal((B, T + 1, hkv, d)).astype(np.float32)
        V = rng.standard_normal((B, T + 1, hkv, d)).astype(np.float32)
        A = (rng.random((B, T + 1, hkv)) < 0.5).astype(np.uint8)
        for k in range(hkv):
            K[0, T - w, k] = dominant_key(Q[0, k * g], d)     # leaves when token T arrives
            A[0, T - w, k] = 1
            K[1, T, k] = dominant_key(Q[1, k * g + 3], d)     # the new token
            K[2, 20, k] = dominant_key(Q[2, k * g + 6], d)    # kept
            A[2, 20, k] = 0
        Kh, Kd = stored(K.reshape(-1, hkv, d), "bf16")
        Vh, Vd = stored(V.reshape(-1, hkv, d), "bf16")
        Kh, Vh = Kh.reshape(B, T + 1, hkv, d), Vh.reshape(B, T + 1, hkv, d)
        Kd, Vd = Kd.view(B, T + 1, hkv, d), Vd.view(B, T + 1, hkv, d)
        ids = torch.arange(B, dtype=torch.int32, device="cuda")
        cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device="cuda")
        cache.append(ids, Kd[:, :T].reshape(-1, hkv, d).contiguous(), Vd[:, :T].reshape(-1, hkv, d).contiguous(),
                     torch.from_numpy(A[:, :T].reshape(-1, hkv).copy()).cuda(), cu_tokens=cu)
        kn, vn = Kd[:, T].contiguous(), Vd[:, T].contiguous()
        an = torch.from_numpy(A[:, T].copy()).cuda()
        if fused:
            out = cache.decode_step(ids, kn, vn, an, Qd, scale=scale, out_dtype=torch.float32)
        else:
            cache.append(ids, kn, vn, an)
            out = cache.decode_attention(ids, Qd, scale=scale, out_dtype=torch.float32)
        torch.cuda.synchronize()
        Qf = W.to_f64(Qh)
        for b in range(B):
            ref = oracle.decode_gqa(Qf[b], W.to_f64(Kh[b]), W.to_f64(Vh[b]), A[b], w, scale)
            compare(out[b], ref)
        # the leaving dominant key really would have dominated: its value row differs
        leaving = W.to_f64(Vh[0, T - w, 0])
        assert float(np.abs(out[0, 0].double().cpu().numpy() - leaving).max()) > 0.1
        assert cache.status() == _native.DMS_OK
    finally:
        cache.close()
