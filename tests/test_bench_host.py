"""Host logic of bench.py across ranks, on CPU with the gloo backend (world size 2).

The decode path shards by sequence with no data-path collective: every rank
runs its own replica on its own GPU. What crosses ranks is only the
reporting: the timed region is the max over ranks, the bytes the sum. These
tests run those reductions and the sequence assignment in two real
processes over gloo, without a GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t_ms = [3.0, 5.5][rank]
        nbytes = [1.0e9, 2.5e9][rank]
        t_max, total = bench.reduce_over_ranks(t_ms, nbytes, world, "cpu")
        seqs = bench.rank_sequences(rank, 16)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"t_max": t_max, "total": total, "seqs": seqs}, f)
    finally:
        dist.destroy_process_group()


def test_reductions_and_sequence_shards_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["t_max"] == 5.5          # max over ranks
        assert r["total"] == 3.5e9        # sum over ranks
    s0, s1 = set(res[0]["seqs"]), set(res[1]["seqs"])
    assert len(s0) == len(s1) == 16 and not (s0 & s1)   # disjoint, equal shards
    assert sorted(s0 | s1) == list(range(32))


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(2.0, 7.0, 1, "cpu") == (2.0, 7.0)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    """`bench.py --impl reference` launched as two ranks: rank 0 times the oracle and
    prints the JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--workload", "tiny"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "GB/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0


def test_code_fingerprint_ignores_comments_only(tmp_path):
    """The profile summaries are matched to the kernel by a hash of its code with comments
    and whitespace removed: a comment edit keeps the match, a code edit breaks it."""
    sys.path.insert(0, ROOT)
    import bench
    a = tmp_path / "a.cu"
    a.write_text("// header\nint f(int x) {  /* a\n block */ return x + 1; }  // tail\n")
    b = tmp_path / "b.cu"
    b.write_text("// another header\n\nint f(int x) {\n  return x + 1;\n}\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench.code_fingerprint(str(a)) == bench.code_fingerprint(str(b))
    assert bench.code_fingerprint(str(a)) != bench.code_fingerprint(str(c))


def test_profile_traffic_needs_the_matching_code_hash():
    """bench.py reports `traffic` from a committed profile summary only while its recorded
    code hash matches the kernel source."""
    sys.path.insert(0, ROOT)
    import bench
    import re as _re
    src = os.path.join(ROOT, "learned_kv_cache_decode_b200", "csrc", "dms_attention.cu")
    path = os.path.join(ROOT, "profiles", "dms_decode_step_mma_qwen-r1-7b-32k.md")
    text = open(path).read()
    recorded = _re.search(r"code_sha256:\s*([0-9a-f]{64})", text).group(1)
    traffic = bench.profile_traffic("qwen-r1-7b-32k", "mma", "dms_decode_step")
    if recorded == bench.code_fingerprint(src):
        assert traffic is not None and traffic > 1e8
    else:
        assert traffic is None
    assert bench.profile_traffic("no-such-workload", "mma", "dms_decode_step") is None
