"""Host-side logic of bench.py, no GPU: the max-over-ranks timing reduction with
two gloo ranks, the reference (oracle) arm's JSON line, and the ncu-traffic
guard that only reports traffic for the kernel source it was measured on."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], dist, "cpu")
    out_q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res[0] == res[1] == [11.0, 5.0]


def test_reference_arm_prints_one_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny-stream",
           "--steps", "2", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, check=True).stdout.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["unit"] == "latent frames/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny-stream",
           "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "causal_dit_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "attention.cu").write_bytes(b"kernel v1 // first\n")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()[:16]
    (tmp_path / "profiles" / "chunk_attention_w.md").write_text(
        f"traffic_bytes_per_launch: 123\nsource_sha256_prefix: {h}\n")
    assert bench.profiled_traffic("w") == 123
    (csrc / "attention.cu").write_bytes(b"// a comment-only edit\nkernel v1 // reworded\n\n")
    assert bench.profiled_traffic("w") == 123
    (csrc / "attention.cu").write_bytes(b"kernel v2")
    assert bench.profiled_traffic("w") is None


def test_fp8_workloads_byte_accounting():
    import bench
    w16, w8 = bench.WORKLOADS["wan1.3b-512x512"], bench.WORKLOADS["wan1.3b-512x512-fp8"]
    keys = bench.steady_keys(w16)
    assert bench.steady_keys(w8) == keys == [7168]
    b16, b8 = bench.attn_bytes(w16, keys), bench.attn_bytes(w8, keys)
    hd, lq = 12 * 128, 1024
    assert b16 == 4 * 7168 * hd + 4 * lq * hd                               # K+V, Q, O in bf16
    # codes for K and V, raw bf16 Q (rotated on load), bf16 O, one K and one V scale per block and head
    assert b8 == 2 * 7168 * hd + 2 * lq * hd + 2 * lq * hd + 2 * 4 * 12 * 56
    assert bench.attn_flops(w8, keys) == bench.attn_flops(w16, keys)
    assert bench.workload_config("x", w8, 1)["kv_format"] == "fp8"
    assert bench.workload_config("x", w16, 1)["kv_format"] == "bf16"
    assert bench.kv_elem(w8) == 1 and bench.kv_elem(w16) == 2
    # 64-token frames: 7 slots of one (half-full) block each, 7 K and 7 V scales per head
    s8 = bench.WORKLOADS["wan1.3b-128x128-b16-fp8"]
    ks = bench.steady_keys(s8)
    assert ks == [448] * 16
    assert bench.attn_bytes(s8, ks) == 16 * (2 * 448 * hd + 2 * 64 * hd + 2 * 64 * hd + 2 * 4 * 12 * 7)


def test_fused_workloads_byte_accounting():
    import bench
    plain, fused = bench.WORKLOADS["wan1.3b-128x128-b16"], bench.WORKLOADS["wan1.3b-128x128-b16-fused"]
    keys = bench.steady_keys(plain)
    assert keys == [448] * 16
    hd, lq = 12 * 128, 64
    # the fused launch also writes the chunk's K and V (bf16) to their ring slots
    assert bench.attn_bytes(fused, keys) == bench.attn_bytes(plain, keys) + 16 * 4 * lq * hd
    assert bench.attn_flops(fused, keys) == bench.attn_flops(plain, keys)
    assert "fused" in bench.workload_config("x", fused, 1)["append"]
    assert "append" not in bench.workload_config("x", plain, 1)
    assert "wan1.3b-128x128-b16-fused" in bench.EXTRA_WORKLOADS
