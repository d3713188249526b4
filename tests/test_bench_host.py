"""Host-side logic of bench.py on CPU: the reference arm's JSON line, the
two-rank launch (only rank 0 prints), and the barrier / max-over-ranks /
whole-job throughput used around the timed regions, on two gloo ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_throughput_counts_every_rank_over_the_slowest():
    assert bench.throughput(8192, 1, 1.0) == pytest.approx(8192e3)
    assert bench.throughput(8192, 4, 2.0) == pytest.approx(4 * 8192 / 2e-3)


def test_single_rank_group_is_a_no_op():
    g = bench.RankGroup()
    g.barrier()
    assert g.max(3.25) == 3.25


def _ranks(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = bench.RankGroup(dist, torch.device("cpu"))
        g.barrier()
        out[rank] = g.max(1.5 + rank)
        g.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ranks, args=(2, free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["metric"] == bench.METRIC and d["value"] > 0 and d["steps"] == 1
    assert d["warmup"] >= 3 and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["seq_len"] == bench.T_PREFILL and "workload" in d["config"]


def test_reference_arm_under_two_ranks_prints_once():
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(free_port()),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"
    assert lines[0]["n_gpus"] == 2


def _shards(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = (bench.head_shard(rank, world), bench.attn_kv_shard(rank, world, True))
        got = [None] * world
        dist.all_gather_object(got, mine)
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_shards_tile_the_layer_on_gloo_ranks(world):
    """bench.py --shard heads: every rank takes whole key-head groups; over the
    ranks the key heads tile 0..15 and the value heads 0..47, and local value
    head j of a rank reads local key head j // 3, i.e. global value head h reads
    global key head h // 3 as in the unsharded layer."""
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shards, args=(world, free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    views = [out[r] for r in range(world)]
    assert all(v == views[0] for v in views)          # every rank sees the same plan
    kh, vh, gk = [], [], []
    for r, ((k0, k1, v0, v1), (g0, g1)) in enumerate(views[0]):
        gk += list(range(g0, g1))
        kh += list(range(k0, k1))
        vh += list(range(v0, v1))
        for j in range(v1 - v0):
            assert k0 + j // 3 == (v0 + j) // 3
        ch = bench.shard_channels(k0, k1, v0, v1)
        assert len(ch) == 2 * (k1 - k0) * 128 + (v1 - v0) * 128
        assert ch[0] == 128 * k0 and ch[(k1 - k0) * 128] == 2048 + 128 * k0
        assert ch[2 * (k1 - k0) * 128] == 4096 + 128 * v0
    assert kh == list(range(16)) and vh == list(range(48))
    assert gk == list(range(4))        # the attention layer's key-value heads tile 0..3
    with pytest.raises(ValueError):
        bench.head_shard(0, 3)
    assert bench.attn_kv_shard(1, 8, True) == (0, 4)   # 4 heads over 8 ranks: replicas
    assert bench.attn_kv_shard(1, 2, False) == (0, 4)


def test_attention_work_formulas():
    """The attention legs' algorithmic work, against sums written out:
    S = Q K^T and O = P V cost 2 * 2 * 256 flops per (query, key) pair and query
    head over the causal triangle; a decode step reads every cached key and value
    row once (fp16, 4 key-value heads of 256) plus its own inputs and output."""
    T = 10
    pairs = sum(t + 1 for t in range(T))
    assert bench.attn_prefill_flop(T) == 4 * 256 * 24 * pairs
    N, L = 3, 7
    kv = 2 * (L + 1) * 4 * 256 * 2           # keys and values of L cached + 1 new rows
    new = 2 * 4 * 256 * 2                    # the new key and value written
    inputs = (24 + 24 + 4 + 4) * 256 * 2     # q, gate, k, v in bf16
    out = 24 * 256 * 2
    assert bench.attn_decode_bytes(N, L) == N * (kv + new + inputs + out)
