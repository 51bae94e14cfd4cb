"""Host side of the N>1 path on CPU: two gloo ranks run bench.py's rank helpers.

The path shards by batch: every rank draws and processes its own batch and no
collective touches the data. What the ranks share is the timing protocol (a
barrier on both sides of each timed region, the max over ranks of the measured
time, the whole-job rate over all ranks' units, rank 0 printing alone); these
tests run exactly those functions over a gloo process group on 127.0.0.1.
"""
import hashlib
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _set_env(rank, world, port):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})


def _rank_timing(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    _set_env(rank, world, port)
    import bench
    from frame_level_delta_b200.inputs import CONFIGS, make_inputs

    r, w, local = bench.rank_env()
    cpu = torch.device("cpu")
    dist = bench.init_ranks(w, cpu, timeout_s=60)
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=bench.rank_seed(cfg, r))
    h = hashlib.sha256()
    for k in sorted(inp):
        h.update(inp[k].contiguous().numpy().tobytes())
    digests = [None] * w
    dist.all_gather_object(digests, h.hexdigest())
    bench.barrier(dist)
    ms = 1.0 + 2.5 * r  # rank r "took" this long
    ms_max = bench.max_over_ranks(dist, ms, cpu)
    rate = bench.whole_job_rate(w, cfg, 7, ms_max)
    bench.barrier(dist)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "local": local, "digests": digests, "ms_max": ms_max,
                   "rate": rate, "head_tokens": cfg.head_tokens}, f)


def _rank_leaves(rank, world, port, out_dir):
    """Rank 1 leaves between steps (before the barrier); rank 0 must end with an
    error from its barrier within the process group's timeout, not wait for good."""
    sys.path.insert(0, ROOT)
    _set_env(rank, world, port)
    import bench

    dist = bench.init_ranks(world, torch.device("cpu"), timeout_s=5)
    if rank == 1:
        os._exit(0)
    t0 = time.monotonic()
    err = None
    try:
        bench.barrier(dist)
        bench.barrier(dist)
    except Exception as e:  # noqa: BLE001 - any error is the expected outcome
        err = type(e).__name__
    with open(os.path.join(out_dir, "rank0.json"), "w") as f:
        json.dump({"error": err, "seconds": time.monotonic() - t0}, f)
    os._exit(0)


def _rank_heads(rank, world, port, out_dir):
    """Head-sharded ranks over one shared batch: each rank computes its heads'
    output (the float64 oracle stands in for the library on CPU), the slices are
    all-gathered, and rank 0 compares the assembly with the single-rank output."""
    sys.path.insert(0, ROOT)
    _set_env(rank, world, port)
    import numpy as np

    import bench
    from frame_level_delta_b200.inputs import CONFIGS, make_inputs
    from frame_level_delta_b200.shard import head_partition
    from oracle.vda_oracle import vda_reference

    r, w, _ = bench.rank_env()
    dist = bench.init_ranks(w, torch.device("cpu"), timeout_s=60)
    cfg = CONFIGS["small"].with_(H=5, T=8, grid_h=4, grid_w=4, L=6, d=16)
    inp = make_inputs(cfg)  # the same batch on every rank
    parts = head_partition(cfg.H, w, (5, 3))
    h0, n = parts[r]
    mine = vda_reference(inp, cfg, heads=[(0, h) for h in range(h0, h0 + n)], keep=False)["O"][:, :, h0:h0 + n]
    slices = [None] * w
    dist.all_gather_object(slices, (h0, n, mine))
    bench.barrier(dist)
    dist.destroy_process_group()
    if r == 0:
        whole = vda_reference(inp, cfg, keep=False)["O"]
        got = np.zeros_like(whole)
        for (a, k, o) in slices:
            got[:, :, a:a + k] = o
        with open(os.path.join(out_dir, "heads.json"), "w") as f:
            json.dump({"parts": [list(p) for p in parts], "equal": bool(np.array_equal(got, whole))}, f)


def _rank_ulysses(rank, world, port, out_dir):
    """Sequence-sharded ranks: each holds a contiguous token range of every head;
    the Ulysses all-to-all hands each rank every token of its heads (uneven 5:3
    split), the oracle stands in for the library on CPU, and the inverse exchange
    brings each rank its tokens of every head back."""
    sys.path.insert(0, ROOT)
    _set_env(rank, world, port)
    import numpy as np

    import bench
    from frame_level_delta_b200.inputs import CONFIGS, make_inputs
    from frame_level_delta_b200.shard import head_partition, heads_to_seq, seq_to_heads
    from oracle.vda_oracle import vda_reference

    r, w, _ = bench.rank_env()
    dist = bench.init_ranks(w, torch.device("cpu"), timeout_s=60)
    cfg = CONFIGS["small"].with_(H=5, T=8, grid_h=4, grid_w=4, L=6, d=16, dtype="f32")
    full = make_inputs(cfg)  # drawn identically on every rank; each keeps only its shard
    N = cfg.T * cfg.U
    n = N // w
    parts = head_partition(cfg.H, w, (5, 3))
    h0, k = parts[r]
    mine = {}
    for name in ("Q", "K", "V"):
        shard = full[name][:, r * n:(r + 1) * n].contiguous()
        mine[name] = seq_to_heads(shard, parts)
    ok_layout = all(torch.equal(mine[x], full[x][:, :, h0:h0 + k]) for x in mine)
    local = dict(full)
    local.update(mine)
    for name in ("K_txt", "V_txt"):
        local[name] = full[name][:, :, h0:h0 + k].contiguous()
    for name in ("alpha", "beta", "beta_txt"):
        local[name] = full[name][:, h0:h0 + k].contiguous()
    O_heads = torch.from_numpy(vda_reference(local, cfg.with_(H=k), keep=False)["O"])
    O_seq = heads_to_seq(O_heads, parts)
    want = vda_reference(full, cfg, keep=False)["O"][:, r * n:(r + 1) * n]
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"ulysses{r}.json"), "w") as f:
        json.dump({"layout": ok_layout, "equal": bool(np.array_equal(O_seq.numpy(), want)),
                   "shape": list(O_seq.shape)}, f)


def test_two_gloo_ranks_ulysses_exchange_round_trip(tmp_path):
    world = 2
    mp.start_processes(_rank_ulysses, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        d = json.loads((tmp_path / f"ulysses{r}.json").read_text())
        assert d["layout"] and d["equal"], d


def test_two_gloo_ranks_head_slices_reassemble_the_output(tmp_path):
    world = 2
    mp.start_processes(_rank_heads, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    d = json.loads((tmp_path / "heads.json").read_text())
    assert d["parts"] == [[0, 3], [3, 2]]
    assert d["equal"]


def test_two_gloo_ranks_barrier_max_and_shards(tmp_path):
    world = 2
    mp.start_processes(_rank_timing, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    for r, d in enumerate(res):
        assert (d["rank"], d["world"], d["local"]) == (r, world, r)
        # every rank sees the slowest rank's time
        assert d["ms_max"] == pytest.approx(1.0 + 2.5 * (world - 1))
        # whole-job rate: all ranks' head-tokens over that time
        assert d["rate"] == pytest.approx(world * d["head_tokens"] * 7 / (d["ms_max"] / 1e3))
    # each rank drew its own batch (independent problems), and both agree on the set
    assert res[0]["digests"] == res[1]["digests"]
    assert len(set(res[0]["digests"])) == world


def test_rank_that_leaves_ends_peer_barrier_with_error(tmp_path):
    world = 2
    ctx = mp.start_processes(_rank_leaves, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                             join=False, start_method="spawn")
    deadline = time.monotonic() + 120
    while not ctx.join(timeout=5):
        assert time.monotonic() < deadline, "rank 0 kept waiting on a rank that left"
    d = json.loads((tmp_path / "rank0.json").read_text())
    assert d["error"] is not None
    assert d["seconds"] < 60


def test_reference_arm_prints_once_under_torchrun():
    """`bench.py --impl reference` under torchrun with two ranks: rank 0 alone
    times the oracle and prints one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl",
           "reference", "--gpus", "2", "--config", "tiny", "--steps", "2", "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_bench_starts_its_own_ranks_without_torchrun():
    """`bench.py --gpus 2` launched as one plain process re-launches itself as two
    ranks under torch.distributed.run (the reference arm runs on CPU here)."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--config", "tiny", "--steps", "2",
           "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2


def test_bench_rejects_a_rank_count_that_differs_from_gpus():
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "3", "--config", "tiny", "--steps", "1",
           "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=120, env=env)
    assert p.returncode != 0 and "WORLD_SIZE" in p.stderr
