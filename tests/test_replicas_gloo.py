"""Multi-process path on CPU (gloo, world size 2): sharding a packed batch
over ranks is exact (each rank computes its share -- here with the oracle,
which stands in for the GPU kernel on a CPU machine -- and the gathered result
equals the single-process result bit for bit), and the timing reduction takes
the max over ranks."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import la_inputs
from linear_attention_blocked_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_packed_balances_and_covers():
    lens = la_inputs.varlen_lengths(8, 1024, 65536, seed=3)
    for world in (1, 2, 3, 4, 8, 11):
        groups = replicas.shard_packed(lens, world)
        assert len(groups) == world
        assert groups[0][0] == 0 and groups[-1][1] == len(lens)
        for (a, b), (c, _) in zip(groups, groups[1:]):
            assert a <= b == c
        if world <= len(lens):
            tok = [int(lens[a:b].sum()) for a, b in groups]
            assert max(tok) - min(tok) <= 2 * int(lens.max())
    assert replicas.shard_packed([], 2) == [(0, 0), (0, 0)]


def _worker(rank, world, port, result_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        lens = [37, 5, 64, 0, 91, 12, 40]
        H, D = 2, 8
        cu = la_inputs.cu_seqlens_from_lengths(lens)
        q, k, v = la_inputs.qkv((int(cu[-1]), H, D), seed=7, scale=0.5)
        Q, K, V = la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v)
        group = replicas.shard_packed(lens, world)[rank]
        t0, t1, lcu = replicas.local_problem(cu, group)
        out, st = oracle.recurrent(Q[t0:t1], K[t0:t1], V[t0:t1], lcu)
        # gather every rank's share on every rank (host-side; no data-path collective on GPUs)
        shares = [None] * world
        dist.all_gather_object(shares, (group, out, st))
        slowest = replicas.max_over_ranks(float(rank + 1))
        if rank == 0:
            full, fst = oracle.recurrent(Q, K, V, cu)
            ok = slowest == float(world)
            for (a, b), o, s in shares:
                ta, tb = int(cu[a]), int(cu[b])
                ok &= np.array_equal(o, full[ta:tb]) and np.array_equal(s, fst[a:b])
            ok &= sum(b - a for (a, b), _, _ in shares) == len(lens)
            with open(result_path, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_single_process(tmp_path, oracle_mod):
    world = 2
    result = tmp_path / "result.txt"
    mp.start_processes(_worker, args=(world, _free_port(), str(result)), nprocs=world, join=True,
                       start_method="spawn")
    assert result.read_text() == "ok"


def test_max_over_ranks_without_group():
    assert replicas.max_over_ranks(3.5) == 3.5


def test_bench_reference_arm_under_two_ranks(tmp_path):
    """The reference arm launched as the multi-GPU run is launched: rank 0 alone
    runs the oracle and prints one JSON line; the other rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "3", "--warmup", "3", "--ref-seconds", "1"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
