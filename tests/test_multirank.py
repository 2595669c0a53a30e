"""The multi-process path of bench.py on CPU with gloo (world size 2): rank
helpers (barrier, max and sum over ranks) and a 2-rank torchrun launch of the
reference arm, where rank 0 alone runs and prints one JSON line."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    mx = d.max(float(rank + 1) * 10.0)
    sm = d.sum(float(rank + 1))
    d.barrier()
    d.close()
    out.put((rank, mx, sm))


def test_dist_helpers_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    assert res == [(0, 20.0, 3.0), (1, 20.0, 3.0)]


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "0", "--layers", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "tokens/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0


def test_attention_reference_arm_two_ranks():
    """The decode-attention reference arm under a 2-rank torchrun: rank 0
    alone times the oracle and prints one line; the other rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "attn_decode", "--gpus", "2", "--steps", "3", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["config"]["workload"] == "attn_decode" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["d2h_bytes_per_step"] == 0


def _store_worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), LOCAL_WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    d = bench.Dist()
    d.init("gloo")
    calls = []

    def fill(view):
        calls.append(rank)
        view[...] = (np.arange(view.size, dtype=np.uint64) % 251).astype(np.uint8).reshape(view.shape)

    st = bench.HostStore((3, 5, 4096), fill, d, pin=False, tag="moe_store_test")
    a = st.tensor.numpy()
    ok = bool(st.shared) and np.array_equal(a.reshape(-1), (np.arange(a.size) % 251).astype(np.uint8))
    # one copy: a write by rank 0 is seen by rank 1
    d.barrier()
    if rank == 0:
        a[1, 2, 7] = 77
    d.barrier()
    seen = int(a[1, 2, 7])
    d.barrier()
    gone = not os.path.exists(os.path.join(bench.HostStore.SHM_DIR, f"moe_store_test_{port}"))
    st.close()
    d.close()
    out.put((rank, ok, calls, seen, gone))


def test_local_ranks_share_one_host_store():
    """Two local ranks (gloo): rank 0 creates and fills one shared segment,
    rank 1 maps it (it never fills), both see the same bytes and each other's
    writes, and the segment's name is gone once both have mapped it."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_store_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    assert res == [(0, True, [0], 77, True), (1, True, [], 77, True)]


def test_host_store_refuses_what_the_host_cannot_hold():
    sys.path.insert(0, ROOT)
    import bench
    import pytest

    class One:
        local_world, local = 1, 0

    class Eight:
        local_world, local = 8, 0

    with pytest.raises(RuntimeError, match="does not fit"):
        bench.HostStore((30, 128, 3345408), lambda v: None, One(), pin=False, avail=8 << 30)
    with pytest.raises(RuntimeError, match="local ranks share one host store"):
        bench.HostStore((30, 128, 3345408), lambda v: None, Eight(), pin=False, avail=8 << 30)
