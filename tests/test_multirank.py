"""Rank logic of bench.py on CPU with gloo, world size 2: max-over-ranks timing, and the
reference arm under torchrun printing one line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    ws, r, _ = bench._dist()
    assert ws == world and r == rank
    slowest = bench._max_over_ranks(1.5 * (rank + 1), ws, "cpu")
    bench._barrier(ws)
    q.put((r, slowest))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 3.0), (1, 3.0)]


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1", "--ref-items", "1", "--workload", "tiny"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def _split_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    ws, r, _ = bench._dist()
    w = W.scaled(W.WORKLOADS["tiny"], H=5)                 # five heads over two ranks: 3 + 2
    heads = bench.head_slice(w.H, r, ws)
    inp = W.make_inputs(w, seed=3, heads=heads)
    eff = W.effective_flops(inp.w, inp.kv_cnt, inp.kv_idx)
    total = bench._sum_over_ranks(eff, ws, "cpu")
    q.put((r, list(heads), eff, total, inp.K.sum().item(), inp.kv_cnt.sum().item()))
    torch.distributed.destroy_process_group()


def test_split_heads_partition_the_workload_with_gloo():
    """--split-heads: the ranks' head slices partition the heads, each slice holds exactly those
    heads of the full workload, and the job's effective FLOPs (summed over ranks) are the full
    workload's."""
    sys.path.insert(0, ROOT)
    import workloads as W
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got[0][1] == [0, 1, 2] and got[1][1] == [3, 4]
    w = W.scaled(W.WORKLOADS["tiny"], H=5)
    full = W.make_inputs(w, seed=3)
    assert abs(got[0][3] - W.effective_flops(w, full.kv_cnt, full.kv_idx)) < 1e-6 * got[0][3]
    assert got[0][3] == got[1][3] == got[0][2] + got[1][2]
    for r, heads, _, _, ksum, cnt in got:
        assert abs(ksum - full.K[:, heads].sum().item()) < 1e-3 * max(1.0, abs(ksum))
        assert cnt == full.kv_cnt[:, heads].sum().item()


def test_traffic_record_follows_the_kernel_code_not_its_comments(tmp_path):
    """The bench line's attention traffic comes from a committed capture whose record names a hash
    of the kernel's code: a comment edit keeps it, a code edit changes it."""
    import bench
    src = tmp_path / "k.cu"
    src.write_text("// header\nint f(int x) {  /* body */\n  return x + 1;  // one\n}\n")
    h0 = bench.source_code_sha1(str(src))
    src.write_text("// another header\n\nint f(int x) { /* other words */ return x + 1; }\n")
    assert bench.source_code_sha1(str(src)) == h0
    src.write_text("int f(int x) { return x + 2; }\n")
    assert bench.source_code_sha1(str(src)) != h0
