"""The multi-rank path of bench.py on the host cores (gloo, world size 2).

bench.py runs one process per GPU and reports the maximum device time over
ranks; without a GPU its process group falls back to gloo, which lets these
tests check, on CPU, the barrier and the maximum over ranks that the timing
uses, and the reference arm under torchrun, where rank 0 alone prints one
JSON line and the other rank leaves without work."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="the host (gloo) path of the multi-rank code")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, out):
    os.environ.update(WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    ctx = bench.init_dist(2)
    bench.barrier(ctx)
    value = bench.max_over_ranks(ctx, 1.5 + rank)
    bench.barrier(ctx)
    out.put((rank, ctx["backend"], ctx["world"], value))
    ctx["dist"].destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    spawn = mp.get_context("spawn")
    q = spawn.Queue()
    port = _free_port()
    procs = [spawn.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, "gloo", 2, 2.5), (1, "gloo", 2, 2.5)]


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"].startswith("mistral7b_32layers")
