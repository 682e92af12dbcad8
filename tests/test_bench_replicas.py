"""The replica (N > 1) plumbing of bench.py on CPU: two gloo ranks, max-over-ranks timing, and
the reference arm printing only on rank 0. The data path has no collective: each rank runs an
independent replica, so only the measurement plumbing is exercised here."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    m = bench.max_over_ranks(float(rank + 1) * 1.5, w)
    bench.barrier(w)

    class A:
        workload = "tiny"
        steps = 2
        warmup = 1
        gpus = world
        ref_tokens = 8
        T = None
        E = None
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(A, w, r)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, m, rc, buf.getvalue()))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, m, rc, out = q.get(timeout=300)
        res[rank] = (m, rc, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 3.0          # max over ranks
    assert res[0][1] == res[1][1] == 0
    assert res[1][2] == ""                          # only rank 0 prints
    line = json.loads(res[0][2].strip())
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # the measured step time of the sampled tokens, and the main arm's config object
    import bench
    from mixture_experts_layer_block_b200 import configs
    assert line["config"] == bench.config_of(configs.TINY, "bf16", 2)
    n = line["tokens_per_step"]
    assert 1 <= n <= 8 and abs(line["value"] * line["ms_per_step"] * 1e-3 - n) < 1e-6 * n


def test_reference_arm_mxfp8_line():
    """--impl reference --precision mxfp8 times the oracle's MXFP8 layer and says so."""
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--precision",
                        "mxfp8", "--workload", "tiny", "--steps", "1", "--warmup", "0", "--ref-tokens", "4"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["precision"] == "mxfp8" and line["config"]["workload"] == "tiny"
