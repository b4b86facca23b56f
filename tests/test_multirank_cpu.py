"""The multi-rank path of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job rate (independent replicas, weak scaling).  No GPU is involved."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 2.0 + 3.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, "cpu")
        out[rank] = (ms, bench.whole_job_rate(1e12, ms, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    for r in range(2):
        ms, rate = res[r]
        assert ms == 5.0
        # two ranks x 1 TFLOP each over the slowest rank's 5 ms
        assert abs(rate - 2 * 1e12 / 5e-3 / 1e12) < 1e-9


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
    assert abs(bench.whole_job_rate(2e12, 4.0, 1) - 500.0) < 1e-9


def test_reference_arm_prints_one_json_line():
    """bench.py --impl reference times the fp64 oracle on the host and prints the line."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "blocksparse_mha_s256_d64", "--steps", "2", "--warmup", "3",
                        "--ref-seconds", "0.2"], capture_output=True, text=True, timeout=300,
                       cwd=root)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "blocksparse_mha_s256_d64"
