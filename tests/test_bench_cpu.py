"""bench.py's host-side pieces, without a GPU: the peak table, the ncu traffic lookup
and the reference arm (the CPU oracle) end to end, with its JSON line."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_peaks_and_traffic():
    pk = bench._peaks()
    assert pk["hbm"] > 1000 and pk["bf16"] > 100 and pk["source"] in ("measured", "fallback")
    for kernel in bench.KERNEL_DEVICE_SOURCES:
        t = bench._traffic(kernel)
        assert t is None or t > 0


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    """One gloo rank: the bench's max-over-ranks reduction on rank-dependent times."""
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench as b
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = b._max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], dist, "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(got, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks(tmp_path):
    """N > 1 host path: every rank ends with the slowest rank's times (gloo, world 2)."""
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert json.load(open(tmp_path / f"rank{r}.json")) == [2.0, 10.0, 0.5]
    assert bench._max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]


def test_reference_arm_under_torchrun_two_ranks():
    """`--impl reference` launched like the driver's N = 2 run: rank 0 alone prints the line,
    rank 1 exits 0 without work, and no process group is needed."""
    port = _free_port()
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                          "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                          "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
