"""The bench's multi-rank plumbing on CPU: two gloo ranks run dist_setup,
dist_barrier and dist_max the way `bench.py --gpus 2` does under torchrun
(replicas only: the max over ranks of the timed region is the one exchange)."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, types
sys.path.insert(0, sys.argv[1])
import torch
import bench
args = types.SimpleNamespace(gpus=2)
world, rank, local = bench.dist_setup(args)
assert world == 2 and rank == local
bench.dist_barrier(world)
got = bench.dist_max(10.0 + rank * 5.5, world)
assert got == 15.5, got
bench.dist_barrier(world)
import torch.distributed as dist
dist.destroy_process_group()
print("ok", rank)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_barrier_and_max_over_ranks():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, WORLD_SIZE="2", RANK=str(r), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD, ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            p.kill()
            out, _ = p.communicate()
        outs.append((p.returncode, out))
    for r, (rc, out) in enumerate(outs):
        assert rc == 0 and f"ok {r}" in out, out[-2000:]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(3.25, 1) == 3.25
    bench.dist_barrier(1)
