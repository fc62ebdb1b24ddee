"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): the timing
reduction takes the maximum over ranks, and the reference arm under torchrun
prints exactly one JSON line (rank 0) while the other rank exits cleanly."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1",
           "--workload", "acausal_n1k_f32"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _args(*argv):
    sys.path.insert(0, ROOT)
    import bench
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench, bench.parse()
    finally:
        sys.argv = old


def test_workload_overrides():
    """--block, --clusters, --iters change the named workload; invalid combinations stop
    before anything runs."""
    bench, a = _args("--workload", "causal_n16k_bf16", "--block", "1024", "--clusters", "32",
                     "--iters", "3")
    w = bench.workload_of(a)
    assert (w.block, w.Cq, w.Ck, w.iters) == (1024, 32, 32, 3)
    assert w.N == 16384 and w.name == "causal_n16k_bf16"
    bench, a = _args("--monopole")
    assert bench.workload_of(a).mode == "acausal"
    for bad in (["--block", "512"],                                   # acausal has no blocks
                ["--workload", "causal_n16k_bf16", "--block", "1000"],  # does not divide N
                ["--workload", "causal_n16k_bf16", "--monopole"],
                ["--monopole", "--partial-dipole"],
                ["--clusters", "100000"],
                ["--heads", "9"],                                      # 8 problems at 8k
                ["--refine-form", "summary", "--monopole"],            # forms: full method only
                ["--workload", "causal_n16k_bf16", "--refine-form", "pair"]):
        bench, a = _args(*bad)
        with pytest.raises(SystemExit):
            bench.workload_of(a)


def test_heads_slice_and_refinement_form():
    """--heads keeps the first H problems of a workload (B = 1); the bench names the
    refinement form the library chooses (summary form at N = 64k, D = 128 only)."""
    bench, a = _args("--workload", "acausal_n64k_d128_bf16", "--heads", "2")
    w = bench.workload_of(a)
    assert (w.B, w.H, w.N, w.D) == (1, 2, 65536, 128)
    assert bench.refine_form_of(w) == "summary"
    assert bench.refine_form_of(w, "pair") == "pair"
    bench, a = _args()
    w8 = bench.workload_of(a)
    assert bench.refine_form_of(w8) == "pair" and bench.refine_form_of(w8, "summary") == "pair"


def test_algorithmic_flops_of_the_block_sweep():
    """The refinement's algorithmic flops per launch: at S = N/2 one square of N/2 x N/2,
    and the multi-level count sums the squares of every level."""
    bench, a = _args("--workload", "causal_n16k_bf16", "--block", "8192")
    w = bench.workload_of(a)
    n = 8192
    one = min(2.0 * 64 * n * 64 * 64 + 2.0 * n * 64 * 64 * 64, 2.0 * n * n * 128)
    assert bench.algorithmic_flops(w) == w.B * w.H * one
    bench, a = _args("--workload", "causal_n16k_bf16", "--block", "4096")
    w2 = bench.workload_of(a)
    sq = lambda s: min(2.0 * 64 * s * 64 * 64 + 2.0 * s * 64 * 64 * 64, 2.0 * s * s * 128)
    assert bench.algorithmic_flops(w2) == w2.B * w2.H * (sq(8192) + 2 * sq(4096))
