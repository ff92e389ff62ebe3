"""Host-side logic of bench.py on the CPU: the whole-job aggregate, the
max-over-ranks timing with two gloo ranks, the reference arm's rank rule, the
workload table and the profile lookup that feeds `roofline.traffic`."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_whole_job_value_counts_every_rank():
    # 2 * M * N * K ops per step, 10 steps, 4 ranks, 0.5 s for the slowest rank
    ops = 2.0 * 4096 * 4096 * 4096
    v = bench.whole_job_value(ops, steps=10, world=4, max_seconds=0.5)
    assert v == pytest.approx(ops * 10 * 4 / 0.5 / 1e12)


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        # each rank's "elapsed time" differs; every rank must see the maximum
        got = bench.reduce_max(10.0 + 5.0 * rank)
        bench.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_reduce_max_is_identity_without_a_process_group():
    assert bench.reduce_max(3.25) == 3.25


def test_reference_arm_runs_on_rank_zero_only():
    ns = type("A", (), dict(workload="tiny", steps=3, warmup=3, ref_seconds=0.5))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(ns, world=2, rank=1, local=1)
    assert buf.getvalue() == ""  # other ranks exit without work
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(ns, world=1, rank=0, local=0)
    line = buf.getvalue().strip()
    import json

    rec = json.loads(line)
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


def test_every_workload_resolves_to_a_case():
    for name in bench.WORKLOADS:
        case = bench.get_case(name)
        if bench.is_attention(name):
            assert case.D == 128 and case.L % 8 == 0 and case.B * case.H >= 1
            continue
        assert case.M > 0 and case.K % 32 == 0 and case.N % 8 == 0
        assert bench.is_w4(name) == ("w4a8" in case.name)
    assert bench.is_gated("dit_mlp_gated") and not bench.is_gated("dit_mlp")


def test_traffic_lookup_follows_the_source_hash(tmp_path):
    csrc = os.path.join(ROOT, "w4a8_quantized_gemm_token_b200", "csrc")
    cases = [("w8a8_gemm_kernel", "gemm_w8a8.cu", "dit_mlp"), ("w4a8_gemm_kernel", "gemm_w4a8.cu", "w4a8_m4096"),
             ("w4a8_gemv1_kernel", "gemv1_w4a8.cu", "w4a8_m1")]
    for tag, src, workload in cases:
        path = os.path.join(csrc, src)
        t = bench.traffic_from_profile(tag, path, workload)
        assert t is None or t > 0  # a number only while the summary matches the source
        # another workload of the same kernel never takes the summary's bytes
        assert bench.traffic_from_profile(tag, path, "tiny") is None
        # any other file never matches the committed hash
        other = tmp_path / src
        other.write_bytes(open(path, "rb").read() + b"\n// edited\n")
        assert bench.traffic_from_profile(tag, str(other), workload) is None


def test_launch_counts_per_call():
    """The launches a W4A8 call makes follow its plan: the GEMM route is the
    quantization kernel, the plane count, the plane build, the gated fold and
    the plane GEMM (5), on a prepared weight 3; W8A8 is the quantization
    kernel + the GEMM."""
    from w4a8_quantized_gemm_token_b200 import build

    build.build()
    from w4a8_quantized_gemm_token_b200 import binding as qk

    assert bench.is_prepared("w4a8_m4096_prepared") and not bench.is_prepared("w4a8_m4096")
    assert all(bench.is_w4(n) for n in bench.WORKLOADS if bench.is_prepared(n))
    assert bench.launches_per_call(4096, 4096, 4096, True, False, qk) == 5
    assert bench.launches_per_call(4096, 4096, 4096, True, False, qk, prepared=True) == 3
    assert bench.launches_per_call(16384, 3072, 12288, False, False, qk) == 2
    assert bench.launches_per_call(1, 4096, 4096, True, False, qk) == 1   # the GEMV quantizing x
