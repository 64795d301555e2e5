"""Host logic of bench.py that needs no GPU: the N>1 plumbing (process group,
barrier, max over ranks, whole-job value) as two gloo ranks on the CPU, the
reduced profiling case, and the source-hash gate on recorded DRAM traffic."""
import json
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from nvfp4_w4a4_gemm_quantize_b200 import synth  # noqa: E402


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "NVFP4_BENCH_BACKEND": "gloo"})
    try:
        r, w, local = bench.dist_setup(world)
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(w)
        # each rank's device time differs; the job time is the slowest rank's
        dev_ms = 10.0 + 5.0 * rank
        max_ms = bench.max_over_ranks(dev_ms, w, "cpu")
        # whole-job value: every rank's units over the max time (weak scaling)
        steps, flops = 4, 1.0e12
        value = w * steps * flops / (max_ms * 1e-3) / 1e12
        q.put((rank, max_ms, value))
        bench.barrier(w)
        dist.destroy_process_group()
    except BaseException as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_agree_on_max_time_and_value():
    world = 2
    port = 29500 + (os.getpid() % 2000)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] != "error" for r in res), res
    res.sort()
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 4 steps x 1 TFLOP in 15 ms
    assert all(abs(r[2] - 2 * 4 * 1.0 / 15e-3) < 1e-9 for r in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    bench.barrier(1)


def test_reference_arm_prints_only_on_rank_zero(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        ref_rows, warmup, steps = 1, 1, 1
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        ref_rows, warmup, steps = 1, 0, 1
    assert bench.run_reference(A()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_sample_is_bounded():
    """The reference arm's rows per step shrink with K so that the timed
    steps stay within the budget (at least one row, at most the layer)."""
    assert bench.ref_rows_for_budget(256, 0.5, 10, budget_s=60.0) == 3072      # 10 steps x 6 s
    assert bench.ref_rows_for_budget(256, 0.5, 500, budget_s=60.0) == 61       # 500 steps x 0.12 s
    assert bench.ref_rows_for_budget(256, 0.5, 10 ** 9) == 1
    assert bench.ref_rows_for_budget(256, 1e-6, 1) == 32768


def test_threaded_oracle_runner_equals_the_oracle():
    """Spreading the oracle over threads by 128-row slices changes nothing:
    the tensor scale, codes, scale layout and FP64 product are the whole-
    tensor oracle's, bit for bit (300 rows: a ragged last slice)."""
    import numpy as np
    import oracle
    x = synth.random_bf16((300, 512), seed=5, dist="token_scaled")
    w = synth.random_bf16((200, 512), seed=6, scale=0.02)
    r = bench.OracleRunner(4)
    assert r.tensor_scale(x) == oracle.tensor_scale(x)
    a, b = r.quantize(x), r.quantize(w)
    a0, b0 = oracle.quantize(x), oracle.quantize(w)
    for u, v in zip(a, a0):
        assert np.array_equal(u, v)
    for u, v in zip(b, b0):
        assert np.array_equal(u, v)
    assert np.array_equal(r.gemm(a, b), oracle.gemm_w4a4(*a0, *b0))


def test_reduced_case_selects_layers_and_rows():
    class A:
        layers, m = "fc1,fc2", 4096
    wl = bench.reduced(synth.WORKLOADS["video_dit"], A())
    assert [L.name for L in wl.layers] == ["fc1", "fc2"]
    assert all(L.M == 4096 for L in wl.layers)

    class B:
        layers, m = "", 0
    assert bench.reduced(synth.WORKLOADS["video_dit"], B()) is synth.WORKLOADS["video_dit"]


def test_recorded_traffic_is_void_when_sources_change(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "nvfp4_w4a4_gemm_quantize_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (prof / "k.txt").write_text(f"kernel: k\nsource_sha256: {h}\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("k.txt") == 12345
    assert bench.profiled_traffic("missing.txt") is None
    (src / "k.cu").write_text("// kernel v2\n")
    assert bench.kernel_source_hash() != h
    assert bench.profiled_traffic("k.txt") is None
    # a summary that names its sources is voided only by those
    (src / "other.cu").write_text("// unrelated kernel\n")
    h2 = bench.kernel_source_hash(["k.cu"])
    (prof / "k2.txt").write_text(f"source_files: k.cu\nsource_sha256: {h2}\ndram_bytes_per_launch: 7\n")
    assert bench.profiled_traffic("k2.txt") == 7
    (src / "other.cu").write_text("// unrelated kernel, changed\n")
    assert bench.profiled_traffic("k2.txt") == 7
    (src / "k.cu").write_text("// kernel v3\n")
    assert bench.profiled_traffic("k2.txt") is None
