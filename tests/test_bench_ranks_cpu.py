"""The bench's multi-rank timing logic on CPU: two gloo ranks, each reports its own
device time, every rank gets the slowest one (no GPU, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.max_over_ranks(10.0 + 5.0 * rank, world, dist, device="cpu")
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 15.0, 1: 15.0}


def test_max_over_ranks_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_reference_arm_runs_on_cpu(capsys, monkeypatch):
    """--impl reference times the fp64 oracle on the host (tiny step count)."""
    import json
    import sys
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "ffn", "--steps", "2",
                                      "--warmup", "3"])
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["host_cpus"] == os.cpu_count() and "cores" in line["cpu_baseline"]


def test_reference_arm_tiny_fp32_and_workload_order(capsys, monkeypatch):
    """The default workload list ends with the headline FFN block; the tiny fp32 block's
    reference line runs the oracle on all 8 rows per step."""
    import json
    import sys
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "fp32", "--steps", "2",
                                      "--warmup", "3"])
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"]["workload"] == "ffn_fp32_M8_h64_f256_t2" and line["value"] > 0

    class A:
        workload, impl, mode, t, h = "all", "ours", "fused", 4, "22528"
    names = [w.name for w in bench.make_workloads(A)]
    assert names[-1] == "ffn_bf16_M2048_h4096_f16384_t4" and len(names) == len(set(names)) == 9
    assert "ffn_bwd_bf16_M2048_h4096_f16384_t4" in names
    assert "attn_bwd_bf16_B2_S2048_h4096_H32_d128_t4_causal" in names
    A.impl = "reference"
    assert bench.make_workloads(A)[-1].headline


def test_kernel_source_hash_ignores_comments_only():
    """The ncu figures are keyed on the kernel sources without comments and layout: a
    comment edit keeps them, any code edit drops them."""
    import bench
    code = "int f(int a) {\n  return a + 1;  // one more\n}\n/* block\n   comment */\n"
    assert bench._code_only(code) == "int f(int a) { return a + 1; }"
    assert bench._code_only(code.replace("// one more", "// a different note")) == bench._code_only(code)
    assert bench._code_only(code.replace("a + 1", "a + 2")) != bench._code_only(code)
    assert len(bench._csrc_sha()) == 16
    # each launch is keyed on the sources that define it
    assert bench._kernel_sha("attention") != bench._kernel_sha("gemm_row_fused_reduce")
    assert bench._kernel_sha("gemm_column_act") == bench._kernel_sha("gemm_row_fused_reduce")
    assert bench._kernel_sha("not_a_kernel") == bench._csrc_sha()


def test_reference_arm_attention_backward(capsys, monkeypatch):
    """The attention backward's reference line: the oracle on one head over one sequence
    per step, credited 1/(B*H) of the workload's FLOPs."""
    import json
    import sys
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "attn_bwd", "--steps", "1",
                                      "--warmup", "3"])
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["config"]["workload"] == "attn_bwd_bf16_B2_S2048_h4096_H32_d128_t4_causal"
    assert line["value"] > 0 and "one head over one sequence" in line["cpu_baseline"]["sample"]
