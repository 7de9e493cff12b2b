"""bench.py host logic on CPU. The N>1 plumbing with gloo (world size 2): every rank
gets the slowest rank's time, and the reference arm runs on rank 0 only. Also the
quantizer's HBM-roofline arithmetic."""
import os
import socket
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        results[rank] = bench.max_over_ranks(1.5 + rank, True, device="cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert dict(results) == {0: 2.5, 1: 2.5}


class RefArgs:
    workload, n, warmup, steps, dtype, hadamard, settle_s, fp8_q = "tiny", None, 3, 1, "fp8", False, 1.0, "fused"


def test_reference_arm_other_ranks_do_no_work(capsys):
    import bench

    bench.run_reference(RefArgs(), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_quantizer_summary_counts_five_bytes_per_element():
    """Per-head scales: the absmax pass reads 2 bytes, the encode pass reads 2 and
    writes 1, over every element of Q, K and V."""
    import bench
    import workloads
    w = workloads.gqa7b()
    s = bench.quantizer_summary(0.1, w, 6545.3)
    assert s["algorithmic_bytes"] == 5 * (32 + 8 + 8) * 128 * 16384
    assert abs(s["achieved"] - s["algorithmic_bytes"] / 1e-4 / 1e9) < 1e-6
    assert abs(s["frac"] - s["achieved"] / 6545.3) < 1e-12 and s["bound"] == "hbm"
    m = bench.quantizer_summary(0.1, workloads.mla(), 6545.3)
    assert m["algorithmic_bytes"] == 5 * 16 * (192 + 192 + 128) * 16384
    assert bench.quantizer_summary(0.0, w, 6545.3) is None
    # Q quantised inside the attention kernel: only K and V pass through the quantizer;
    # Q per 128-token block: one pass over Q (2 bytes read, 1 written)
    kv = 5 * (8 + 8) * 128 * 16384
    assert bench.quantizer_summary(0.1, w, 6545.3, q_bytes=0.0)["algorithmic_bytes"] == kv
    assert bench.quantizer_summary(0.1, w, 6545.3, q_bytes=3.0)["algorithmic_bytes"] == kv + 3 * 32 * 128 * 16384


def test_reference_arm_line_on_rank_zero(capsys):
    """The reference arm's JSON line: the oracle on a bounded sample, the same workload
    string as the GPU arm, and the keys the line must carry."""
    import json
    import bench

    t0 = time.perf_counter()
    bench.run_reference(RefArgs(), rank=0, world=1)
    wall_ms = (time.perf_counter() - t0) * 1e3
    line = json.loads(capsys.readouterr().out.strip())
    # a step is a measured sample (one query head), so the timed steps fit in the run
    assert 0 < line["ms_per_step"] * line["steps"] <= wall_ms
    w = bench.make_workload("tiny", None)
    assert line["config"] == bench.run_config(RefArgs(), w, 1)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.workload_desc(bench.make_workload("tiny", None))
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["steps"] == 1 and line["warmup"] == 3 and line["dtype"] == "f64"


def test_kernel_hash_ignores_comments_and_follows_code():
    """The traffic figures are keyed to a hash of the kernel code: a comment or
    blank-space edit leaves it unchanged, a code edit changes it."""
    import bench
    code = "int f(int x) {\n  return x + 1;  // add one\n}\n/* block\n comment */\n"
    assert bench._code_only(code) == bench._code_only("int f(int x) { return x + 1; }")
    assert bench._code_only(code) != bench._code_only("int f(int x) { return x + 2; }")
    assert len(bench.kernel_sources_sha()) == 16


@pytest.mark.parametrize("env,fused,expect", [
    ({}, False, "attn_fwd_kernel<128,128,fp8,lean,block-scaled>"),
    ({"B200ATTN_FP8_P": "lean"}, False, "attn_fwd_kernel<128,128,fp8,lean>"),
    ({"B200ATTN_FP8_P": "mufu"}, False, "attn_fwd_kernel<128,128,fp8,mufu>"),
    ({"B200ATTN_SHARED_S": "0"}, False, "attn_fwd_kernel<128,128,fp8,lean,private-S>"),
    ({"B200ATTN_FP8_PAIR": "1"}, False, "attn_fwd_pair_kernel<128,128,fp8,lean>"),
    ({"B200ATTN_FP8_TILE": "1"}, False, "attn_fwd_tile_kernel<128,128,fp8,lean>"),
    ({}, True, "attn_fwd_kernel<128,128,fp8,lean,block-scaled,fused-q>"),
    ({"B200ATTN_FP8_P": "mufu"}, True, "attn_fwd_kernel<128,128,fp8,mufu,fused-q>"),
])
def test_kernel_name_follows_the_library_dispatch(env, fused, expect, monkeypatch):
    """bench.py names the kernel the library runs for the FP8 step under each switch."""
    import bench
    import workloads
    for k in ("B200ATTN_FP8_P", "B200ATTN_SHARED_S", "B200ATTN_FP8_PAIR", "B200ATTN_FP8_TILE"):
        monkeypatch.delenv(k, raising=False)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    assert bench.kernel_name("fp8", workloads.gqa7b(), fused_q=fused) == expect


def test_varlen_workload_recipe_is_fixed():
    """bench.py --varlen: 24 seeded log-uniform lengths in [256, 8192]; the same on every call."""
    import bench
    a, b = bench.varlen_lengths(), bench.varlen_lengths()
    assert a == b and len(a) == 24
    assert all(256 <= n <= 8192 for n in a)
    assert a != bench.varlen_lengths(seed=6)
