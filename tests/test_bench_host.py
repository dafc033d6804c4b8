"""Host-side logic of bench.py without a GPU: clock parsing and rejection,
max/sum over ranks with a 2-process gloo group, and the reference arm."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parse_clock_lines_and_rejection():
    text = "\n".join([
        "1800, 1965, 900.1, Not Active, Not Active, Not Active, Active",
        "1327, 1965, 997.0, Not Active, Not Active, Not Active, Active",
        "1400, 1965, 990.0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ])
    clk = bench.parse_clock_lines(text)
    assert clk["sm_mhz"] == 1400 and clk["sm_max_mhz"] == 1965 and clk["samples"] == 3
    assert clk["reasons"] == ["sw_power_cap"]
    assert not bench.clocks_rejected(clk)
    hot = bench.parse_clock_lines("1500, 1965, 1000, Not Active, Active, Not Active, Not Active")
    assert bench.clocks_rejected(hot)
    locked = bench.parse_clock_lines("700, 1965, 400, Not Active, Not Active, Not Active, Not Active")
    assert bench.clocks_rejected(locked)
    assert bench.parse_clock_lines("") is None


def test_recorded_traffic_follows_the_kernel_sources(monkeypatch):
    rec_path = os.path.join(ROOT, "profiles", "dram_traffic_T16384_d5120_V152064.json")
    with open(rec_path) as f:
        rec = json.load(f)
    # a workload without a capture has no recorded traffic
    assert bench.recorded_traffic(64, 128, 1024, "dw_gemm") is None
    assert bench.recorded_traffic(16384, 5120, 152064, "validate") is None
    # with the sources the capture was taken with, the record's per-launch bytes come back
    got = bench.recorded_traffic(16384, 5120, 152064, "dw_gemm")
    k = rec["kernels"]["dw_gemm"]
    expect = k["dram_read_bytes_per_launch"] + k["dram_write_bytes_per_launch"]
    assert got is None or got == expect
    # any other source set (a changed kernel) gives null
    monkeypatch.setitem(bench._TRAFFIC_SOURCES, "gemm", ["resolver.cu"])
    assert bench.recorded_traffic(16384, 5120, 152064, "dw_gemm") is None


def test_source_digest_ignores_comments():
    code = "int a = 1;  // one\n\n/* block\n comment */int b = 2;\n"
    assert bench.source_code_only(code) == "int a = 1;\nint b = 2;"
    assert bench.source_code_only(code.replace("one", "uno")) == bench.source_code_only(code)
    assert bench.source_code_only(code.replace("= 2", "= 3")) != bench.source_code_only(code)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.reduce_max(10.0 + rank, torch.device("cpu"))
        sm = bench.reduce_sum(1.5 * (rank + 1), torch.device("cpu"))
        bench.barrier()
        q.put((rank, mx, sm))
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 11.0, 4.5), (1, 11.0, 4.5)]


def test_reduce_without_group_is_identity():
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5


def test_reference_arm_only_on_rank_zero():
    class A:
        workload = 1
        steps = 1
        warmup = 0
        ref_rows = 2
    assert bench.run_reference(A(), rank=1, world=2) is None


def test_reference_arm_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "1", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert res.returncode == 0, res.stderr
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_recorded_traffic_per_row_scales_to_the_average_launch(tmp_path, monkeypatch):
    import hashlib
    csrc = tmp_path / "sampling_transform_lm_b200" / "csrc"
    csrc.mkdir(parents=True)
    h = hashlib.sha256()
    for name in bench._TRAFFIC_SOURCES["resolve"]:
        (csrc / name).write_text(f"int {name.split('.')[0]} = 1;  // a comment\n")
        h.update(bench.source_code_only((csrc / name).read_text()).encode())
    (tmp_path / "profiles").mkdir()
    rec = {"sources": {"resolve": h.hexdigest()[:16]},
           "kernels": {"resolve": {"dram_bytes_per_row": 100.0}}}
    (tmp_path / "profiles" / "dram_traffic_T8_d4_V16.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic(8, 4, 16, "resolve", 2) == 400  # 8 rows over 2 launches
    assert bench.recorded_traffic(8, 4, 16, "resolve") is None    # launches unknown
    (csrc / "resolver.cu").write_text("int changed = 2;\n")
    assert bench.recorded_traffic(8, 4, 16, "resolve", 2) is None


def test_config_names_the_chunk_the_library_picks():
    import sampling_transform_lm_b200 as sts
    import workloads

    wl4, wl3 = workloads.WORKLOADS[4], workloads.WORKLOADS[3]
    cfg = bench.workload_config(wl4, wl4.T, wl4.V, 1)
    # the library's default for the headline shape: 111 x 256 columns
    assert cfg["vocab_chunk"] == sts.sts_vocab_chunk(wl4.T, wl4.d, wl4.V) == 28416
    assert (wl4.T // 128) * (cfg["vocab_chunk"] // 256) % 148 == 0  # dz tiles: whole waves
    assert (wl4.d // 128) * (cfg["vocab_chunk"] // 256) % 148 == 0  # dW tiles: whole waves
    # a workload that states its chunk keeps it; a small vocabulary clamps it
    assert bench.workload_config(wl3, wl3.T, wl3.V, 1)["vocab_chunk"] == 8192
    wl1 = workloads.WORKLOADS[1]
    assert bench.workload_config(wl1, wl1.T, wl1.V, 1)["vocab_chunk"] == 1024


def test_recorded_gemm_traffic_scales_to_the_average_launch(tmp_path, monkeypatch):
    import hashlib
    csrc = tmp_path / "sampling_transform_lm_b200" / "csrc"
    csrc.mkdir(parents=True)
    h = hashlib.sha256()
    for name in bench._TRAFFIC_SOURCES["gemm"]:
        (csrc / name).write_text(f"int {name.split('.')[0]} = 1;\n")
        h.update(bench.source_code_only((csrc / name).read_text()).encode())
    (tmp_path / "profiles").mkdir()
    T, d, V = 8, 4, 16
    rec = {"sources": {"gemm": h.hexdigest()[:16]},
           "kernels": {"logits_gemm": {"dram_bytes_per_logit": 10.0},
                       "dw_gemm": {"dram_read_bytes_per_launch": 900,
                                   "dram_write_bytes_per_launch": 100,
                                   "capture_flops": 2 * T * d * 8}}}
    (tmp_path / "profiles" / f"dram_traffic_T{T}_d{d}_V{V}.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # projection: 8 rows over 2 launches, 16 logits each, 10 bytes per logit
    assert bench.recorded_traffic(T, d, V, "logits_gemm", 2) == 4 * 16 * 10
    assert bench.recorded_traffic(T, d, V, "logits_gemm") is None
    # a full-chunk launch (8 columns) scaled to the average of 4 launches over V = 16
    assert bench.recorded_traffic(T, d, V, "dw_gemm") == 1000
    assert bench.recorded_traffic(T, d, V, "dw_gemm", 4) == 500
