"""bench.py host logic on CPU: multi-rank timing reduction (gloo, 2 ranks),
aggregation, seeding, clock parsing, peaks fallback and the reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    t = bench.reduce_max(10.0 + 5.0 * rank)          # rank 1 is slower
    q.put((rank, t, bench.rank_seed(2, rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [t for _, t, _ in res] == [15.0, 15.0]   # every rank sees the max
    assert len({s for _, _, s in res}) == world     # independent batches


def test_aggregate_is_whole_job_over_slowest_rank():
    assert bench.aggregate(100.0, 4, [2.0, 2.5, 1.0]) == pytest.approx(160.0)
    assert bench.reduce_max(3.5) == 3.5   # no process group: identity


def test_step_flops_formula():
    fwd, bwd = bench.step_flops([8192, 8192], 16, 128, True)
    assert fwd == pytest.approx(0.5 * 4 * 16 * 2 * 8192 ** 2 * 128)
    assert bwd == pytest.approx(2.5 * fwd)


def test_parse_clock_rows():
    text = ("1965, 1965, 700.5, Not Active, Not Active, Not Active, Active\n"
            "1350, 1965, 990.0, Not Active, Not Active, Not Active, Active\n"
            "1400, 1965, 980.0, Not Active, Not Active, Not Active, Not Active\n"
            "garbage\n")
    c = bench.parse_clock_rows(text)
    assert c["sm_mhz"] == 1400 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]


def test_peaks_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["bf16_tflops"] == 1590.0 and p["hbm_gbs"] == 6650.0


def test_tensor_peak_follows_length_of_timed_region():
    peaks = {"bf16_tflops": 1644.9, "bf16_tflops_sustained": 1403.3}
    # The driver's 20-step run lasts well under a second: burst clocks.
    assert bench.tensor_peak(peaks, 0.15) == (1644.9, "burst")
    # A seconds-long loop settles under the power cap.
    assert bench.tensor_peak(peaks, 1.5) == (1403.3, "sustained")


def test_default_workload_is_the_largest_single_gpu_configuration():
    from exact_io_aware_tmem_b200.workloads import WORKLOADS, flops
    w = WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert w.backward and w.D == 128 and w.N >= 4096
    def work(x):
        return sum(flops([x.N] * x.B, x.H, x.D, x.causal)) if not x.varlen else 0.0
    assert work(w) == max(work(x) for x in WORKLOADS.values())


def test_recorded_traffic_needs_matching_source(monkeypatch, tmp_path):
    (tmp_path / "profiles").mkdir()
    rec = {"bwd_dkdv_kernel": {"workload": "w", "source_sha": "stale", "bytes_per_launch": 5}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_sha", lambda *n: "fresh")
    assert bench.recorded_traffic("bwd_dkdv_kernel", "w") is None
    rec["bwd_dkdv_kernel"]["source_sha"] = "fresh"
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("bwd_dkdv_kernel", "w") == 5
    assert bench.recorded_traffic("bwd_dkdv_kernel", "other") is None
    # several workloads of one kernel: a list of records
    rec["bwd_dkdv_kernel"] = [dict(rec["bwd_dkdv_kernel"]),
                              {"workload": "v", "source_sha": "fresh", "bytes_per_launch": 7}]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("bwd_dkdv_kernel", "w") == 5
    assert bench.recorded_traffic("bwd_dkdv_kernel", "v") == 7
    assert real_root


def test_reference_arm_prints_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "f32_b1_h2_n128_d64", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "f32_b1_h2_n128_d64"], capture_output=True, text=True,
                         timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_warmup_below_three_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    import bench
    csrc = tmp_path / "exact_io_aware_tmem_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// header\nint a = 1;  // trailing\n\nint b = 2;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_sha("k.cu")
    (csrc / "k.cu").write_text("// a different header\n// more\nint a = 1;  // other words\nint b = 2;\n")
    assert bench.source_sha("k.cu") == h0
    (csrc / "k.cu").write_text("// header\nint a = 1;\nint b = 3;\n")
    assert bench.source_sha("k.cu") != h0
    # a quoted "//" inside code is code
    (csrc / "k.cu").write_text('// header\nconst char* s = "a//b";\nint b = 2;\n')
    h1 = bench.source_sha("k.cu")
    (csrc / "k.cu").write_text('// header\nconst char* s = "a//c";\nint b = 2;\n')
    assert bench.source_sha("k.cu") != h1


def test_decode_bytes_and_flops_formulas():
    from exact_io_aware_tmem_b200.workloads import (DECODE_WORKLOADS, decode_bytes,
                                                    decode_flops)
    # K and V, every cached token of every kv head, bf16
    assert decode_bytes([10, 6], 2, 64) == 2 * 16 * 2 * 64 * 2
    # two products of 2 * D flops per (query row, key)
    assert decode_flops([10, 6], 3, 4, 64) == 4.0 * 3 * 4 * 64 * 16
    w = DECODE_WORKLOADS["bf16_decode_b16_h32_kv8_d128_q1"]
    L = w.lengths()
    assert len(L) == 16 and min(L) >= 4096 and max(L) <= 32768
    assert L == w.lengths()       # seeded
