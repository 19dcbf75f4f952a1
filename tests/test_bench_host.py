"""Host logic of bench.py on CPU: the multi-rank timing reduction (gloo,
world size 2), the algorithmic-work accounting, and the reference arm's JSON
line (the fp64 oracle on the host cores) on the tiny workload."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r = bench.init_dist("gloo")
    assert (w, r) == (world, rank)
    bench.barrier()
    got = bench.max_over_ranks(10.0 + 5.0 * rank)       # rank-dependent step time
    q.put((rank, got))
    bench.cleanup()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def _share_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    bench.init_dist("gloo")
    w = synth.BY_NAME["tiny_f32_F32_P64_C64"]
    got = bench.shared_host_inputs(w, rank, world, pinned=False)
    ref = bench.host_inputs(w, pinned=False)
    same = all(got[n].shape == ref[n].shape and bool((got[n] == ref[n]).all())
               for n in bench.INPUT_NAMES)
    q.put((rank, same))
    bench.cleanup()


def test_inputs_generated_once_and_broadcast_gloo_world2():
    """Rank 0 generates the seeded inputs and broadcasts them; every rank ends
    with exactly what host_inputs() gives."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_share_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: True, 1: True}


def test_kernel_work_accounting():
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    work = bench.kernel_work(w)
    S = 2560 * 1024 * 320 * 2
    assert work["dual_attn"]["bytes"] == 4 * S
    assert work["groupnorm_global"]["bytes"] == 3 * S
    assert work["temporal_conv"]["flops"] == 6 * 320 * 320 * 2560 * 1024


def test_reference_arm_prints_contract_line(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny_f32_F32_P64_C64", "--steps", "2",
                    "--warmup", "1", "--cpu-seconds", "0.5"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(bench.parse_args(["--impl", "reference"]))
    assert buf.getvalue() == ""


def test_clock_anomaly_rules():
    ok = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 9}
    assert bench.clock_anomaly(ok) is None
    assert bench.clock_anomaly({**ok, "sm_mhz": 1500, "reasons": ["sw_power_cap"]}) is None
    assert "no reason" in bench.clock_anomaly({**ok, "sm_mhz": 1597})
    assert "hw_slowdown" in bench.clock_anomaly({**ok, "reasons": ["hw_slowdown"]})
    assert bench.clock_anomaly({**ok, "sm_mhz": None, "reasons": ["unsampled"]}) is None


def test_tensor_peak_follows_the_timed_region():
    """Burst figure for a short region at full clock; the sustained figure only
    for a region of seconds whose SM clock sat well below the maximum."""
    peaks = {"bf16_tflops": 1610.6, "bf16_tflops_sustained": 1373.6, "hbm_gbs": 6537.3}
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    capped = {"sm_mhz": 1300, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.choose_tensor_peak(peaks, 0.065, full) == (1610.6, "bf16_tflops")
    assert bench.choose_tensor_peak(peaks, 0.065, capped) == (1610.6, "bf16_tflops")
    assert bench.choose_tensor_peak(peaks, 5.0, full) == (1610.6, "bf16_tflops")
    assert bench.choose_tensor_peak(peaks, 5.0, capped) == (1373.6, "bf16_tflops_sustained")
    assert bench.choose_tensor_peak(peaks, 5.0, {"sm_mhz": None, "sm_max_mhz": None}) == \
        (1610.6, "bf16_tflops")


def test_traffic_record_holds_only_for_the_sources_it_was_taken_with(tmp_path, monkeypatch):
    """roofline.traffic comes from profiles/traffic.json only while the
    kernel's source files hash to what the capture recorded; any change to
    them turns it into null, and a workload without a capture is null too."""
    import shutil
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    real = bench.load_traffic("temporal_conv", w)
    assert isinstance(real, int) and real > 0            # the committed record holds
    assert bench.load_traffic("temporal_conv", synth.BY_NAME["bf16_F128_P2560_C320"]) is None
    # a copy of the tree whose conv source differs by one byte
    root = tmp_path / "tree"
    shutil.copytree(os.path.join(ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(ROOT, "clip_temporal_modules_b200", "csrc"),
                    root / "clip_temporal_modules_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.load_traffic("temporal_conv", w) == real
    src = root / "clip_temporal_modules_b200" / "csrc" / "temporal_conv_tc.cu"
    src.write_bytes(src.read_bytes() + b"\n")
    assert bench.load_traffic("temporal_conv", w) is None
