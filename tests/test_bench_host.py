"""Host-side logic of bench.py on CPU: max-over-ranks aggregation with a
2-rank gloo group, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [2.0, 3.0][rank]                 # rank 1 is the slow one
    value, ms = bench.aggregate(local_ms, steps=10, world=world)
    q.put((rank, value, ms))
    dist.destroy_process_group()


def test_aggregate_takes_max_over_ranks():
    import bench
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms in res:
        assert ms == pytest.approx(3.0)          # the slowest rank sets the time
        assert value == pytest.approx(2 * bench.STEP_FLOPS / 3e-3 / 1e12)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--ref-tokens", "32"], capture_output=True, text=True, timeout=300,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_profile_traffic_is_null_once_the_kernel_changes(tmp_path, monkeypatch):
    """`roofline.traffic` comes from a committed ncu summary only while the summary's
    source hash matches the kernel sources; any edit of them turns it into null."""
    import hashlib
    import bench
    srcs = ["csrc/k.cuh", "csrc/h.cuh"]
    root = tmp_path / "repo"
    (root / "csrc").mkdir(parents=True)
    (root / "profiles").mkdir()
    (root / srcs[0]).write_text("kernel\n")
    (root / srcs[1]).write_text("header\n")
    digest = hashlib.sha256(b"kernel\nheader\n").hexdigest()[:16]
    (root / "profiles" / "k.txt").write_text(
        "# a summary\ndram__bytes_read.sum: 1 MB\ntraffic_bytes_per_launch: 12345\n"
        f"kernel_source_sha256_16: {digest}\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.profile_traffic("k.txt", srcs) == pytest.approx(12345.0)
    with open(root / srcs[0], "a") as f:
        f.write("// edited\n")
    assert bench.profile_traffic("k.txt", srcs) is None
    assert bench.profile_traffic("missing.txt", srcs) is None


def test_committed_gemm_profile_matches_the_kernel_source():
    """The committed GEMM summary was taken on the kernel as it stands (else the
    bench would report no traffic)."""
    import bench
    t = bench.profile_traffic("mx_gemm_kernel_moe_G8_K4096_N4096.txt",
                              ["mxfp8_block_scaled_cast_b200/csrc/mx_gemm.cuh",
                               "mxfp8_block_scaled_cast_b200/csrc/mx_sm100.cuh"])
    assert t is not None and 2e8 < t < 4e8


def test_peak_follows_the_length_of_the_timed_region_and_the_power_cap():
    """The in-step GEMM rate is held against the burst peak for a short region
    and against the sustained one for a long or power-capped region."""
    import bench
    peaks = {"bf16_tflops": 1665.9, "bf16_tflops_sustained": 1414.4}
    kind, peak, why = bench.select_peak(16.3, [], peaks)
    assert (kind, peak) == ("burst", 1665.9) and "16.3 ms" in why
    kind, peak, why = bench.select_peak(16.3, ["sw_power_cap"], peaks)
    assert (kind, peak) == ("sustained", 1414.4) and "power cap" in why
    assert bench.select_peak(250.0, [], peaks)[:2] == ("sustained", 1414.4)
    # a measured file without a figure falls back to the recorded ones
    assert bench.select_peak(16.3, [], {})[1] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert bench.select_peak(250.0, [], {})[1] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_clock_sampler_process_keeps_the_readings_inside_a_region(tmp_path):
    """The NVML sampler runs as a process of its own (a fake NVML module here):
    its readings carry their own monotonic stamps, and a region keeps exactly
    the readings stamped inside it, with the clock-event reasons they flag
    (gpu_idle left out) and how the device was found."""
    import time
    import bench
    fake = tmp_path / "fake"
    fake.mkdir()
    (fake / "pynvml.py").write_text(
        "NVML_CLOCK_SM = 0\n"
        "def nvmlInit(): pass\n"
        "def nvmlDeviceGetHandleByUUID(u): return u\n"
        "def nvmlDeviceGetHandleByIndex(i): return i\n"
        "def nvmlDeviceGetClockInfo(h, c): return 1800\n"
        "def nvmlDeviceGetCurrentClocksEventReasons(h): return 0x5\n")      # gpu_idle | sw_power_cap
    out = tmp_path / "clocks.txt"
    out.write_text("")
    env = dict(os.environ, PYTHONPATH=str(fake))
    proc = subprocess.Popen([sys.executable, "-c", bench._SAMPLER_SRC, "GPU-0", "0.001", "2", str(out), "0",
                             str(os.getpid())], env=env)
    try:
        time.sleep(0.5)
        region = bench.ClockSampler.__new__(bench.ClockSampler)
        region.sampler = (str(out), 1965)
        with region:
            time.sleep(0.2)
    finally:
        proc.wait(timeout=30)
    s = region.summary()
    assert s["samples"] >= 20 and s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["nvml_device_by"] == "uuid"
    readings = sum(1 for line in open(out) if not line.startswith("#"))
    assert readings > s["samples"]                      # the readings outside the region are left out


def test_clock_sampler_process_ends_with_its_parent(tmp_path):
    """A sampler whose parent is gone stops at once (a rank ended by a signal
    runs no exit handlers), long before its own deadline."""
    import time
    import bench
    fake = tmp_path / "fake"
    fake.mkdir()
    (fake / "pynvml.py").write_text(
        "NVML_CLOCK_SM = 0\n"
        "def nvmlInit(): pass\n"
        "def nvmlDeviceGetHandleByUUID(u): return u\n"
        "def nvmlDeviceGetClockInfo(h, c): return 1800\n"
        "def nvmlDeviceGetCurrentClocksEventReasons(h): return 0\n")
    out = tmp_path / "clocks.txt"
    out.write_text("")
    env = dict(os.environ, PYTHONPATH=str(fake))
    t0 = time.monotonic()
    proc = subprocess.Popen([sys.executable, "-c", bench._SAMPLER_SRC, "GPU-0", "0.001", "60", str(out), "0",
                             "1"], env=env)           # parent id 1: not its parent, as after the parent died
    proc.wait(timeout=30)
    assert time.monotonic() - t0 < 30 and proc.returncode == 0
