"""bench.py's reference arm runs on the host (the fp64 oracle): its JSON line
keeps the benchmark line's contract.  The GPU arm is covered on a B200."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_gpus_flag_starts_the_ranks_itself():
    # --gpus 2 without WORLD_SIZE: bench.py runs itself as two ranks under
    # torch.distributed.run; with the CPU-only reference arm rank 0 prints the
    # line (n_gpus 2) and rank 1 exits without work
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_world_size_that_differs_from_gpus_is_refused():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 2 and "WORLD_SIZE" in r.stderr


def test_clock_summary_keeps_only_samples_inside_the_timed_region():
    # rows as nvidia-smi prints them: idle samples at the maximum clock before
    # and after the region, power-capped samples inside it
    import importlib.util
    import datetime
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def row(dt_ms, mhz, cap):
        ts = (base + datetime.timedelta(milliseconds=dt_ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return [ts, "0", str(mhz), "1965", "700.0", "0x4" if cap else "0x0", "Not Active", "Not Active",
                "Not Active", "Active" if cap else "Not Active"]

    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.samples = ([row(t, 1965, False) for t in range(-500, 0, 20)] + [row(t, 1520, True) for t in range(0, 300, 20)]
                 + [row(t, 1965, False) for t in range(420, 900, 20)])
    s.t0, s.t1 = base.timestamp(), base.timestamp() + 0.29
    out = s.stop()
    assert out["sm_mhz"] == 1520 and out["sm_min_mhz"] == 1520 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 15


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0
