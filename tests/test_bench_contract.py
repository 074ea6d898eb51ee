"""bench.py's output contract, on the CPU: the reference arm (the oracle on the
host cores) prints one JSON line with the keys the measurement needs, and the
DRAM traffic taken from an ncu summary is reported only while the profiled
kernel's sources are unchanged."""
import json
import shutil
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "cpu_baseline", "e2e", "gpu_launches")


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in REQUIRED:
        assert k in line, k
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 1
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("tiny")
    # the same config keys as the GPU arm's line
    assert set(line["config"]) == set(bench_config_keys())


def bench_config_keys():
    import bench
    from attention_kl_distillation_b200.inputs import WORKLOADS
    return bench.run_config(bench.parse_args([]), WORKLOADS["tiny"], "fwd", 1).keys()


def test_reference_arm_does_not_load_the_library():
    """The reference arm runs only the oracle: the CUDA library must not be mapped."""
    code = ("import sys; sys.argv = ['bench.py']; import bench; "
            "bench.main(['--impl', 'reference', '--workload', 'tiny', '--steps', '1', "
            "'--warmup', '0']); "
            "maps = open('/proc/self/maps').read(); "
            "assert 'libstreamkl' not in maps, 'libstreamkl.so mapped'; "
            "assert 'liboracle' in maps")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    import bench
    csrc = tmp_path / "attention_kl_distillation_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("bwd_sm100.cu", "fwd_sm100.cu", "kernels.h", "sm100.cuh"):
        shutil.copy(ROOT / "attention_kl_distillation_b200" / "csrc" / name, csrc / name)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    sha = bench.kernel_sources_sha1("bwd_sm100.cu")
    prof = tmp_path / "profiles" / "bwd_fused_key_tiles_kernel_case.md"
    prof.write_text(f"source-sha1: {sha}\n- dram-bytes-per-full-launch: 12345\n")
    assert bench.profiled_traffic("bwd_fused_key_tiles_kernel_case.md") == 12345
    # another kernel's file does not matter
    (csrc / "fwd_sm100.cu").write_text("// changed\n")
    assert bench.profiled_traffic("bwd_fused_key_tiles_kernel_case.md") == 12345
    # the profiled kernel's own file or a shared header does
    (csrc / "sm100.cuh").write_text("// changed\n")
    assert bench.profiled_traffic("bwd_fused_key_tiles_kernel_case.md") is None
    assert bench.profiled_traffic("missing.md") is None


@pytest.mark.parametrize("argv,expect", [
    ([], {"gpus": 1, "steps": 40, "warmup": 5, "impl": "ours", "workload": "fwdbwd16k"}),
    (["--nq", "1", "--splitk", "--phase", "fwd"], {"nq": 1, "splitk": True, "phase": "fwd"}),
    (["--shard", "heads"], {"shard": "heads"}),
])
def test_bench_arguments(argv, expect):
    import bench
    a = bench.parse_args(argv)
    for k, v in expect.items():
        assert getattr(a, k) == v
