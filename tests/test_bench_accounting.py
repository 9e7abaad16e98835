"""The benchmark's algorithmic FLOP and byte counts, without a GPU.

The roofline fractions the benchmark reports divide these counts by measured
times, so they are checked here against the per-workload figures worked out
independently from the shapes (GFLOP and MB, each tensor read or written
once, padding not credited).
"""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


# workload: (GFLOP, MB) of one step
EXPECTED = {
    "fwd_bf16": (10.07, 102.9),          # x + y + T
    "train_bf16": (30.21, 258.0),        # x, y, dY, x, dX, T, dT
    "sweep_w7": (10.07, 411.1),
    "sweep_w14": (40.28, 411.4),
    "sweep_w28": (161.13, 412.6),
    "hires_cached_dw": (15.80, 161.5),   # x, z, M, 3x3 weights; y stays on chip
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_step_counts(bench, name):
    import synth
    wl = synth.WORKLOADS[name]
    gflop, mb = EXPECTED[name]
    assert bench.step_flops(wl) / 1e9 == pytest.approx(gflop, abs=0.006)
    assert bench.step_bytes(wl) / 1e6 == pytest.approx(mb, abs=0.06)


def test_training_call_counts(bench):
    import synth
    wl = synth.WORKLOADS["train_bf16"]
    m = 128 * 256 * 28 * 28 * 2
    # the step is one forward call and one backward call; dY is counted once
    # in the backward call, x and the table once in each call (the step's
    # count takes the table once)
    assert bench.kernel_bytes(wl, "forward") + bench.kernel_bytes(wl, "backward") == \
        bench.step_bytes(wl) + 256 * 729 * 2
    assert bench.kernel_bytes(wl, "backward") == 3 * m + 256 * 729 * (2 + 4)
    assert bench.kernel_flops(wl, "forward") + bench.kernel_flops(wl, "backward") == \
        bench.step_flops(wl)
    # the gradients alone: input and output map each, plus their table
    assert bench.kernel_bytes(wl, "backward_dx") == 2 * m + 256 * 729 * 2
    assert bench.kernel_bytes(wl, "backward_dt") == 2 * m + 256 * 729 * 4


def test_arithmetic_intensity_sides_of_the_ridge(bench):
    # w <= 14 sits below the ridge of the measured peaks (HBM-bound), w = 28 above
    import synth
    peaks = bench.load_peaks()
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    ai = {n: bench.step_flops(synth.WORKLOADS[n]) / bench.step_bytes(synth.WORKLOADS[n])
          for n in ("sweep_w7", "sweep_w14", "sweep_w28")}
    assert ai["sweep_w7"] < ai["sweep_w14"] < ridge < ai["sweep_w28"]


def test_merge_counts(bench):
    import synth
    wl = synth.WORKLOADS["hires_reparam"]
    # 96 merged 196 x 196 matrices written, a 27^2 and a 13^2 table read
    assert bench.kernel_bytes(wl, "reparam_merge") == 96 * (196 * 196 + 729 + 169) * 2
    assert bench.step_bytes(wl) == 2 * 8 * 96 * 224 * 224 * 2 + 96 * 196 * 196 * 2


def _run_bench(args, env_extra, code_tail=""):
    import subprocess
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.update(env_extra)
    code = ("import sys, runpy; sys.argv = ['bench.py'] + %r\n"
            "try:\n    runpy.run_path('bench.py', run_name='__main__')\n"
            "except SystemExit as e:\n    print('EXIT', e.code)\n%s" % (list(args), code_tail))
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=600)


def test_gpus_flag_must_match_the_launched_ranks():
    # one process launched (WORLD_SIZE=1) but --gpus 2 asked: refused loudly,
    # before any device work, instead of timing one GPU as if it were two
    r = _run_bench(["--gpus", "2", "--steps", "3", "--warmup", "3"], {"WORLD_SIZE": "1"})
    assert "EXIT 2" in r.stdout
    assert "--gpus 2 but WORLD_SIZE=1" in r.stderr


def test_reference_arm_maps_no_wbmm_library():
    # the oracle arm runs the CPU oracle only: the CUDA library is never loaded
    tail = ("maps = open('/proc/self/maps').read()\n"
            "print('LIBWBMM' if 'libwbmm' in maps else 'CLEAN')\n"
            "print('ORACLE' if 'liboracle' in maps else 'NO-ORACLE')\n")
    r = _run_bench(["--impl", "reference", "--workload", "fwd", "--steps", "1", "--warmup", "0"],
                   {}, tail)
    assert r.returncode == 0, r.stderr
    assert '"impl": "reference"' in r.stdout
    assert "CLEAN" in r.stdout and "ORACLE" in r.stdout
