"""bench.py's host-side contract, on CPU: the algorithmic work and bytes it divides by,
the stored ncu traffic it reports (only while the kernel sources match), the text-only
profiles folder, and the reference arm's JSON line."""
import glob
import importlib.util
import json
import os
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def _shape(M, N, K, E=1):
    return types.SimpleNamespace(M=M, N=N, K=K, E=E)


def test_algorithmic_bytes_of_the_benchmarked_shapes():
    """Each operand read once and Y written once: codes K/2 and scales K/16 bytes per
    row, BF16 activations 2 bytes per element (the per-unit figures of the roofline)."""
    b = _bench()
    flops, nbytes = b.algorithmic(_shape(4096, 5376, 14336), "w4a4")
    assert flops == 2.0 * 4096 * 5376 * 14336
    assert nbytes == (4096 + 5376) * (7168 + 896) + 4096 * 5376 * 2 == 120_422_400
    assert b.algorithmic(_shape(16, 5376, 14336), "w4a16")[1] == 43_982_848
    assert b.algorithmic(_shape(4096, 0, 14336), "quantize")[1] == 150_470_660
    assert b.algorithmic(_shape(8192, 14336, 4096, E=8), "grouped")[1] == 517_996_544
    assert b.algorithmic(_shape(4096, 5376, 14336), "w4a8")[1] == 146_112_512


KERNEL_PATH = {"w4a4_pair_kernel": "w4a4", "grouped_pair_kernel": "grouped",
               "via_fp8_kernel": "via_fp8", "w4a8_kernel": "w4a8", "w4a16_ldg_kernel": "w4a16"}


def _kv(path):
    kv = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln:
                k, v = ln.split(":", 1)
                kv[k.strip()] = v.strip()
    return kv


@pytest.mark.parametrize("fn", sorted(glob.glob(os.path.join(ROOT, "profiles", "traffic_*.txt"))),
                         ids=os.path.basename)
def test_stored_traffic_matches_the_current_kernel_source(fn):
    """A stored DRAM-traffic figure is reported only for the source it was measured on;
    every committed one must match the kernels as they stand."""
    b = _bench()
    kv = _kv(fn)
    kernel = kv["kernel"]
    path = "quantize" if kernel.startswith("amax_bf16_kernel") else KERNEL_PATH[kernel]
    assert kv["source_hash"] == b.kernel_source_hash(path), f"{os.path.basename(fn)} is stale"
    assert int(kv["dram_bytes_per_launch"]) > 0
    assert kv["capture"].startswith("ncu ") and "--clock-control none" in kv["capture"]


def test_profiles_hold_short_text_summaries_only():
    for fn in glob.glob(os.path.join(ROOT, "profiles", "*")):
        assert fn.endswith((".md", ".txt")), fn
        assert os.path.getsize(fn) < 16 * 1024, fn


def test_reference_arm_prints_its_line_on_the_host():
    """`--impl reference` times the oracle on the host cores and prints one JSON line
    with the base contract's keys, a cpu_baseline and a zero-copy e2e."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("ffn_down")


def test_other_paths_summarise_each_run_and_record_failures(monkeypatch):
    """The default line's other_paths: one short run per other workload (at most 30
    timed steps, 3 warm-up, no e2e or CPU baseline), summarised; a failing path is
    recorded with its error instead of stopping the line."""
    b = _bench()
    seen = []

    def fake_run(sub, emit=True):
        assert emit is False
        seen.append((sub.workload, sub.steps, sub.warmup, sub.no_e2e, sub.no_cpu_baseline,
                     sub.no_other_paths))
        if sub.workload == "w4a8":
            raise RuntimeError("boom")
        return {"metric": "m", "value": 1.0, "unit": "u", "ms_per_step": 0.5, "steps": sub.steps,
                "roofline": {"frac": 0.5, "bound": "tensor"}, "gpu_launches": 2, "clocks": {}}

    monkeypatch.setattr(b, "run_ours", fake_run)
    args = types.SimpleNamespace(workload="ffn_down", steps=200, warmup=10, no_e2e=False,
                                 no_cpu_baseline=False, no_other_paths=False, gpus=1,
                                 impl="ours", no_graph=False)
    out = b.other_paths(args)
    assert [s[0] for s in seen] == b.OTHER_PATHS
    assert all(s[1:] == (30, 3, True, True, True) for s in seen)
    assert out["w4a8"] == {"error": "RuntimeError: boom"}
    assert out["grouped"]["value"] == 1.0 and out["grouped"]["roofline"]["frac"] == 0.5
    assert args.steps == 200 and args.no_e2e is False  # the headline's own arguments untouched
