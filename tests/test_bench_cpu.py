"""bench.py's reference arm (the CPU oracle) prints the contract's JSON line (CPU)."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=600, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_json_line():
    d = run_bench("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "Gelem/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    import oracle
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] == oracle.host_threads()      # every host core
    assert d["cpu_baseline"]["nproc"] == os.cpu_count()
    assert "multi-threaded oracle step" in d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_warmup_below_three_is_rejected():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--warmup", "2"], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_reference_arm_momentum_rule():
    d = run_bench("--impl", "reference", "--workload", "tiny", "--rule", "momentum", "--steps", "2",
                  "--warmup", "3")
    assert d["config"]["rule"] == "momentum" and d["value"] > 0
    assert "momentum rule" in d["cpu_baseline"]["sample"]


def test_byte_model_of_the_one_pass_step():
    """The one-pass step moves g and err (read and write) per worker, plus m, v, p."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    wl = WL.get_workload("gpt2xl-flat")
    assert bench.step_bytes_per_elem(wl, "compressed", "momentum") == 2 + 8 + 20
    bl = WL.get_workload("bert-large")
    assert bench.step_bytes_per_elem(bl, "compressed", "momentum") == 16 * 12 + 20
    lamb = WL.get_workload("lamb-1.3b")
    assert bench.step_bytes_per_elem(lamb, "compressed", "momentum") == 4 * 12 + 16 + 16


def test_byte_model_of_the_two_bit_step():
    """Three passes: the worker sums (both scales), the two-plane pack with the
    server sums, and the server/update pass."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    wl = WL.get_workload("gpt2xl-flat")
    assert bench.step_bytes_per_elem(wl, "compressed", "twobit") == 6 + 14.25 + 28.5


def test_reference_arm_two_bit_rule():
    d = run_bench("--impl", "reference", "--workload", "tiny", "--rule", "twobit", "--steps", "2",
                  "--warmup", "3")
    assert d["config"]["rule"] == "twobit" and d["value"] > 0


def test_small_workloads_are_timed_with_an_l2_flush():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    assert bench.flushes_l2(WL.get_workload("tiny"))
    assert "flushed" in bench.workload_config(WL.get_workload("tiny"), 1)["l2"]
    for name in ("bert-base", "gpt2xl-flat", "bert-large", "lamb-1.3b"):
        assert not bench.flushes_l2(WL.get_workload(name))
        assert bench.workload_config(WL.get_workload(name), 1)["l2"].startswith("inputs larger than L2")


def test_byte_model_with_the_cached_server_value():
    """From W = 4 on pass 2 also writes c_srv and pass 3 reads it instead of the
    workers' words and the server error."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    bl = WL.get_workload("bert-large")          # W = 16, fp32 gradients and errors
    assert bench.step_bytes_per_elem(bl) == 8 * 16 + (12 * 16 + 2 + 4 + 4) + (4 + 4 + 0.125 + 20)
    assert bench.step_bytes_per_elem(bl.with_(W=2)) == 8 * 2 + (12 * 2 + 0.25 + 4) + (0.25 + 8 + 0.125 + 20)


def test_cpu_baseline_both_legs():
    """The bench's cpu_baseline record: the single-thread leg and the all-cores
    leg on the same chunk sample, the all-cores figure as its value."""
    import types

    import bench
    import oracle
    import workloads as WL
    wl = WL.get_workload("tiny").with_(sizes=(70_000, 4_096, 33), W=2)
    args = types.SimpleNamespace(phase="compressed", rule="scaled")
    rec = bench.cpu_baseline(wl, args)
    assert rec["kind"] == "oracle" and rec["unit"] == "Gelem/s"
    assert rec["cores"] == oracle.host_threads() and rec["nproc"] == os.cpu_count()
    one, allc = rec["legs"]
    assert one["cores"] == 1 and allc["cores"] == rec["cores"]
    assert rec["value"] == allc["value"] and one["value"] > 0 and allc["value"] > 0


def test_byte_model_of_the_data_parallel_stages():
    """Per-element bytes of the data-parallel stage kernels: the worker stage and
    the update on a one-worker ctx, the server stage on the owner's W-worker ctx."""
    import bench
    import workloads as WL
    wl = WL.get_workload("gpt2xl-flat")              # bf16 gradients, f32 error buffers, Adam
    assert bench.dp_bytes_per_elem("k_worker_norm", "worker", wl, 8, "scaled") == 2 + 4
    assert bench.dp_bytes_per_elem("k_worker_pack", "worker", wl, 8, "scaled") == 2 + 8 + 1 / 8
    assert bench.dp_bytes_per_elem("k_server_update", "worker", wl, 8, "scaled") == 1 / 8 + 20
    assert bench.dp_bytes_per_elem("k_server_norm", "server", wl, 8, "scaled") == 1 + 4
    assert bench.dp_bytes_per_elem("k_server_update", "server", wl, 8, "scaled") == 1 + 8 + 1 / 8
    assert bench.dp_bytes_per_elem("k_finalize_scale", "worker", wl, 8, "scaled") == 0
    assert bench.dp_bytes_per_elem("k_worker_norm", "worker", wl, 8, "momentum") == 0
    assert bench.dp_bytes_per_elem("k_tb_pack", "worker", wl, 8, "twobit") == 2 + 8 + 1 / 4
    assert bench.dp_bytes_per_elem("k_tb_server_norm", "server", wl, 8, "twobit") == 2 + 4
    assert bench.dp_bytes_per_elem("k_ternary_compress", "worker", wl, 8, "momentum") == 2 + 8 + 1
    assert bench.dp_bytes_per_elem("k_ternary_server", "server", wl, 8, "momentum") == 9
    assert bench.dp_bytes_per_elem("k_ternary_update", "worker", wl, 8, "momentum") == 21
