"""bench.py on the CPU: the reference arm's JSON line, and the ncu records in
profiles/ that the GPU line's roofline `traffic` is read from."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # the same config keys as the GPU arm prints, with the pool's state size
    for key in ("workload", "B", "H", "P", "int8_heads", "l2", "parallelism", "int8_head_choice",
                "int8_head_list", "seq_tokens_per_s"):
        assert key in line["config"], key
    assert "larger than L2" in line["config"]["l2"]
    # ms_per_step is the time of the sample actually run (one sequence, one period)
    H, P = line["config"]["H"], line["config"]["P"]
    assert abs(line["ms_per_step"] - 1000.0 * H * P / line["value"]) <= 1e-6 * line["ms_per_step"]
    assert line["extrapolated_from_heads"] == H


def test_profiles_hold_traffic_for_the_current_kernel_sources():
    """Every ncu traffic record the roofline reads belongs to the kernel sources
    as they are: a change to a kernel without a new capture fails here."""
    bench = _bench_module()
    for kernel in ("decode_step", "commit"):
        digest = bench.kernel_source_digest(kernel)
        traffic = bench.ncu_traffic(kernel, digest)
        assert traffic is not None and traffic > 0, (kernel, digest)


def test_source_digest_ignores_comments_only():
    """A traffic record stays valid across comment edits and not across code
    edits: the digest is taken over the code with comments left out."""
    bench = _bench_module()
    code = 'int f(int x) {\n  // a comment\n  return x + 1; /* and\n another */\n}\n'
    same = 'int f(int x) {\n  // another comment entirely\n  return x + 1;\n}\n'
    changed = 'int f(int x) {\n  return x + 2;\n}\n'
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(changed)
    assert "comment" not in bench._code_only(code)
