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


def test_algorithmic_bytes_count_the_pool_as_laid_out():
    """The roofline's algorithmic bytes against the library's own layout: the
    records one decode launch reads (and one commit reads and writes once)
    add up to the pool's state region, and a period's buffered rows (k, v,
    alpha, beta in the io dtype) to the buffer's row and gate blocks."""
    sys.path.insert(0, ROOT)
    import bit_recurrent_state_pace_b200 as pace
    import pace_synth
    bench = _bench_module()
    for name, over in (("concurrency_stress", {}), ("mixed_4_8", {}), ("gdn_layer_4b", {"io_dtype": "f32"})):
        w = pace_synth.workload(name, **over)
        bits = pace_synth.head_bits(w, 0)
        BH = w.B * w.H
        axis = pace.PACE_SCALE_COL if w.axis == "col" else pace.PACE_SCALE_ROW
        io = pace.PACE_IO_BF16 if w.io_dtype == "bf16" else pace.PACE_IO_F32
        state, _, _ = pace.pace_pool_bytes(w.B, w.H, w.d_k, w.d_v, w.P, axis, io, bits)
        dec1, com, *_ = bench.alg_bytes(w, bits, 1)
        esz = 2 if w.io_dtype == "bf16" else 4
        # a decode at buffer position 1: the records, the token in, its row
        # buffered, o out, the fill read and written
        per_head = (2 * w.d_k + w.d_v + 2) * esz + (w.d_k + w.d_v + 2) * esz + 4 * w.d_v + 8
        assert dec1 - BH * per_head == state, name
        # the commit: every record read and written, P buffered rows read
        _, buf1, _ = pace.pace_pool_bytes(w.B, w.H, w.d_k, w.d_v, w.P, axis, io, bits)
        rows = com - 2 * state - 8 * BH
        assert rows == BH * w.P * (w.d_k + w.d_v + 2) * esz, name
        assert rows <= buf1, name
