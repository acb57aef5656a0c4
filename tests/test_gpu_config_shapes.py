"""The gated-delta layer, mixed 4/8-bit and period-sweep workloads at their
stated shapes, run for their stated numbers of decode steps.

* gdn_layer_4b: B = 64 x H = 32, d = 128, P = 8, all INT4, 256 decode steps,
  with column scales and with row scales;
* mixed_4_8: B = 256 x H = 32, P = 8, 8 of 32 heads INT8 (the long-memory
  heads), 512 decode steps, with column scales and with row scales;
* period_sweep: B = 512 x H = 32, all INT4, 1024 decode steps for each
  P in {1, 2, 4, 8, 16} (P = 1 rounds after every token).

Each starts from the workload's 512-token unquantised warm-up prefill: every
head of the pool is warmed by the fp32 GPU step and encoded by the library,
and a seeded sample of heads (corners, random heads, INT8 heads) gets the
oracle's warm-up from the same tokens, encoded by the oracle.  Then the whole
pool decodes and commits through pace_decode_step / pace_commit_period, the
calls and launch shapes bench.py times, so that the kernels run their
multi-head pipelines over a full pool.  The sampled heads are teacher-forced:
each period starts from the oracle's committed records.  Per token their
outputs must be within 2e-3 maximum relative error of the oracle's; per
period their committed codes may differ from the oracle's only by +-1 at
rounding ties, at most 0.1 % of them.  On every head: outputs finite, fills
advancing together, no device status flag.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu

SEED = 0
TOKEN_SEED = 3


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


def _sample_heads(w, bits, n_random, n_int8=0, seed=4321):
    rng = np.random.RandomState(seed)
    heads = {(0, 0), (w.B - 1, w.H - 1), (w.B - 1, 0), (0, w.H - 1)}
    while len(heads) < 4 + n_random:
        heads.add((int(rng.randint(w.B)), int(rng.randint(w.H))))
    int8 = [h for h in range(w.H) if bits[h] == 8]
    for _ in range(n_int8 if int8 else 0):
        heads.add((int(rng.randint(w.B)), int(int8[rng.randint(len(int8))])))
    return sorted(heads)


def _warm_pool_state(pace, w):
    """All B x H heads through the workload's warm-up prefill on the GPU (fp32 steps)."""
    BH = w.B * w.H
    io = pace.PACE_IO_BF16 if w.io_dtype == "bf16" else pace.PACE_IO_F32
    S = torch.zeros(BH, w.d_v, w.d_k, dtype=torch.float32, device="cuda")
    for t in range(w.warmup):
        x = pace_synth.token_inputs(w, t, seed=SEED, device="cuda", phase="warmup")
        pace.pace_gdn_step_f32(S, x["q"], x["k"], x["v"], x["alpha"], x["beta"], io, None, BH,
                               w.d_k, w.d_v)
    torch.cuda.synchronize()
    return S.view(w.B, w.H, w.d_v, w.d_k)


def _run(w, bits, heads, S_warm, state):
    """w.steps decode tokens over the whole pool; teacher-forced oracle checks
    on `heads`.  Returns the worst relative output error seen."""
    pace = _pace()
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.load(S_warm)
    torch.cuda.synchronize()
    worst = 0.0
    t = 0
    assert w.steps % w.P == 0
    for per in range(w.steps // w.P):
        pu.load_state(pool, heads, state)
        toks_host, outs = [], []
        for n in range(w.P):
            x = pace_synth.token_inputs(w, t, seed=TOKEN_SEED, device="cuda")
            t += 1
            o = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
            outs.append(pu.host_tokens({"o": o}, heads)["o"])
            toks_host.append(pu.host_tokens(x, heads))
            if n == w.P - 1 and (per % 16 == 0 or per == w.steps // w.P - 1):
                assert bool(torch.isfinite(o).all()), (per, n)
        if per % 16 == 0:
            assert bool((pool.fill() == w.P).all()), per
        pool.commit_period()

        outs_ref, S_end, committed, _ = orc.period_reference(state, toks_host, w.P)
        for n in range(w.P):
            err = orc.relative_error(outs[n], outs_ref[n])
            worst = max(worst, float(err.max()))
            assert err.max() <= pu.O_TOL, (w.name, w.P, per, n, float(err.max()))
        gc, gs = pu.read_state(pool, heads)
        pu.judge_commit(gc, gs, committed, S_end, w.axis)
        state = committed
    assert pool.status() == 0, pace.pace_status_string(pool.status())
    assert bool((pool.fill() == 0).all())
    return worst


@pytest.mark.parametrize("axis", ["col", "row"])
def test_gdn_layer_4b_full_shape(axis):
    w = pace_synth.workload("gdn_layer_4b", axis=axis)
    assert (w.B, w.H, w.P, w.steps, w.warmup) == (64, 32, 8, 256, 512)
    bits = pace_synth.head_bits(w, SEED)
    heads = _sample_heads(w, bits, n_random=28)
    S = _warm_pool_state(_pace(), w)
    state = pu.oracle_warm_state(w, heads, [bits[h] for _, h in heads], seed=SEED, device="cuda")
    worst = _run(w, bits, heads, S, state)
    print(f"gdn_layer_4b ({axis}): {len(heads)} heads x {w.steps} tokens, worst relative error {worst:.3e}")


@pytest.mark.parametrize("axis", ["col", "row"])
def test_mixed_4_8_full_shape(axis):
    w = pace_synth.workload("mixed_4_8", axis=axis)
    bits = pace_synth.head_bits(w, SEED)
    assert (w.B, w.H, w.steps) == (256, 32, 512) and sum(b == 8 for b in bits) == 8
    heads = _sample_heads(w, bits, n_random=20, n_int8=12)
    assert sum(bits[h] == 8 for _, h in heads) >= 8
    S = _warm_pool_state(_pace(), w)
    state = pu.oracle_warm_state(w, heads, [bits[h] for _, h in heads], seed=SEED, device="cuda")
    worst = _run(w, bits, heads, S, state)
    print(f"mixed_4_8 ({axis}): {len(heads)} heads x {w.steps} tokens, worst relative error {worst:.3e}")


@pytest.fixture(scope="module")
def sweep_start():
    """The period-sweep workload's warm state: the tokens do not depend on P,
    so one warm-up serves every period length."""
    w = pace_synth.workload("period_sweep")
    bits = pace_synth.head_bits(w, SEED)
    heads = _sample_heads(w, bits, n_random=16)
    S = _warm_pool_state(_pace(), w)
    state = pu.oracle_warm_state(w, heads, [bits[h] for _, h in heads], seed=SEED, device="cuda")
    yield bits, heads, S, state
    del S
    torch.cuda.empty_cache()


@pytest.mark.parametrize("P", pace_synth.PERIOD_SWEEP)
def test_period_sweep_full_shape(P, sweep_start):
    bits, heads, S, state = sweep_start
    w = pace_synth.workload("period_sweep", P=P)
    assert (w.B, w.H, w.steps) == (512, 32, 1024) and set(bits) == {4}
    worst = _run(w, bits, heads, S, state)
    print(f"period_sweep P={P}: {len(heads)} heads x {w.steps} tokens, worst relative error {worst:.3e}")
