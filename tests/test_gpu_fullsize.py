"""The bench workload at full size, in the launch configuration bench.py times.

concurrency_stress: B = 4096 slots x H = 48 heads, d = 128, P = 8, bf16 io,
12 of 48 heads INT8, column scales (196,608 heads, a 2.06 GB pool).  The
whole pool runs through pace_decode_step / pace_commit_period exactly as in
bench.py; the fp64 oracle checks a seeded sample of heads one by one
(teacher-forced from oracle-written records, corners and INT8 heads
included), and properties that hold at any size are checked on every head.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu

PERIODS = 2


def _sample_heads(w, bits, n_random=48, n_int8=12, seed=1234):
    rng = np.random.RandomState(seed)
    int8 = [h for h in range(w.H) if bits[h] == 8]
    heads = {(0, 0), (w.B - 1, w.H - 1), (w.B - 1, 0), (0, w.H - 1)}
    while len(heads) < 4 + n_random:
        heads.add((int(rng.randint(w.B)), int(rng.randint(w.H))))
    for _ in range(n_int8):
        heads.add((int(rng.randint(w.B)), int(int8[rng.randint(len(int8))])))
    return sorted(heads)


def test_concurrency_stress_full_size_sampled_parity():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("concurrency_stress")
    bits = pace_synth.head_bits(w, 0)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)

    # every head starts non-zero (the library's encoder fills the pool) ...
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=7, device="cuda",
                                column_outliers=[3, 77])
    pool.load(S.view(w.B, w.H, w.d_v, w.d_k))
    torch.cuda.synchronize()
    del S
    torch.cuda.empty_cache()

    # ... and the sampled heads start from records the oracle wrote
    heads = _sample_heads(w, bits)
    hb = [bits[h] for _, h in heads]
    assert sum(b == 8 for b in hb) >= 8
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=11, column_outliers=[3, 77]).numpy()
    state, _ = orc.PoolState.from_fp32(S0, hb, w.axis)

    t = 0
    worst = 0.0
    for per in range(PERIODS):
        pu.load_state(pool, heads, state)
        toks_host, outs = [], []
        for n in range(w.P):
            inp = pace_synth.token_inputs(w, t, seed=3, device="cuda")
            t += 1
            o = pool.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
            # properties over every head: finite outputs, fill advanced everywhere
            assert bool(torch.isfinite(o).all())
            outs.append(pu.host_tokens({"o": o.view(w.B, w.H, w.d_v)}, heads)["o"])
            toks_host.append(pu.host_tokens(inp, heads))
            del inp
        assert bool((pool.fill() == w.P).all())
        pool.commit_period()
        assert pool.status() == 0
        assert bool((pool.fill() == 0).all())

        outs_ref, S_end, committed, _ = orc.period_reference(state, toks_host, w.P)
        for n in range(w.P):
            err = orc.relative_error(outs[n], outs_ref[n])
            worst = max(worst, float(err.max()))
            assert err.max() <= pu.O_TOL, (per, n, float(err.max()))
        gc, gs = pu.read_state(pool, heads)
        pu.judge_commit(gc, gs, committed, S_end, w.axis)
        state = committed
    print(f"full-size sampled parity: {len(heads)} heads, worst relative error {worst:.3e}")

    # every head's committed scales are finite and non-negative
    for h in range(w.H):
        off, nbytes, stride = pace.pace_pool_layout(pool.handle, h)
        code_bytes = w.d_v * w.d_k * bits[h] // 8
        raw = pool.state.view(w.B, stride)[:, off + code_bytes: off + code_bytes + 2 * w.d_k]
        sc = raw.contiguous().view(torch.float16).float()
        assert bool(torch.isfinite(sc).all()) and bool((sc >= 0).all()), h
