"""Edge cases of the decode and commit path against the fp64 oracle: the
largest head count, one slot with one head, empty slot ranges, a zero state
that nothing writes to, and gates at their limits (alpha = 0 forgets the
whole state every token; alpha = 1 with beta = 0 keeps it unchanged)."""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu
from tests.test_gpu_decode import _run_periods

pytestmark = pytest.mark.gpu


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


def test_largest_head_count():
    # 256 heads per slot (the layout's limit), a quarter of them INT8
    w = pace_synth.workload("mixed_4_8", B=2, H=256, d_k=32, d_v=32, P=4, outliers=False)
    assert sum(b == 8 for b in pace_synth.head_bits(w)) == 64
    _run_periods(w, periods=2, random_init=True)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_one_slot_one_head(frac):
    w = pace_synth.workload("mixed_4_8", B=1, H=1, int8_fraction=frac)
    assert pace_synth.head_bits(w) == [8 if frac else 4]
    _run_periods(w, periods=2, random_init=True)


def test_empty_slot_ranges_are_noops():
    pace = _pace()
    w = pace_synth.workload("tiny", B=3)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, pace_synth.head_bits(w, 0), io=w.io_dtype)
    pool.load(pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=1, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k))
    before = (pool.state.clone(), pool.buffer.clone(), pool.aux.clone())
    x = pace_synth.token_inputs(w, 0, device="cuda")
    o = torch.full((w.B, w.H, w.d_v), 7.0, device="cuda")
    for b0 in (0, w.B):
        pool.decode_step_range(b0, 0, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o)
        pool.commit_period_range(b0, 0)
    pace.pace_prefill_range(pool.handle, 1, 0, 1, x["q"][None], x["k"][None], x["v"][None],
                            x["alpha"][None], x["beta"][None], None, None)
    torch.cuda.synchronize()
    assert pool.status() == 0
    assert bool((o == 7.0).all())
    for a, b in zip(before, (pool.state, pool.buffer, pool.aux)):
        assert torch.equal(a, b)


def _teacher_forced_period(w, edit, seed=0, state_edit=None, engine=None):
    """One period from a random stored state (changed by state_edit(S0) when
    given) with the token inputs changed by edit(inputs) (device tensors),
    against the oracle; returns (outputs, the oracle's committed state, the
    GPU's codes and scales)."""
    pace = _pace()
    bits = pace_synth.head_bits(w, seed)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed).numpy()
    if state_edit is not None:
        S0 = state_edit(S0)
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    if engine is not None:
        pool.set_commit_engine(engine)
    pu.load_state(pool, heads, state)
    toks, outs = [], []
    for t in range(w.P):
        x = edit(pace_synth.token_inputs(w, t, seed=seed, device="cuda"))
        outs.append(pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"]).cpu().numpy()
                    .reshape(len(heads), w.d_v))
        toks.append(pu.host_tokens(x, heads))
    pool.commit_period()
    assert pool.status() == 0
    o_ref, S_end, committed, _ = orc.period_reference(state, toks, w.P)
    for n in range(w.P):
        assert orc.relative_error(outs[n], o_ref[n]).max() <= pu.O_TOL, n
    gc, gs = pu.read_state(pool, heads)
    pu.judge_commit(gc, gs, committed, S_end, w.axis)
    return outs, o_ref, committed, (gc, gs), toks


def test_zero_state_without_writes_stays_zero():
    w = pace_synth.workload("mixed_4_8", B=2, H=4)
    pace = _pace()
    bits = pace_synth.head_bits(w, 0)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.load(torch.zeros(w.B, w.H, w.d_v, w.d_k, device="cuda"))
    for t in range(w.P):
        x = pace_synth.token_inputs(w, t, device="cuda")
        x["beta"] = torch.zeros_like(x["beta"])
        o = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        assert bool((o == 0).all()), t
    pool.commit_period()
    assert pool.status() == 0
    # an all-zero group: scale +0 and codes 0
    assert int(pool.state.count_nonzero()) == 0


def test_alpha_zero_forgets_everything():
    w = pace_synth.workload("mixed_4_8", B=2, H=4)

    def edit(x):
        x["alpha"] = torch.zeros_like(x["alpha"])
        return x
    outs, o_ref, committed, _, toks = _teacher_forced_period(w, edit)
    # with alpha = 0 only the token's own write survives: o = beta (k . q) v
    last = toks[-1]
    direct = (last["beta"] * np.sum(last["k"] * last["q"], axis=1))[:, None] * last["v"]
    assert orc.relative_error(o_ref[-1], direct).max() < 1e-12
    assert orc.relative_error(outs[-1], direct).max() <= pu.O_TOL


def test_alpha_one_beta_zero_keeps_the_state():
    w = pace_synth.workload("mixed_4_8", B=2, H=4)

    def edit(x):
        x["alpha"] = torch.ones_like(x["alpha"])
        x["beta"] = torch.zeros_like(x["beta"])
        return x
    _, _, committed, (gc, gs), _ = _teacher_forced_period(w, edit)
    # S_P = S~0 exactly, and re-encoding a decoded state reproduces it
    S0 = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=0).numpy()
    bits = pace_synth.head_bits(w, 0)
    st, _ = orc.PoolState.from_fp32(S0, [bits[h] for _ in range(w.B) for h in range(w.H)], w.axis)
    for i in range(w.B * w.H):
        assert np.array_equal(gc[i], st.codes[i])
        assert np.array_equal(gs[i].view(np.uint16), st.scales[i].view(np.uint16))


@pytest.mark.parametrize("axis,engine", [("col", "mma"), ("col", "tcgen05"), ("row", "mma")])
@pytest.mark.parametrize("bits8", [False, True])
def test_group_scale_in_the_fp16_subnormal_range(axis, engine, bits8):
    """A group whose values are a few 2^-24: its stored FP16 scale is the
    subnormal 2^-23, and after one period of decay with no writes
    (gamma_P = 0.7346) the new absmax / qmax = 1.47 * 2^-24 rounds down to the
    scale 2^-24.  The largest |x / s| is then about 10.3 (INT4) / 186 (INT8),
    so the encoder clamps codes at qmax; every other group keeps normal
    scales.  The commit must give the oracle's clamped codes, not codes past
    qmax."""
    w = pace_synth.workload("gdn_layer_4b", B=2, H=2, P=4, axis=axis, outliers=False,
                            int8_fraction=1.0 if bits8 else 0.0)
    qmax = 127 if bits8 else 7
    tiny = 2.0 * qmax * 2.0 ** -24          # absmax with amax / qmax = 2^-23 exactly

    def state_edit(S0):
        S0 = S0.copy()
        for m in range(S0.shape[0]):
            g = S0[m, :, 5] if axis == "col" else S0[m, 5, :]
            g[:] = np.clip(g / np.abs(g).max(), -1.0, 1.0) * tiny
        return S0.astype(np.float32)

    def edit(x):
        x["beta"] = torch.zeros_like(x["beta"])
        x["alpha"] = torch.full_like(x["alpha"], 0.92578125)   # bf16; gamma_4 = 0.7346
        return x

    pace = _pace()
    eng = pace.PACE_COMMIT_TCGEN05 if engine == "tcgen05" else pace.PACE_COMMIT_MMA
    _, _, committed, (gc, gs), _ = _teacher_forced_period(w, edit, state_edit=state_edit, engine=eng)
    for m in range(len(committed.codes)):
        assert int(committed.scales[m].view(np.uint16)[5]) == 0x0001
        assert int(np.abs(np.asarray(gc[m], np.int64)).max()) <= qmax
        c = committed.codes[m]
        assert int(np.abs(c[:, 5] if axis == "col" else c[5, :]).max()) == qmax
