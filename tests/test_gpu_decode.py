"""Decode and commit through the C ABI against the fp64 oracle.

Every period starts from a stored state produced by the oracle and written
into the pool's records (teacher forcing from the oracle side): the GPU then
runs P decode steps and one commit; outputs o_t must be within 2e-3 max
relative error, and the committed codes/scales must equal the oracle's up
to +-1 code flips at rounding ties (<= 0.1% of codes).
"""
from typing import List, Sequence, Tuple

import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


def _run_periods(w, periods: int, seed: int = 0, warm_tokens: int = None, check_commit=True,
                 random_init=False, engine=None):
    """Teacher-forced periods over every head of a small pool (commit engine:
    the pool's default unless given)."""
    pace = _pace()
    bits = pace_synth.head_bits(w, seed)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    if engine is not None:
        pool.set_commit_engine(engine)
    if random_init:
        S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed).numpy()
        state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    elif w.warmup or warm_tokens:
        state = pu.oracle_warm_state(w, heads, [bits[h] for _, h in heads], seed=seed,
                                     tokens=warm_tokens)
    else:
        zero = np.zeros((len(heads), w.d_v, w.d_k), np.float32)
        state, _ = orc.PoolState.from_fp32(zero, [bits[h] for _, h in heads], w.axis)
    worst, stats = 0.0, []
    t = 0
    for per in range(periods):
        pu.load_state(pool, heads, state)
        toks_host, outs_gpu = [], []
        for n in range(w.P):
            inp = pace_synth.token_inputs(w, t, seed=seed, device="cpu")
            t += 1
            dev = {k: v.cuda() for k, v in inp.items()}
            o = pool.decode_step(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
            outs_gpu.append(o.cpu().numpy().reshape(len(heads), w.d_v))
            toks_host.append(pu.host_tokens(inp, heads))
        fill = pool.fill().cpu().numpy()
        assert np.all(fill == w.P)
        pool.commit_period()
        assert pool.status() == 0
        assert np.all(pool.fill().cpu().numpy() == 0)
        outs_ref, S_end, committed, flags = orc.period_reference(state, toks_host, w.P)
        for n in range(w.P):
            err = orc.relative_error(outs_gpu[n], outs_ref[n])
            worst = max(worst, float(err.max()))
            assert err.max() <= pu.O_TOL, (per, n, float(err.max()))
        gc, gs = pu.read_state(pool, heads)
        if check_commit:
            stats.append(pu.judge_commit(gc, gs, committed, S_end, w.axis))
        state = committed
    return worst, stats


def test_tiny_all_heads():
    w = pace_synth.workload("tiny")
    worst, stats = _run_periods(w, periods=w.steps // w.P)
    print("tiny worst rel err", worst, stats)


@pytest.mark.parametrize("axis", ["col", "row"])
def test_gdn_layer_shape_reduced_batch(axis):
    w = pace_synth.workload("gdn_layer_4b", B=3, H=4, axis=axis)
    worst, stats = _run_periods(w, periods=2, warm_tokens=128)
    print(axis, "worst", worst, stats)


def test_mixed_int8_long_memory_heads():
    w = pace_synth.workload("mixed_4_8", B=2, H=8)
    assert sum(b == 8 for b in pace_synth.head_bits(w)) == 2
    worst, stats = _run_periods(w, periods=2, warm_tokens=128)
    print("mixed worst", worst, stats)


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5, 12, 16])
def test_period_sweep_small(P):
    w = pace_synth.workload("period_sweep", B=2, H=3, P=P)
    worst, stats = _run_periods(w, periods=2 if P < 16 else 1, random_init=True)
    print("P", P, "worst", worst)


@pytest.mark.parametrize("io,axis,d,P", [("f32", "col", 128, 8), ("f32", "row", 64, 16),
                                         ("bf16", "row", 32, 8), ("bf16", "col", 64, 5),
                                         ("f32", "col", 32, 3)])
def test_io_axis_dim_period_matrix(io, axis, d, P):
    """Mixed 4/8-bit heads across io dtypes, scale axes, head sizes and
    periods (exact-period and general-period kernels)."""
    w = pace_synth.workload("mixed_4_8", B=2, H=4, d_k=d, d_v=d, P=P, io_dtype=io, axis=axis,
                            int8_fraction=0.5)
    assert 8 in pace_synth.head_bits(w) and 4 in pace_synth.head_bits(w)
    worst, _ = _run_periods(w, periods=2, random_init=True)
    print(io, axis, d, P, "worst", worst)


@pytest.mark.parametrize("d", [32, 64])
def test_smaller_head_dims(d):
    w = pace_synth.workload("gdn_layer_4b", B=2, H=3, d_k=d, d_v=d, outliers=False)
    _run_periods(w, periods=2, random_init=True)


def test_phases_differ_per_head():
    """Heads with different numbers of buffered tokens in one launch; commit
    touches only full buffers."""
    pace = _pace()
    w = pace_synth.workload("gdn_layer_4b", B=2, H=2, P=4, outliers=False)
    bits = [4, 8]
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis="col", io="bf16")
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=11).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], "col")
    pu.load_state(pool, heads, state)
    # pre-fill head (1, 0) with 2 tokens by decoding with only that head
    # mattering: run two steps, then reset every other head's buffer.
    pre = []
    for t in range(2):
        inp = pace_synth.token_inputs(w, 100 + t, device="cpu")
        dev = {k: v.cuda() for k, v in inp.items()}
        pool.decode_step(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
        pre.append(pu.host_tokens(inp, heads))
    fill = pool.fill()
    for b, h in heads:
        if (b, h) != (1, 0):
            fill[b, h] = 0
    torch.cuda.synchronize()
    # now run 2 more steps: head (1,0) reaches P = 4, others hold 2 tokens
    new = []
    outs = []
    for t in range(2):
        inp = pace_synth.token_inputs(w, 200 + t, device="cpu")
        dev = {k: v.cuda() for k, v in inp.items()}
        outs.append(pool.decode_step(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"]).cpu().numpy())
        new.append(pu.host_tokens(inp, heads))
    assert pool.fill().cpu().numpy().tolist() == [[2, 2], [4, 2]]
    before = pu.read_state(pool, heads)
    pool.commit_period()
    after = pu.read_state(pool, heads)
    assert pool.fill().cpu().numpy().tolist() == [[2, 2], [0, 2]]
    for idx, (b, h) in enumerate(heads):
        sub = orc.PoolState([state.codes[idx]], [state.scales[idx]], [state.bits[idx]], "col")
        pick = lambda tok: {k: v[idx:idx + 1] for k, v in tok.items()}
        if (b, h) == (1, 0):
            toks = [pick(x) for x in pre + new]
            o_ref, S_end, committed, _ = orc.period_reference(sub, toks, 4)
            for n in range(2):
                err = orc.relative_error(outs[n][b, h][None], o_ref[2 + n])
                assert err.max() <= pu.O_TOL
            pu.judge_commit([after[0][idx]], [after[1][idx]], committed, S_end, "col")
        else:
            toks = [pick(x) for x in new]
            o_ref, _, _, _ = orc.period_reference(sub, toks, 4)
            for n in range(2):
                err = orc.relative_error(outs[n][b, h][None], o_ref[n])
                assert err.max() <= pu.O_TOL
            assert np.array_equal(before[0][idx], after[0][idx])
            assert np.array_equal(before[1][idx].view(np.uint16), after[1][idx].view(np.uint16))


def test_decode_into_full_buffer_is_flagged():
    pace = _pace()
    w = pace_synth.workload("tiny")
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, [4, 4], axis="col", io="f32")
    pool.load(torch.zeros(w.B, w.H, w.d_v, w.d_k, device="cuda"))
    for t in range(w.P):
        inp = {k: v.cuda() for k, v in pace_synth.token_inputs(w, t).items()}
        o = pool.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
    assert pool.status() == 0
    buf_before = pool.buffer.clone()
    inp = {k: v.cuda() for k, v in pace_synth.token_inputs(w, 99).items()}
    o = pool.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
    assert pool.status() & pace.PACE_FLAG_BUFFER_FULL
    assert torch.isnan(o).all()
    assert torch.equal(pool.buffer, buf_before)
    assert (pool.fill() == w.P).all()
    pool.clear_status()
    assert pool.status() == 0
    pool.commit_period()
    assert (pool.fill() == 0).all()


def test_nonfinite_input_is_flagged_at_commit():
    pace = _pace()
    w = pace_synth.workload("tiny")
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, [4, 8], axis="col", io="f32")
    pool.load(torch.randn(w.B, w.H, w.d_v, w.d_k, device="cuda"))
    for t in range(w.P):
        inp = {k: v.cuda() for k, v in pace_synth.token_inputs(w, t).items()}
        if t == 1:
            inp["v"][0, 1, 3] = float("nan")
        pool.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
    pool.commit_period()
    assert pool.status() & pace.PACE_FLAG_NONFINITE
    codes, scales = pu.read_head(pool, 0, 1)
    assert np.isnan(scales).any()
    codes_ok, scales_ok = pu.read_head(pool, 1, 1)
    assert not np.isnan(scales_ok).any()


def test_pool_load_export_layout():
    pace = _pace()
    w = pace_synth.workload("mixed_4_8", B=3, H=8)
    bits = pace_synth.head_bits(w)
    for axis in ("col", "row"):
        pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=axis, io="bf16")
        S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=5, column_outliers=[7]).numpy()
        pool.load(torch.from_numpy(S).cuda().view(w.B, w.H, w.d_v, w.d_k))
        exp = pool.export().cpu().numpy().reshape(-1, w.d_v, w.d_k)
        for b in range(w.B):
            for h in range(w.H):
                i = b * w.H + h
                c_ref, s_ref, _ = orc.quantize(S[i:i + 1], bits[h], axis)
                c, s = pu.read_head(pool, b, h)
                assert np.array_equal(c, c_ref[0])
                assert np.array_equal(s.view(np.uint16), s_ref[0].view(np.uint16))
                assert np.array_equal(exp[i], orc.dequantize(c_ref, s_ref, axis)[0])
        assert (pool.fill() == 0).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unquantised_step_paths(dtype):
    pace = _pace()
    w = pace_synth.workload("gdn_layer_4b", B=4, H=3, io_dtype="bf16")
    n = w.B * w.H
    S0 = pace_synth.random_state(n, w.d_v, w.d_k, seed=2).numpy()
    if dtype == "f32":
        S = torch.from_numpy(S0).cuda()
        step = pace.pace_gdn_step_f32
    else:
        S = torch.from_numpy(S0).to(torch.bfloat16).cuda().view(torch.int16)
        S0 = torch.from_numpy(S0).to(torch.bfloat16).double().numpy()
        step = pace.pace_gdn_step_bf16
    ref = S0.astype(np.float64)
    for t in range(6):
        inp = pace_synth.token_inputs(w, t)
        dev = {k: v.cuda() for k, v in inp.items()}
        o = torch.empty(n, w.d_v, device="cuda")
        step(S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], pace.PACE_IO_BF16, o, n,
             w.d_k, w.d_v)
        tok = {k: v.reshape(n, -1).double().numpy().squeeze(-1) if v.dim() == 2 else
               v.reshape(n, -1).double().numpy() for k, v in inp.items()}
        ref, o_ref = orc.gdn_step(ref, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        tol = 1e-5 if dtype == "f32" else 3e-2
        assert orc.relative_error(o.cpu().numpy(), o_ref).max() <= tol
