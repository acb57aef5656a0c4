"""Chunked fp32 prefill (pace_prefill) against the fp64 oracle.

The oracle runs the gated delta rule token by token in fp64 from the stored
(dequantised) state and rounds the final state once; the GPU must give every
token's output within the 2e-3 bar and the same codes up to +-1 flips at
rounding ties.  Ragged token counts (a partial last chunk), both scale axes,
both io dtypes, mixed 4/8-bit heads and smaller head sizes are covered.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu


def _run(w, T, seed=0):
    import bit_recurrent_state_pace_b200 as pace
    bits = pace_synth.head_bits(w, 0)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed + 17).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    pu.load_state(pool, heads, state)
    toks = [pace_synth.token_inputs(w, t, seed=seed, device="cuda") for t in range(T)]
    stack = {key: torch.stack([x[key] for x in toks]).contiguous() for key in toks[0]}
    o = torch.full((T, w.B, w.H, w.d_v), float("nan"), device="cuda")
    pool.prefill(stack["q"], stack["k"], stack["v"], stack["alpha"], stack["beta"], o)
    assert pool.status() == 0
    assert bool((pool.fill() == 0).all())
    host = [pu.host_tokens(x, heads) for x in toks]
    S_end, outs = orc.sequential(state.dequantized(), host)
    committed, _ = orc.commit(S_end, state.bits, state.axis)
    worst = 0.0
    for t in range(T):
        og = o[t].reshape(len(heads), w.d_v).cpu().numpy()
        err = orc.relative_error(og, outs[t])
        worst = max(worst, float(err.max()))
        assert err.max() <= pu.O_TOL, (t, float(err.max()))
    gc, gs = pu.read_state(pool, heads)
    stats = pu.judge_commit(gc, gs, committed, S_end, w.axis)
    return worst, stats


@pytest.mark.parametrize("T", [1, 8, 21, 64])
def test_prefill_lengths(T):
    w = pace_synth.workload("mixed_4_8", B=2, H=4, int8_fraction=0.5)
    worst, stats = _run(w, T)
    print("T", T, "worst", worst, stats)


@pytest.mark.parametrize("io,axis,d", [("bf16", "row", 128), ("f32", "col", 128), ("bf16", "col", 64),
                                       ("f32", "row", 32)])
def test_prefill_io_axis_dims(io, axis, d):
    w = pace_synth.workload("mixed_4_8", B=2, H=4, d_k=d, d_v=d, io_dtype=io, axis=axis,
                            int8_fraction=0.5)
    worst, stats = _run(w, 19)
    print(io, axis, d, "worst", worst, stats)


def test_prefill_then_decode_continues_from_the_prefilled_state():
    """After a prefill the pool is at a period start: a decode step reads the
    prefilled codes like any stored state."""
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("gdn_layer_4b", B=2, H=2)
    bits = pace_synth.head_bits(w, 0)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.state.zero_()
    T = 16
    toks = [pace_synth.token_inputs(w, t, device="cuda") for t in range(T + 1)]
    stack = {key: torch.stack([x[key] for x in toks[:T]]).contiguous() for key in toks[0]}
    pool.prefill(stack["q"], stack["k"], stack["v"], stack["alpha"], stack["beta"])
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    gc, gs = pu.read_state(pool, heads)
    state = orc.PoolState(gc, gs, [bits[h] for _, h in heads], w.axis)
    x = toks[T]
    o = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    ref, _, _, _ = orc.period_reference(state, [pu.host_tokens(x, heads)], w.P)
    assert orc.relative_error(o.reshape(len(heads), w.d_v).cpu().numpy(), ref[0]).max() <= pu.O_TOL


def test_prefill_skips_heads_with_buffered_tokens():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("gdn_layer_4b", B=1, H=2, P=4)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, [4, 4], axis=w.axis, io=w.io_dtype)
    pool.state.zero_()
    x = pace_synth.token_inputs(w, 0, device="cuda")
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    before = pool.state.clone()
    stack = {key: x[key].unsqueeze(0).contiguous() for key in x}
    pool.prefill(stack["q"], stack["k"], stack["v"], stack["alpha"], stack["beta"])
    assert pool.status() & pace.PACE_FLAG_BUFFER_FULL
    assert torch.equal(pool.state, before)
    pool.clear_status()
