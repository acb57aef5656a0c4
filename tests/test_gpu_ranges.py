"""Slot-range decode and commit (continuous batching with staggered phases).

A range call must do, for its slots, exactly what the full-pool call does,
whatever the launch width and whatever runs beside it on another stream:
per-head arithmetic never depends on the grid, so the results are compared
bit for bit.  A partial range is also checked against the fp64 oracle with
teacher forcing, and slots outside the range must stay untouched.
"""
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


def _pool(w, bits, S):
    pace = _pace()
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.load(S)
    return pool


def _inputs(w, t):
    return pace_synth.token_inputs(w, t, seed=9, device="cuda")


def test_ranges_on_two_streams_match_full_calls_bit_for_bit():
    w = pace_synth.workload("mixed_4_8", B=24)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=4, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    ref, stag = _pool(w, bits, S), _pool(w, bits, S)
    # staggered phases: slots [0, 10) start one token later than slots [10, 24)
    groups = [(0, 10), (10, 14)]
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    o_ref = torch.empty(w.B, w.H, w.d_v, device="cuda")
    o_st = torch.empty_like(o_ref)
    # group 1 takes its first token alone (both pools, same calls)
    x = _inputs(w, 0)
    for pool, o in ((ref, o_ref), (stag, o_st)):
        pool.decode_step_range(10, 14, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o)
    torch.cuda.synchronize()
    for t in range(1, 3 * w.P + 1):
        x = _inputs(w, t)
        # reference: one stream, default launch width, one range after the other
        for b0, nb in groups:
            ref.commit_period_range(b0, nb)
            ref.decode_step_range(b0, nb, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o_ref)
        # staggered: group 0 on stream a, group 1 on stream b, one block per SM each
        ev = torch.cuda.Event()
        ev.record()
        for (b0, nb), st in zip(groups, (sa, sb)):
            st.wait_event(ev)
            with torch.cuda.stream(st):
                stag.commit_period_range(b0, nb, blocks_per_sm=1, stream=st)
                stag.decode_step_range(b0, nb, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o_st,
                                       blocks_per_sm=1, stream=st)
        torch.cuda.current_stream().wait_stream(sa)
        torch.cuda.current_stream().wait_stream(sb)
        torch.cuda.synchronize()
        assert torch.equal(o_ref, o_st), t
    assert ref.status() == 0 and stag.status() == 0
    assert torch.equal(ref.state, stag.state)
    assert torch.equal(ref.buffer, stag.buffer)
    assert torch.equal(ref.fill(), stag.fill())


def test_partial_range_against_oracle_leaves_other_slots_untouched():
    w = pace_synth.workload("gdn_layer_4b", B=6, H=4)
    bits = pace_synth.head_bits(w, 0)
    pace = _pace()
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=2, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    pool.load(S)
    b0, nb = 2, 3
    heads = [(b, h) for b in range(b0, b0 + nb) for h in range(w.H)]
    state, _ = orc.PoolState.from_fp32(
        pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=3).numpy(), [bits[h] for _, h in heads],
        w.axis)
    pu.load_state(pool, heads, state)
    torch.cuda.synchronize()
    before = pool.state.clone()
    o = torch.full((w.B, w.H, w.d_v), 7.0, device="cuda")
    toks, outs = [], []
    for t in range(w.P):
        x = pace_synth.token_inputs(w, t, seed=1, device="cpu")
        d = {k: v.cuda() for k, v in x.items()}
        pool.decode_step_range(b0, nb, d["q"], d["k"], d["v"], d["alpha"], d["beta"], o)
        outs.append(pu.host_tokens({"o": o}, heads)["o"])
        toks.append(pu.host_tokens(x, heads))
    fill = pool.fill().cpu().numpy()
    assert np.all(fill[b0:b0 + nb] == w.P) and np.all(fill[:b0] == 0) and np.all(fill[b0 + nb:] == 0)
    pool.commit_period_range(b0, nb)
    assert pool.status() == 0
    ref_o, S_end, committed, _ = orc.period_reference(state, toks, w.P)
    for n in range(w.P):
        assert orc.relative_error(outs[n], ref_o[n]).max() <= pu.O_TOL
    gc, gs = pu.read_state(pool, heads)
    pu.judge_commit(gc, gs, committed, S_end, w.axis)
    # rows of o and records outside the range were not written
    assert bool((o[:b0] == 7.0).all()) and bool((o[b0 + nb:] == 7.0).all())
    stride = pool.slot_stride
    assert torch.equal(pool.state[: b0 * stride], before[: b0 * stride])
    assert torch.equal(pool.state[(b0 + nb) * stride:], before[(b0 + nb) * stride:])


@pytest.mark.parametrize("args", [(-1, 2, 0), (0, 7, 0), (5, 2, 0), (0, 2, 9), (0, 2, -1)])
def test_bad_ranges_are_rejected(args):
    pace = _pace()
    w = pace_synth.workload("tiny", B=6)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, pace_synth.head_bits(w, 0), io=w.io_dtype)
    x = pace_synth.token_inputs(w, 0, device="cuda")
    o = torch.empty(w.B, w.H, w.d_v, device="cuda")
    b0, nb, bps = args
    with pytest.raises(pace.PaceError):
        pool.decode_step_range(b0, nb, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o,
                               blocks_per_sm=bps)
    with pytest.raises(pace.PaceError):
        pool.commit_period_range(b0, nb, blocks_per_sm=bps)
