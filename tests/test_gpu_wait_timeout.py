"""The decode's bounded mbarrier waits give up, report and leave the context usable.

pace_debug_wait_fault makes the one head of a one-head pool arm its staging
barrier for 16 bytes more than its bulk copies deliver.  Every copy lands,
so nothing is in flight when the wait runs out after 1 ms: the launch must
end by itself, write a NaN output row, leave the pool's records, buffer and
fill untouched, and set PACE_FLAG_TIMEOUT.  After the defaults are restored
the same pool decodes normally.  No wait here is unbounded and nothing
faults: the failure is a barrier that nothing completes.
"""
import pytest
import torch

import pace_synth

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000


def _pool_and_token():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("gdn_layer_4b", B=1, H=1)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, pace_synth.head_bits(w, 0), axis=w.axis,
                         io=w.io_dtype)
    pool.load(pace_synth.random_state(1, w.d_v, w.d_k, seed=5, device="cuda").view(1, 1, w.d_v, w.d_k))
    x = pace_synth.token_inputs(w, 0, seed=1, device="cuda")
    torch.cuda.synchronize()
    return pace, w, pool, x


def test_wait_runs_out_and_reports_timeout():
    pace, w, pool, x = _pool_and_token()
    before = (pool.state.clone(), pool.buffer.clone(), pool.fill().clone())
    pace.pace_debug_wait_fault(pool.handle, LIMIT_NS, 16)
    o = torch.zeros(w.B, w.H, w.d_v, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], o)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    flags = pool.status()
    assert flags & pace.PACE_FLAG_TIMEOUT, pace.pace_status_string(flags)
    assert bool(torch.isnan(o).all())
    assert 0.9 <= ms < 200.0, ms          # gave up after about the limit, not the 2 s default
    assert int(pool.fill()[0, 0]) == 0
    for x0, x1 in zip(before, (pool.state, pool.buffer, pool.fill())):
        assert torch.equal(x0, x1)

    # defaults back: the same pool and context decode normally
    pace.pace_debug_wait_fault(pool.handle, 0, 0)
    pool.clear_status()
    o2 = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    torch.cuda.synchronize()
    assert pool.status() == 0
    assert bool(torch.isfinite(o2).all())
    assert int(pool.fill()[0, 0]) == 1


def test_same_output_as_a_pool_that_never_timed_out():
    pace, w, pool, x = _pool_and_token()
    ref = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"]).clone()
    _, _, pool2, _ = _pool_and_token()
    pace.pace_debug_wait_fault(pool2.handle, LIMIT_NS, 16)
    pool2.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    torch.cuda.synchronize()
    assert pool2.status() & pace.PACE_FLAG_TIMEOUT
    pace.pace_debug_wait_fault(pool2.handle, 0, 0)
    pool2.clear_status()
    got = pool2.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    torch.cuda.synchronize()
    assert pool2.status() == 0
    assert torch.equal(got, ref)


def test_debug_arguments_are_checked_on_the_host():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("gdn_layer_4b", B=2, H=1)
    big = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, [4], axis=w.axis, io=w.io_dtype)
    _, _, one, _ = _pool_and_token()
    bad = [(big, LIMIT_NS, 16),            # more than one head
           (one, 20_000_000, 16),          # limit above 10 ms with a missing transfer
           (one, LIMIT_NS, 8),             # not a multiple of 16
           (one, LIMIT_NS, 32),            # more than 16
           (one, 10, 0),                   # below 1 us
           (one, 3_000_000_000, 0)]        # above the default
    for pool, lim, extra in bad:
        with pytest.raises(pace.PaceError) as e:
            pace.pace_debug_wait_fault(pool.handle, lim, extra)
        assert e.value.status == pace.PACE_ERR_INVALID_ARG
    pace.pace_debug_wait_fault(big.handle, LIMIT_NS, 0)     # a shorter bound alone is fine
    pace.pace_debug_wait_fault(big.handle, 0, 0)
