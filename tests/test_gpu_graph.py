"""The period step as a CUDA graph.

A period (P pace_decode_step launches and one pace_commit_period) makes no
host synchronisation and allocates nothing, and every launch reads its work
from device-side fill counters, so it can be captured once and replayed.
Two pools start from the same stored state: one runs the period eagerly, the
other replays a captured graph of the same calls on the same input buffers.
Outputs and stored records must be identical, bit for bit, after every
period, for both commit engines (d = 128 column-scale pools) and for the
mma.sync commit alone (row scales).
"""
import pytest
import torch

import pace_synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("axis,engine", [("col", "tcgen05"), ("col", "mma"), ("row", "mma")])
def test_captured_period_equals_eager(axis, engine):
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("mixed_4_8", B=16, axis=axis)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=21, device="cuda").view(w.B, w.H, w.d_v, w.d_k)
    eng = pace.PACE_COMMIT_TCGEN05 if engine == "tcgen05" else pace.PACE_COMMIT_MMA
    eager = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    graphed = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    for pool in (eager, graphed):
        pool.set_commit_engine(eng)
        pool.load(S)
    # input and output buffers the graph reads and writes; refilled each period
    toks = [pace_synth.token_inputs(w, t, seed=22, device="cuda") for t in range(w.P)]
    outs_e = [torch.empty(w.B, w.H, w.d_v, device="cuda") for _ in range(w.P)]
    outs_g = [torch.empty(w.B, w.H, w.d_v, device="cuda") for _ in range(w.P)]

    def period(pool, outs, stream=None):
        for n in range(w.P):
            x = toks[n]
            pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], outs[n], stream)
        pool.commit_period(stream)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        period(graphed, outs_g, side.cuda_stream)
    torch.cuda.synchronize()
    # capture records the launches without running them: both pools are
    # still at the start of period 0
    assert bool((graphed.fill() == 0).all())

    for per in range(3):
        for n, x in enumerate(pace_synth.token_inputs(w, 100 * per + t, seed=23, device="cuda")
                              for t in range(w.P)):
            for key in x:
                toks[n][key].copy_(x[key])
        period(eager, outs_e)
        graph.replay()
        torch.cuda.synchronize()
        for n in range(w.P):
            assert torch.equal(outs_e[n], outs_g[n]), (per, n)
        assert torch.equal(eager.state, graphed.state), per
        assert bool((graphed.fill() == 0).all())
    assert eager.status() == 0 and graphed.status() == 0
