"""The allocation-free window step (pace_window_step_static) against the
window step that takes caller scratch (pace_window_step), through the C ABI.

pace_window_step_static serves callers that cannot allocate device memory
themselves -- a plugin whose host engine owns the device budget and hands out
only a call's inputs and outputs, or a hot loop that must not call
cudaMalloc.  It keeps its scratch in a device array inside the library, so
this file checks that it gives the results of the entry point it stands in
for: two pools loaded with the same state take the same tokens, one through
each entry point, for several calls in a row.  Outputs must agree within the
readout tolerance of the other parity tests (they come out identical: the
same kernels run on the same data), the stored records and fill counters bit
for bit.  A pool too large for the library's array is refused before
anything is launched.

The file name makes pytest collect it last; it passes alone in a fresh
process as well as after every other test.
"""
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


@pytest.mark.parametrize("name,over", [
    ("mixed_4_8", dict(B=3, H=8)),
    ("gdn_layer_4b", dict(B=2, H=4, d_k=64, d_v=64, P=5, io_dtype="f32", outliers=False)),
])
def test_static_scratch_matches_caller_scratch(name, over):
    pace = _pace()
    w = pace_synth.workload(name, **over)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=7, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    ref = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    new = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    assert pace.pace_window_scratch_bytes(new.handle) <= pace.PACE_WINDOW_STATIC_SCRATCH_BYTES
    ref.load(S)
    new.load(S)
    scratch = torch.empty(pace.pace_window_scratch_bytes(ref.handle), dtype=torch.uint8, device="cuda")
    shape = (w.B, w.H, w.d_v)
    # more than one window length, so that pairs are merged into the history
    for t in range(w.P + 3):
        x = pace_synth.token_inputs(w, t, seed=8, device="cuda")
        args = (x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        o_ref = torch.empty(shape, dtype=torch.float32, device="cuda")
        o_new = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        pace.pace_window_step(ref.handle, *args, o_ref, scratch)
        pace.pace_window_step_static(new.handle, *args, o_new)
        torch.cuda.synchronize()
        err = orc.relative_error(o_new.view(-1, w.d_v).double().cpu().numpy(),
                                 o_ref.view(-1, w.d_v).double().cpu().numpy())
        assert float(err.max()) <= pu.O_TOL, (t, float(err.max()))
        assert torch.equal(new.state, ref.state), t
        assert torch.equal(new.fill(), ref.fill()), t
    assert ref.status() == 0 and new.status() == 0


def test_pool_beyond_the_static_limit_is_refused():
    pace = _pace()
    # bf16 io, d = 128: 512 scratch bytes per head; 16,416 heads need more than 8 MiB
    B, H = 513, 32
    pool = pace.PacePool(B, H, 128, 128, 8, [4] * H)
    assert pace.pace_window_scratch_bytes(pool.handle) > pace.PACE_WINDOW_STATIC_SCRATCH_BYTES
    q = torch.zeros(B, H, 128, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(B, H, dtype=torch.bfloat16, device="cuda")
    o = torch.full((B, H, 128), 7.0, device="cuda")
    before = pool.state.clone()
    with pytest.raises(pace.PaceError) as e:
        pace.pace_window_step_static(pool.handle, q, q, q, g, g, o)
    assert e.value.status == 2   # PACE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and torch.equal(pool.state, before)
    assert bool((pool.fill() == 0).all())
