"""Both commit engines (PACE_COMMIT_TCGEN05, the default where it is built
for the shape, and PACE_COMMIT_MMA) against the fp64 oracle, teacher-forced
per period as in test_gpu_decode: outputs within 2e-3, committed codes equal
up to +-1 at rounding ties (<= 0.1 %).  Pools of 192 heads make every CTA of
the persistent grid carry several heads through its pipeline.  Also: the two engines commit the same codes from the same
buffered tokens, and shapes the engine is not built for are refused."""
import numpy as np
import pytest
import torch

import pace_synth
from tests import parity_utils as pu
from tests.test_gpu_decode import _run_periods

pytestmark = pytest.mark.gpu


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


@pytest.mark.parametrize("engine", ["tcgen05", "mma"])
@pytest.mark.parametrize("name,over", [
    ("gdn_layer_4b", dict(B=6)),
    ("mixed_4_8", dict(B=6)),
    ("mixed_4_8", dict(B=6, P=5)),
    ("mixed_4_8", dict(B=6, P=16)),
    ("mixed_4_8", dict(B=3, P=8, io_dtype="f32")),
    ("gdn_layer_4b", dict(B=3, P=1)),
])
def test_commit_engines_against_oracle(name, over, engine):
    pace = _pace()
    w = pace_synth.workload(name, **over)
    eng = pace.PACE_COMMIT_TCGEN05 if engine == "tcgen05" else pace.PACE_COMMIT_MMA
    worst, stats = _run_periods(w, periods=2, seed=3, warm_tokens=32, engine=eng)
    assert worst <= pu.O_TOL
    print(name, over, "worst", worst, [s["codes_differing"] for s in stats])


@pytest.mark.parametrize("P", [8, 6])
def test_engines_commit_the_same_codes(P):
    pace = _pace()
    w = pace_synth.workload("mixed_4_8", B=8, P=P)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=9, device="cuda").view(w.B, w.H, w.d_v, w.d_k)
    a = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    b = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    a.set_commit_engine(pace.PACE_COMMIT_MMA)
    b.set_commit_engine(pace.PACE_COMMIT_TCGEN05)
    a.load(S)
    b.load(S)
    heads = [(x, h) for x in range(w.B) for h in range(w.H)]
    for t in range(3 * w.P):
        x = pace_synth.token_inputs(w, t, seed=10, device="cuda")
        oa = a.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        ob = b.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        assert torch.equal(oa, ob), t   # same stored state: same outputs
        a.commit_period()
        b.commit_period()
        if (t + 1) % w.P == 0:
            ca, sa = pu.read_state(a, heads)
            cb, sb = pu.read_state(b, heads)
            diff = np.concatenate([(u.astype(int) - v.astype(int)).ravel() for u, v in zip(ca, cb)])
            assert np.abs(diff).max() <= 1 and np.mean(diff != 0) <= pu.CODE_DIFF_FRACTION, t
            sd = np.concatenate([np.abs(u.view(np.uint16).astype(int) - v.view(np.uint16).astype(int)).ravel()
                                 for u, v in zip(sa, sb)])
            assert sd.max() <= 1, t
            b.state.copy_(a.state)   # continue from one stored state
    assert a.status() == 0 and b.status() == 0


def test_engine_choice_is_validated():
    pace = _pace()
    row = pace.PacePool(2, 4, 128, 128, 8, [4] * 4, axis="row")
    with pytest.raises(pace.PaceError) as e:
        row.set_commit_engine(pace.PACE_COMMIT_TCGEN05)
    assert e.value.status == 2
    small = pace.PacePool(2, 4, 64, 64, 8, [4] * 4)
    with pytest.raises(pace.PaceError) as e:
        small.set_commit_engine(pace.PACE_COMMIT_TCGEN05)
    assert e.value.status == 2
    f32p16 = pace.PacePool(2, 4, 128, 128, 16, [4] * 4, io="f32")
    with pytest.raises(pace.PaceError) as e:
        f32p16.set_commit_engine(pace.PACE_COMMIT_TCGEN05)
    assert e.value.status == 2
    with pytest.raises(pace.PaceError) as e:
        row.set_commit_engine(7)
    assert e.value.status == 1
    row.set_commit_engine(pace.PACE_COMMIT_MMA)
