"""Free-running drift of the GPU path (reported; not a parity gate).

Both sides start from the same oracle-encoded warm state and then run on
their own for 256 tokens (32 periods of P = 8): the GPU through the C ABI,
the fp64 oracle through its periodic driver.  Printed per horizon, as the
mean over heads of ||o - o_ref||_inf / ||o_ref||_inf:

* GPU vs the free-running PACE oracle (how far rounding-order differences
  and tie flips carry);
* GPU, PACE oracle and per-token rounding (P = 1) against the unquantised
  fp64 trajectory from the same start.

End-to-end drift has no reference value on the pages, so only loose things
are asserted: the GPU stays within two roundings' distance of the PACE
oracle, and periodic rounding (oracle and GPU) ends no worse than rounding
after every token, the effect the pages report
("PACE: four-bit recurrent state by rounding less often", TL;DR (1)).
"""
import numpy as np
import pytest

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu

TOKENS = 256


def _mean_err(o, ref):
    return float(np.mean(orc.relative_error(o, ref)))


def test_free_running_drift_report():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("gdn_layer_4b", B=4)
    bits = pace_synth.head_bits(w, 0)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    hb = [bits[h] for _, h in heads]
    state = pu.oracle_warm_state(w, heads, hb, seed=0)

    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pu.load_state(pool, heads, state)
    toks, gpu = [], []
    for t in range(TOKENS):
        inp = pace_synth.token_inputs(w, t, seed=5, device="cpu")
        dev = {k: v.cuda() for k, v in inp.items()}
        o = pool.decode_step(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
        gpu.append(o.cpu().numpy().reshape(len(heads), w.d_v))
        toks.append(pu.host_tokens(inp, heads))
        if (t + 1) % w.P == 0:
            pool.commit_period()
    assert pool.status() == 0

    pace_o, _, _, _, _ = orc.pace_run(state, toks, w.P, step=orc.gdn_step_delta)
    tok_o, _ = orc.per_token_rounding(state, toks, step=orc.gdn_step_delta)
    _, exact_o = orc.sequential(state.dequantized(), toks, step=orc.gdn_step_delta)

    rows = []
    for t in (7, 63, 127, TOKENS - 1):
        rows.append((t + 1, _mean_err(gpu[t], pace_o[t]), _mean_err(gpu[t], exact_o[t]),
                     _mean_err(pace_o[t], exact_o[t]), _mean_err(tok_o[t], exact_o[t])))
    print("\ntokens  gpu-vs-pace  gpu-vs-exact  pace-vs-exact  per-token-vs-exact")
    for r in rows:
        print(f"{r[0]:6d}  {r[1]:.3e}    {r[2]:.3e}     {r[3]:.3e}      {r[4]:.3e}")

    late = slice(TOKENS // 2, TOKENS)
    gpu_vs_pace = np.mean([_mean_err(gpu[t], pace_o[t]) for t in range(TOKENS)[late]])
    pace_vs_exact = np.mean([_mean_err(pace_o[t], exact_o[t]) for t in range(TOKENS)[late]])
    tok_vs_exact = np.mean([_mean_err(tok_o[t], exact_o[t]) for t in range(TOKENS)[late]])
    gpu_vs_exact = np.mean([_mean_err(gpu[t], exact_o[t]) for t in range(TOKENS)[late]])
    # tie flips may decorrelate the two roundings over time, but never by more
    # than two independent roundings of the same trajectory would
    assert gpu_vs_pace <= max(2.0 * pace_vs_exact, 1e-4), (gpu_vs_pace, pace_vs_exact)
    assert pace_vs_exact <= tok_vs_exact, (pace_vs_exact, tok_vs_exact)
    assert gpu_vs_exact <= tok_vs_exact, (gpu_vs_exact, tok_vs_exact)
