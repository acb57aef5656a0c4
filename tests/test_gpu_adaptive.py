"""Adaptive period (a commit threshold on the accumulated update) against the
fp64 oracle.

Every head advances one token per step; after each step the GPU has marked
the heads whose update since their last rounding reached the threshold (or
whose buffer is full), and pace_commit_period commits exactly those.  The
oracle follows each head from the state the GPU stored at its last commit
(teacher forcing per head) and checks, every step:
  * o_n within the 2e-3 max relative error;
  * the decision: GPU and oracle agree, except where the oracle's fp64 norm is
    within a relative 1e-3 of tau^2 (fp32 against fp64: either is valid);
  * the committed codes of the marked heads against the oracle's encoding of
    its own S_n (ties only, <= 0.1 % of codes).
A threshold too large to reach must reproduce the fixed-period kernels.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth
from tests import parity_utils as pu

pytestmark = pytest.mark.gpu

FILL_COMMIT = 0x100
DECISION_BAND = 1e-3


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


def _setup(w, seed):
    bits = pace_synth.head_bits(w, seed)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    return bits, heads, state


def _run_adaptive(w, tau_rule, T, seed=0):
    pace = _pace()
    bits, heads, state = _setup(w, seed)
    N = len(heads)
    inputs = [pace_synth.token_inputs(w, t, seed=seed, device="cpu") for t in range(T)]
    toks = [pu.host_tokens(x, heads) for x in inputs]
    if tau_rule == "zero":
        tau = 0.0
    else:
        # the median accumulated update after 3 tokens of a fixed period
        _, _, _, norms, _ = orc.pace_run_adaptive(state, toks[:3], w.P, float("inf"))
        tau = float(np.sqrt(np.median(norms[2])))
    tau = float(np.float32(tau))
    tau2 = tau * tau
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pu.load_state(pool, heads, state)
    pool.set_commit_threshold(tau)
    S0 = state.dequantized()
    S = S0.copy()
    gamma = np.ones(N)
    n = np.zeros(N, dtype=np.int64)
    worst, early, late, band = 0.0, 0, 0, 0
    hbits = [bits[h] for _, h in heads]
    for t in range(T):
        dev = {k: v.cuda() for k, v in inputs[t].items()}
        o = pool.decode_step(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"])
        fill = pool.fill().cpu().numpy().reshape(-1).astype(np.int64)
        tok = toks[t]
        S, o_ref = orc.gdn_step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        gamma = gamma * tok["alpha"]
        n += 1
        err = orc.relative_error(o.cpu().numpy().reshape(N, w.d_v), o_ref)
        worst = max(worst, float(err.max()))
        assert err.max() <= pu.O_TOL, (t, float(err.max()))
        assert np.array_equal(fill & 0xff, n), (t, fill, n)
        norm2 = orc.update_norm2(S, S0, gamma)
        gpu_due = ((fill & FILL_COMMIT) != 0) | (fill == w.P)
        ref_due = (n == w.P) | (norm2 >= tau2)
        off = gpu_due != ref_due
        assert np.all(np.abs(norm2[off] - tau2) <= DECISION_BAND * tau2), (t, norm2[off], tau2)
        band += int(off.sum())
        pool.commit_period()
        assert pool.status() == 0
        idx = np.nonzero(gpu_due)[0]
        if idx.size:
            committed, _ = orc.commit(S[idx], [hbits[i] for i in idx], w.axis)
            gc, gs = pu.read_state(pool, [heads[i] for i in idx])
            pu.judge_commit(gc, gs, committed, S[idx], w.axis)
            for j, i in enumerate(idx):
                early += int(n[i] < w.P)
                late += int(n[i] == w.P)
                S0[i] = orc.dequantize(gc[j], gs[j], w.axis)
                S[i] = S0[i]
                gamma[i] = 1.0
                n[i] = 0
        fill = pool.fill().cpu().numpy().reshape(-1)
        assert np.array_equal(fill, n), t
    return worst, early, late, band


@pytest.mark.parametrize("name,axis,over", [
    ("mixed_4_8", "col", {}),
    ("mixed_4_8", "row", {}),
    ("gdn_layer_4b", "col", dict(d_k=64, d_v=64, P=5, io_dtype="f32", outliers=False)),
])
def test_threshold_against_oracle(name, axis, over):
    w = pace_synth.workload(name, B=2, H=4, axis=axis, **over)
    worst, early, late, band = _run_adaptive(w, "median", T=3 * w.P)
    print(name, axis, over, "worst", worst, "early", early, "full", late, "in band", band)
    assert early > 0 and late >= 0


def test_zero_threshold_commits_every_token():
    w = pace_synth.workload("mixed_4_8", B=2, H=4)
    worst, early, late, band = _run_adaptive(w, "zero", T=6)
    assert early == 2 * 4 * 6 and late == 0 and band == 0


@pytest.mark.parametrize("P", [6, 8])
def test_unreachable_threshold_is_the_fixed_period(P):
    """tau = 1e30 runs the tracking kernels (tau^2 overflows to inf in fp32,
    so no head is ever marked early).  With P = 6 both pools run the same
    commit kernel (general period) and must agree bit for bit throughout.
    With P = 8 the fixed pool's commit is the compile-time-period build: the
    commits happen at the same tokens, the committed codes differ at most by
    one at <= 0.1 %, and from the same stored state (copied after each
    commit) the outputs are equal bit for bit."""
    pace = _pace()
    w = pace_synth.workload("mixed_4_8", B=6, P=P)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=3, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    fixed = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    track = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    fixed.load(S)
    track.load(S)
    track.set_commit_threshold(1e30)
    exact = P not in (4, 8, 16)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    for t in range(2 * w.P + 3):
        x = pace_synth.token_inputs(w, t, seed=4, device="cuda")
        o_f = fixed.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        o_t = track.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        assert torch.equal(o_f, o_t), t
        assert torch.equal(fixed.fill(), track.fill()), t
        fixed.commit_period()
        track.commit_period()
        if exact:
            assert torch.equal(fixed.state, track.state), t
        elif (t + 1) % w.P == 0:
            cf, _ = pu.read_state(fixed, heads)
            ct, _ = pu.read_state(track, heads)
            diff = np.concatenate([(a.astype(int) - b.astype(int)).ravel() for a, b in zip(cf, ct)])
            assert np.abs(diff).max() <= 1 and np.mean(diff != 0) <= pu.CODE_DIFF_FRACTION, t
            track.state.copy_(fixed.state)
    assert fixed.status() == 0 and track.status() == 0


def test_marked_head_is_skipped_until_committed():
    pace = _pace()
    w = pace_synth.workload("gdn_layer_4b", B=1, H=2)
    bits = [4, 8]
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=5, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.load(S)
    pool.set_commit_threshold(0.0)
    x = pace_synth.token_inputs(w, 0, seed=6, device="cuda")
    pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    assert torch.all(pool.fill().cpu() == (1 | FILL_COMMIT))
    o = pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    assert torch.isnan(o).all()
    assert pool.status() & pace.PACE_FLAG_BUFFER_FULL
    pool.clear_status()
    pool.commit_period()
    assert torch.all(pool.fill().cpu() == 0) and pool.status() == 0
    for bad in (-1.0, float("nan")):
        with pytest.raises(pace.PaceError):
            pool.set_commit_threshold(bad)
    pool.set_commit_threshold(float("inf"))
    for _ in range(w.P):
        pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    assert torch.all(pool.fill().cpu() == w.P)
