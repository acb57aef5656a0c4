"""Pure-write window (pace_window_step) against the fp64 oracle.

Teacher forcing per step: before each step the oracle reads the GPU's
stored history and the pairs in its window; it then
  * rounds the token's k, v to E4M3 itself, and the pair the GPU stored must
    equal it bit for bit;
  * reads out o_t from the history advanced exactly through the window and
    the new pair (2e-3 max relative error);
  * when the window was full, merges the oldest pair into the history and
    encodes it, and the GPU's new history must match (ties only, R15).
A window of one step must be the period-one path on E4M3-rounded inputs,
bit for bit.  The pairs are held either as E4M3 bytes (a pool created with
buffer_e4m3) or as E4M3 values in the io dtype.
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


def _e4m3_table():
    """Value of every E4M3 byte, decoded from its fields (NaN for S.1111.111)."""
    t = np.empty(256)
    for c in range(256):
        s, E, m = c >> 7, (c >> 3) & 15, c & 7
        v = np.nan if (E == 15 and m == 7) else (m * 2.0 ** -9 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7))
        t[c] = -v if s else v
    return t


E4M3 = _e4m3_table()


def _window_rows(pool, w, n):
    """Host copies of the first n window pairs of every head: k, v [N][n][d],
    alpha, beta [N][n] (float64), read through the documented buffer layout."""
    esz = 2 if w.io_dtype == "bf16" else 4
    dt = torch.bfloat16 if esz == 2 else torch.float32
    BH, P, D = w.B * w.H, w.P, w.d_k
    ru = lambda x, a: (x + a - 1) // a * a
    resz = 1 if pool.buffer_e4m3 else esz
    kv_bytes = BH * P * (w.d_k + w.d_v) * resz
    if pool.buffer_e4m3:
        kv = E4M3[pool.buffer[:kv_bytes].cpu().numpy().astype(np.int64)].reshape(BH, P, w.d_k + w.d_v)
    else:
        kv = pool.buffer[:kv_bytes].view(dt).view(BH, P, w.d_k + w.d_v).to(torch.float64).cpu().numpy()
    ab_stride = ru(2 * P * esz, 16)
    ab_off = ru(kv_bytes, 256)
    ab = pool.buffer[ab_off:ab_off + BH * ab_stride].view(BH, ab_stride)[:, :2 * P * esz]
    ab = ab.contiguous().view(dt).view(BH, P, 2).to(torch.float64).cpu().numpy()
    return kv[:, :n, :D], kv[:, :n, D:], ab[:, :n, 0], ab[:, :n, 1]


def _run(w, T, seed=0, e4m3_rows=False):
    pace = _pace()
    bits = pace_synth.head_bits(w, seed)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=seed).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype,
                         buffer_e4m3=e4m3_rows)
    pu.load_state(pool, heads, state)
    hbits = [bits[h] for _, h in heads]
    worst, merges = 0.0, 0
    for t in range(T):
        n_before = int(pool.fill()[0, 0])
        assert bool((pool.fill() == n_before).all())
        hc, hs = pu.read_state(pool, heads)
        H = orc.PoolState(hc, hs, hbits, w.axis)
        K, V, A, B = _window_rows(pool, w, n_before)
        x = pace_synth.token_inputs(w, t, seed=seed, device="cuda")
        tok = pu.host_tokens(x, heads)
        o = pool.window_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"]).cpu().numpy().reshape(
            len(heads), w.d_v)
        assert pool.status() == 0
        k8, v8 = orc.e4m3(tok["k"]), orc.e4m3(tok["v"])
        # readout: history through the window's pairs and the new one
        S_t = H.dequantized()
        for s in range(n_before):
            S_t, _ = orc.gdn_step(S_t, tok["q"], K[:, s], V[:, s], A[:, s], B[:, s])
        S_t, o_ref = orc.gdn_step(S_t, tok["q"], k8, v8, tok["alpha"], tok["beta"])
        err = orc.relative_error(o, o_ref)
        worst = max(worst, float(err.max()))
        assert err.max() <= pu.O_TOL, (t, float(err.max()))
        n_after = n_before + 1
        if n_after == w.P:
            # the oldest pair (row 0, or the new one when P = 1) merges into the history
            if n_before:
                old = (K[:, 0], V[:, 0], A[:, 0], B[:, 0])
            else:
                old = (k8, v8, tok["alpha"], tok["beta"])
            S_h, _ = orc.gdn_step(H.dequantized(), tok["q"], *old)
            committed, _ = orc.commit(S_h, hbits, w.axis)
            gc, gs = pu.read_state(pool, heads)
            pu.judge_commit(gc, gs, committed, S_h, w.axis)
            merges += 1
            n_after -= 1
        assert bool((pool.fill() == n_after).all()), t
        # the new pair sits in the window exactly as E4M3
        if n_after:
            Kn, Vn, _, _ = _window_rows(pool, w, n_after)
            assert np.array_equal(Kn[:, n_after - 1], k8) and np.array_equal(Vn[:, n_after - 1], v8), t
    return worst, merges


@pytest.mark.parametrize("e4m3_rows", [True, False])
@pytest.mark.parametrize("name,over", [
    ("mixed_4_8", {}),
    ("mixed_4_8", dict(axis="row")),
    ("gdn_layer_4b", dict(d_k=64, d_v=64, P=5, io_dtype="f32", outliers=False)),
    ("mixed_4_8", dict(d_k=32, d_v=32, P=16)),
    # 1024-byte fp32 rows: the shift moves two 16-byte pieces per lane, and
    # P = 6 leaves a partial group of four rows
    ("gdn_layer_4b", dict(P=6, io_dtype="f32", outliers=False)),
])
def test_window_against_oracle(name, over, e4m3_rows):
    """The window's pairs as E4M3 bytes (the pool's buffer_e4m3 layout) or as
    E4M3 values in the io dtype."""
    w = pace_synth.workload(name, B=2, H=4, **over)
    worst, merges = _run(w, T=2 * w.P + 3, e4m3_rows=e4m3_rows)
    print(name, over, "e4m3 rows" if e4m3_rows else "io rows", "worst", worst, "merges", merges)
    assert merges == w.P + 4


def test_period_with_an_e4m3_buffer_against_oracle():
    """pace_decode_step / pace_commit_period on a pool whose buffer holds E4M3
    bytes: one teacher-forced period of the oracle on E4M3-rounded k, v."""
    pace = _pace()
    w = pace_synth.workload("mixed_4_8", B=2, H=4)
    bits = pace_synth.head_bits(w, 0)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    S0 = pace_synth.random_state(len(heads), w.d_v, w.d_k, seed=2).numpy()
    state, _ = orc.PoolState.from_fp32(S0, [bits[h] for _, h in heads], w.axis)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype,
                         buffer_e4m3=True)
    pu.load_state(pool, heads, state)
    toks, outs = [], []
    for t in range(w.P):
        x = pace_synth.token_inputs(w, t, seed=2, device="cuda")
        outs.append(pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"]).cpu().numpy()
                    .reshape(len(heads), w.d_v))
        tok = pu.host_tokens(x, heads)
        toks.append(dict(tok, k=orc.e4m3(tok["k"]), v=orc.e4m3(tok["v"])))
    pool.commit_period()
    assert pool.status() == 0
    o_ref, S_end, committed, _ = orc.period_reference(state, toks, w.P)
    for n in range(w.P):
        assert orc.relative_error(outs[n], o_ref[n]).max() <= pu.O_TOL, n
    gc, gs = pu.read_state(pool, heads)
    pu.judge_commit(gc, gs, committed, S_end, w.axis)


def test_window_of_one_is_period_one_on_rounded_inputs():
    pace = _pace()
    w = pace_synth.workload("mixed_4_8", B=3, H=4, P=1)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=4, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    win = pace.PacePool(w.B, w.H, w.d_k, w.d_v, 1, bits, axis=w.axis, io=w.io_dtype)
    per = pace.PacePool(w.B, w.H, w.d_k, w.d_v, 1, bits, axis=w.axis, io=w.io_dtype)
    win.load(S)
    per.load(S)
    for t in range(6):
        x = pace_synth.token_inputs(w, t, seed=5, device="cuda")
        o_w = win.window_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        # the same pair rounded by the oracle, through the period-one path
        r = {key: torch.from_numpy(orc.e4m3(x[key].to(torch.float64).cpu().numpy())).to(
            x[key].dtype).cuda() for key in ("k", "v")}
        o_p = per.decode_step(x["q"], r["k"], r["v"], x["alpha"], x["beta"])
        per.commit_period()
        assert torch.equal(o_w, o_p), t
        assert torch.equal(win.state, per.state), t
        assert torch.equal(win.fill(), per.fill()), t
    assert win.status() == 0 and per.status() == 0


def test_window_rejects_a_threshold_pool():
    pace = _pace()
    w = pace_synth.workload("tiny")
    e = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, pace_synth.head_bits(w, 0), io=w.io_dtype,
                      buffer_e4m3=True)
    with pytest.raises(pace.PaceError):
        e.set_commit_threshold(1.0)
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, pace_synth.head_bits(w, 0), io=w.io_dtype)
    pool.set_commit_threshold(1.0)
    x = pace_synth.token_inputs(w, 0, device="cuda")
    with pytest.raises(pace.PaceError):
        pool.window_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"])
