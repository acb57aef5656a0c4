"""The pins are strong enough: each plausible mistake planted in a copy of an
oracle function (dropped term, wrong sign, transposed operand, wrong index,
wrong rounding, wrong group axis, wrong nibble order) fails at least one pin.

The mutants live here, on the CPU, and are never used by anything else.
"""
import numpy as np
import pytest

import oracle as orc
from tests import oracle_checks as ck


# ---------------- recurrence mutants ----------------

def _step_factory(kind):
    def step(S, q, k, v, alpha, beta):
        S = np.asarray(S, dtype=np.float64)
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        a = np.asarray(alpha, dtype=np.float64)[:, None, None]
        b = np.asarray(beta, dtype=np.float64)[:, None, None]
        d_k = S.shape[-1]
        kk = k[:, :, None] * k[:, None, :]
        sign = 1.0 if kind == "sign" else -1.0
        trans = np.eye(d_k)[None] + sign * b * kk
        decay = 1.0 if kind == "no_alpha" else a
        prod = np.matmul(S, trans) if kind != "left_multiply" else np.matmul(trans[:, :S.shape[1], :S.shape[1]], S)
        write = v[:, :, None] * k[:, None, :]
        if kind == "alpha_on_write":
            write = a * write
        if kind == "beta_dropped_write":
            S_new = decay * prod + write
        else:
            S_new = decay * prod + b * write
        o = np.matmul(S_new, q[:, :, None])[:, :, 0]
        if kind == "o_before_update":
            o = np.matmul(S, q[:, :, None])[:, :, 0]
        return S_new, o
    return step


STEP_MUTANTS = ["sign", "no_alpha", "left_multiply", "alpha_on_write", "beta_dropped_write",
                "o_before_update"]


def _fails(fn, *args):
    try:
        fn(*args)
    except (AssertionError, ValueError, IndexError):
        return True
    return False


@pytest.mark.parametrize("kind", STEP_MUTANTS)
def test_step_mutant_is_caught(kind):
    mutant = _step_factory(kind)
    caught = (_fails(ck.check_gdn_golden, mutant) or _fails(ck.check_gdn_bruteforce, mutant)
              or _fails(ck.check_gdn_closed_forms, mutant))
    assert caught, kind


def _chunk_factory(kind):
    def chunk(S0, K, V, alpha, beta, q=None):
        N, n, _ = K.shape
        al, be = np.asarray(alpha, float), np.asarray(beta, float)
        gam = np.ones((N, n + 1, n + 1))
        for t in range(1, n + 1):
            for s in range(0, t):
                lo = s + 1 if kind == "gamma_index" else s
                gam[:, t, s] = np.prod(al[:, lo:t], axis=1)
        gamma = gam[:, 1:, 0]
        X = np.matmul(S0, np.swapaxes(K, 1, 2))
        gram = np.matmul(K, np.swapaxes(K, 1, 2))
        rhs = be[:, :, None] * (V - gamma[:, :, None] * np.swapaxes(X, 1, 2))
        U = np.zeros_like(rhs)
        for t in range(n):
            acc = rhs[:, t, :].copy()
            for s in range(t):
                a_ts = be[:, t] * gam[:, t + 1, s + 1] * gram[:, t, s]
                if kind == "sign":
                    acc += a_ts[:, None] * U[:, s, :]
                elif kind == "beta_of_s":
                    acc -= (be[:, s] * gam[:, t + 1, s + 1] * gram[:, t, s])[:, None] * U[:, s, :]
                else:
                    acc -= a_ts[:, None] * U[:, s, :]
            U[:, t, :] = acc
        g_last = gam[:, n, 1:]
        if kind == "no_final_decay":
            g_last = np.ones_like(g_last)
        S_n = gam[:, n, 0][:, None, None] * S0 + np.matmul(np.swapaxes(g_last[:, :, None] * U, 1, 2), K)
        kq = np.matmul(K, q[:, :, None])[:, :, 0]
        o = gam[:, n, 0][:, None] * np.matmul(S0, q[:, :, None])[:, :, 0] + np.sum((g_last * kq)[:, :, None] * U, axis=1)
        return S_n, U, o
    return chunk


@pytest.mark.parametrize("kind", ["sign", "gamma_index", "beta_of_s", "no_final_decay"])
def test_chunk_mutant_is_caught(kind):
    assert _fails(ck.check_chunk_vs_sequential, _chunk_factory(kind), orc.gdn_step), kind


# ---------------- encoder mutants ----------------

def _quant_factory(kind):
    def quantize(S, bits, axis="col"):
        S = np.asarray(S, dtype=np.float32)
        qmax = {4: 7, 8: 127}[bits]
        red = -2 if axis == "col" else -1
        if kind == "axis_swapped":
            red = -1 if axis == "col" else -2
        finite = np.isfinite(S).all(axis=red, keepdims=True)
        absS = np.where(np.isfinite(S), np.abs(S), np.float32(0))
        amax = absS.max(axis=red, keepdims=True).astype(np.float32)
        div = np.float32(qmax + 1 if kind == "qmax_plus_one" else qmax)
        s32 = (amax / div).astype(np.float32)
        with np.errstate(over="ignore"):
            s16 = s32.astype(np.float16)
        s16 = np.where((amax > 0) & (s16 == 0), np.float16(2 ** -24), s16)
        s16 = np.where(np.isinf(s16), np.float16(65504), s16)
        sf = s16.astype(np.float32) if kind != "unrounded_scale" else s32
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = (S / np.where(sf == 0, np.float32(1), sf)).astype(np.float32)
        if kind == "half_up":
            codes = np.floor(ratio + np.float32(0.5))
        elif kind == "truncate":
            codes = np.trunc(ratio)
        else:
            codes = np.rint(ratio)
        lo = -qmax - 1 if kind == "asymmetric_clamp" else -qmax
        codes = np.clip(codes, lo, qmax)
        codes = np.where(sf == 0, 0, codes)
        codes = np.where(finite, codes, 0).astype(np.int8)
        s16 = np.where(finite, s16, np.float16(np.nan)).astype(np.float16)
        flags = 0 if finite.all() else orc.FLAG_NONFINITE
        return codes, np.squeeze(s16, axis=red), flags
    return quantize


@pytest.mark.parametrize("kind", ["axis_swapped", "qmax_plus_one", "unrounded_scale", "half_up",
                                  "truncate", "asymmetric_clamp"])
def test_encoder_mutant_is_caught(kind):
    q = _quant_factory(kind)
    caught = (_fails(ck.check_encoder_golden, q, orc.pack_codes)
              or _fails(ck.check_encoder_bruteforce, q)
              or _fails(ck.check_encoder_invariants, q, orc.dequantize)
              or _fails(ck.check_encoder_special_cases, q, orc.FLAG_NONFINITE, orc.FLAG_SCALE_OVERFLOW))
    assert caught, kind


def test_unmutated_copy_passes():
    """The mutant factory without a mutation is the oracle: every pin passes,
    so the failures above come from the planted mistakes alone."""
    q = _quant_factory("none")
    ck.check_encoder_golden(q, orc.pack_codes)
    ck.check_encoder_bruteforce(q)
    ck.check_encoder_invariants(q, orc.dequantize)
    ck.check_chunk_vs_sequential(_chunk_factory("none"), orc.gdn_step)
    ck.check_gdn_golden(_step_factory("none"))
    ck.check_gdn_bruteforce(_step_factory("none"))
    ck.check_gdn_closed_forms(_step_factory("none"))


def test_pack_mutant_is_caught():
    def pack_swapped(codes, bits):
        codes = np.asarray(codes, dtype=np.int8)
        if bits == 8:
            return codes.view(np.uint8).copy()
        lo = codes[..., 1::2].astype(np.int16) & 0xF
        hi = codes[..., 0::2].astype(np.int16) & 0xF
        return (lo | (hi << 4)).astype(np.uint8)
    assert _fails(ck.check_encoder_golden, orc.quantize, pack_swapped)


# ---------------- tie-checker mutants ----------------

def _ratios_factory(kind):
    def commit_ratios(S_fp64, scales, axis):
        S = np.asarray(S_fp64, dtype=np.float64)
        if kind != "no_fp32_cast":
            S = S.astype(np.float32).astype(np.float64)
        sf = np.asarray(scales, dtype=np.float16).astype(np.float64)
        group = -2 if axis == "col" else -1
        if kind == "axis_swapped":
            group = -1 if axis == "col" else -2
        sf = np.expand_dims(sf, group)
        with np.errstate(divide="ignore", invalid="ignore"):
            return S / sf
    return commit_ratios


@pytest.mark.parametrize("kind", ["no_fp32_cast", "axis_swapped"])
def test_commit_ratios_mutant_is_caught(kind):
    assert _fails(ck.check_commit_ratios, _ratios_factory(kind)), kind


def test_commit_ratios_unmutated_copy_passes():
    ck.check_commit_ratios(_ratios_factory("none"))


# ---------------- adaptive-period mutants ----------------

def _norm_factory(kind):
    def update_norm2(S_n, S0, gamma_n):
        S_n = np.asarray(S_n, dtype=np.float64)
        S0 = np.asarray(S0, dtype=np.float64)
        g = np.asarray(gamma_n, dtype=np.float64)[:, None, None]
        if kind == "no_gamma":
            g = np.ones_like(g)
        if kind == "gamma_squared":
            g = g * g
        delta = S_n - g * S0
        if kind == "max_not_sum":
            return np.max(delta * delta, axis=(1, 2))
        r = np.sum(delta * delta, axis=(1, 2))
        return np.sqrt(r) if kind == "not_squared" else r
    return update_norm2


NORM_MUTANTS = ["no_gamma", "gamma_squared", "max_not_sum", "not_squared"]


@pytest.mark.parametrize("kind", NORM_MUTANTS + ["none"])
def test_update_norm_mutant_is_caught(kind):
    caught = _fails(ck.check_update_norm_closed_forms, _norm_factory(kind), orc.gdn_step)
    assert caught == (kind != "none"), kind


def _adaptive_factory(kind):
    def run(state, tokens, P, tau, step=orc.gdn_step):
        S0 = state.dequantized()
        S = S0.copy()
        N = S.shape[0]
        codes, scales = list(state.codes), list(state.scales)
        gamma, n = np.ones(N), np.zeros(N, dtype=np.int64)
        tau2 = float(tau) * float(tau)
        outs, rounded, norms = [], [], []
        for tok in tokens:
            S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
            outs.append(o)
            gamma = gamma * np.asarray(tok["alpha"], dtype=np.float64)
            n += 1
            norm2 = orc.update_norm2(S, S0, gamma)
            if kind == "strict":
                due = (n == P) | (norm2 > tau2)
            elif kind == "period_off_by_one":
                due = (n == P + 1) | (norm2 >= tau2)
            elif kind == "norm_not_squared_threshold":
                due = (n == P) | (norm2 >= float(tau))
            else:
                due = (n == P) | (norm2 >= tau2)
            for i in np.nonzero(due)[0]:
                c, sc, _ = orc.quantize(S[i:i + 1].astype(np.float32), state.bits[i], state.axis)
                codes[i], scales[i] = c[0], sc[0]
                S0[i] = orc.dequantize(c[0], sc[0], state.axis)
                if kind != "no_restart":
                    S[i] = S0[i]
                if kind != "no_gamma_reset":
                    gamma[i] = 1.0
                n[i] = 0
            rounded.append(due)
            norms.append(norm2)
        return outs, orc.PoolState(codes, scales, state.bits, state.axis), rounded, norms, 0
    return run


ADAPTIVE_MUTANTS = ["strict", "period_off_by_one", "norm_not_squared_threshold", "no_restart",
                    "no_gamma_reset"]


@pytest.mark.parametrize("kind", ADAPTIVE_MUTANTS + ["none"])
def test_adaptive_driver_mutant_is_caught(kind):
    run = _adaptive_factory(kind)
    caught = (_fails(ck.check_adaptive_limits, run, orc.pace_run, orc.per_token_rounding,
                     orc.PoolState, orc.quantize)
              or _fails(ck.check_adaptive_driver_per_head, run, orc.chunk_form, orc.PoolState,
                        orc.quantize, orc.dequantize))
    assert caught == (kind != "none"), kind


# ---------------- pure-write window mutants ----------------

def _e4m3_factory(kind):
    def e4m3(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        _, E = np.frexp(a)
        e = np.maximum(E - 1, -7 if kind == "subnormal_quantum" else -6)
        q = np.ldexp(1.0, e - (2 if kind == "two_mantissa_bits" else 3))
        with np.errstate(invalid="ignore"):
            r = (np.floor(a / q + 0.5) if kind == "ties_away" else np.round(a / q)) * q
        if kind != "no_saturation":
            r = np.minimum(r, 448.0)
        r = np.where(np.isnan(x), np.nan, r)
        return np.copysign(r, x)
    return e4m3


E4M3_MUTANTS = ["subnormal_quantum", "two_mantissa_bits", "ties_away", "no_saturation"]


@pytest.mark.parametrize("kind", E4M3_MUTANTS + ["none"])
def test_e4m3_mutant_is_caught(kind):
    assert _fails(ck.check_e4m3, _e4m3_factory(kind)) == (kind != "none"), kind


def _pw_factory(kind):
    def run(state, tokens, S, step=orc.gdn_step):
        window, outs = [], []
        for tok in tokens:
            k = tok["k"] if kind == "k_not_rounded" else orc.e4m3(tok["k"])
            window.append(dict(tok, k=k, v=orc.e4m3(tok["v"])))
            if kind == "merge_before_readout" and len(window) == S:
                old = window.pop(0)
                S_h, _ = step(state.dequantized(), tok["q"], old["k"], old["v"], old["alpha"], old["beta"])
                state, _ = orc.commit(S_h, state.bits, state.axis)
            S_t = state.dequantized()
            o = np.einsum("nij,nj->ni", S_t, np.asarray(tok["q"], dtype=np.float64))
            for w in window:
                S_t, o = step(S_t, tok["q"], w["k"], w["v"], w["alpha"], w["beta"])
            outs.append(o)
            limit = S + 1 if kind == "window_one_longer" else S
            if kind != "merge_before_readout" and len(window) == limit:
                old = window.pop(-1 if kind == "merge_newest" else 0)
                S_h, _ = step(state.dequantized(), tok["q"], old["k"], old["v"], old["alpha"], old["beta"])
                state, _ = orc.commit(S_h, state.bits, state.axis)
        return outs, state, window, 0
    return run


PW_MUTANTS = ["k_not_rounded", "merge_before_readout", "window_one_longer", "merge_newest"]


@pytest.mark.parametrize("kind", PW_MUTANTS + ["none"])
def test_pw_mutant_is_caught(kind):
    run = _pw_factory(kind)
    caught = (_fails(ck.check_pw_limits, run, orc.per_token_rounding, orc.sequential, orc.e4m3,
                     orc.PoolState, orc.quantize)
              or _fails(ck.check_pw_replay, run, orc.chunk_form, orc.e4m3, orc.PoolState, orc.quantize,
                        orc.dequantize))
    assert caught == (kind != "none"), kind
