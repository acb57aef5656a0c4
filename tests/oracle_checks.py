"""Pins of the fp64 oracle against things other than itself.

Each ``check_*`` function takes the oracle function(s) it pins as arguments,
so ``test_oracle_pins.py`` runs them on the oracle and
``test_oracle_mutants.py`` runs them on deliberately broken copies of it (the
planted mistakes live only in those CPU-side copies).  A check raises
``AssertionError`` when the implementation disagrees with the pin.

What the pins are (none of them re-types an oracle formula in the oracle's own
arithmetic):

* hand-derived worked examples in ``tests/golden/`` (the pages print none);
* exact rational brute force of the encoder and of the recurrence on tiny
  inputs, with an exact round-to-nearest-even routine written here;
* closed forms of the gated delta rule (no write, no decay, the overwrite
  property of the delta rule, orthonormal keys);
* invariants of the encoder (error bound, idempotence, exhaustive scale
  round trip, the absmax entry maps to +-qmax, axis transposition);
* consistency between independently written forms (chunk vs sequential,
  periodic without rounding vs sequential, P = 1 vs per-token rounding).
"""
from __future__ import annotations

import os
from fractions import Fraction
from typing import Dict, List

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# exact rounding (independent of numpy's float types)
# --------------------------------------------------------------------------

def round_rne(r: Fraction, mant_bits: int, emin: int, emax: int) -> Fraction:
    """Round a rational to the nearest binary float with ``mant_bits`` stored
    significand bits, min normal exponent ``emin`` and max exponent ``emax``;
    ties to even; overflow returns +-inf as a float."""
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - mant_bits)
    m = a / quantum
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    res = n * quantum
    if res >= Fraction(2) ** (emax + 1):
        return float("inf") * sign
    return sign * res


def rne_fp32(r: Fraction):
    return round_rne(r, 23, -126, 127)


def rne_fp16(r: Fraction):
    return round_rne(r, 10, -14, 15)


def rint_even(r: Fraction) -> int:
    n = r.numerator // r.denominator
    rem = r - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def exact_encode_group(xs: List[float], qmax: int):
    """Brute-force encoder of one finite group: every step in exact rationals
    followed by an explicit rounding to the format the step produces."""
    fx = [Fraction(float(x)) for x in xs]
    amax = max(abs(x) for x in fx)
    s32 = rne_fp32(amax / qmax)
    s16 = rne_fp16(s32)
    if s16 == float("inf"):
        s16 = Fraction(65504)
    if amax > 0 and s16 == 0:
        s16 = Fraction(1, 2 ** 24)
    if s16 == 0:
        return [0] * len(xs), s16
    codes = []
    for x in fx:
        r32 = rne_fp32(x / s16)
        codes.append(max(-qmax, min(qmax, rint_even(r32))))
    return codes, s16


# --------------------------------------------------------------------------
# golden fixtures
# --------------------------------------------------------------------------

def load_encoder_example():
    rows, cases = [], []
    with open(os.path.join(GOLDEN, "encoder_worked_example.txt")) as f:
        cur = None
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "matrix":
                rows.append([float(x) for x in tok[1:]])
            elif tok[0] == "case":
                cur = {"bits": int(tok[1]), "axis": tok[2]}
                cases.append(cur)
            elif tok[0] == "scales":
                cur["scales"] = [int(x, 16) for x in tok[1:]]
            elif tok[0] == "codes":
                cur["codes"] = [int(x) for x in tok[1:]]
            elif tok[0] == "bytes":
                cur["bytes"] = [int(x, 16) for x in tok[1:]]
    return np.array(rows, dtype=np.float32), cases


def load_gdn_example():
    data: Dict[str, list] = {}
    toks = []
    with open(os.path.join(GOLDEN, "gdn_two_token_example.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "token":
                d = {}
                i = 2
                while i < len(tok):
                    key = tok[i]
                    n = 2 if key in ("k", "v", "q") else 1
                    d[key] = [Fraction(x) for x in tok[i + 1:i + 1 + n]]
                    i += 1 + n
                toks.append(d)
            else:
                data.setdefault(tok[0], []).append([Fraction(x) for x in tok[1:]])
    return data, toks


# --------------------------------------------------------------------------
# encoder checks
# --------------------------------------------------------------------------

def check_encoder_golden(quantize, pack_codes):
    S, cases = load_encoder_example()
    for c in cases:
        codes, scales, flags = quantize(S[None], c["bits"], c["axis"])
        assert flags == 0
        assert codes[0].ravel().tolist() == c["codes"], c
        assert scales[0].view(np.uint16).tolist() == c["scales"], c
        assert pack_codes(codes[0], c["bits"]).ravel().tolist() == c["bytes"], c


def check_encoder_bruteforce(quantize, seed=0, n_groups=60):
    rng = np.random.default_rng(seed)
    for bits, qmax in ((4, 7), (8, 127)):
        for g in range(n_groups):
            size = int(rng.integers(1, 6))
            mag = 10.0 ** rng.uniform(-9, 6)
            xs = (rng.standard_normal(size) * mag).astype(np.float32)
            if g % 7 == 0:          # place exact ties x / s = k + 1/2
                s = np.float32(np.float16(mag / qmax * 0.9))
                if s > 0:
                    xs[0] = np.float32(qmax) * s
                    if size > 1:
                        xs[1] = np.float32(2.5) * s
            exp_codes, exp_s16 = exact_encode_group(list(xs), qmax)
            S = xs.reshape(1, size, 1)                     # one column
            codes, scales, _ = quantize(S, bits, "col")
            assert codes[0, :, 0].tolist() == exp_codes, (bits, xs)
            assert Fraction(float(scales[0, 0])) == exp_s16, (bits, xs)


def check_encoder_invariants(quantize, dequantize, seed=0):
    rng = np.random.default_rng(seed)
    for bits, qmax in ((4, 7), (8, 127)):
        for axis in ("col", "row"):
            S = rng.standard_normal((3, 12, 20)).astype(np.float32)
            S[:, :, 3] *= 40.0          # a loud column
            S[:, 5, :] *= 0.01          # a quiet row
            codes, scales, flags = quantize(S, bits, axis)
            assert flags == 0
            assert codes.min() >= -qmax and codes.max() <= qmax
            Sh = dequantize(codes, scales, axis)
            red = -2 if axis == "col" else -1
            sf = np.expand_dims(scales.astype(np.float32), red)
            # error bound |x - x_hat| <= sf / 2
            assert np.all(np.abs(S.astype(np.float64) - Sh) <= sf.astype(np.float64) / 2 + 0.0)
            # the absmax entry of every group maps to +-qmax
            amax_codes = np.take_along_axis(
                np.abs(codes), np.expand_dims(np.argmax(np.abs(S), axis=red), red), axis=red)
            assert np.all(amax_codes == qmax)
            # idempotence: quant(deq(quant(S))) == quant(S)
            c2, s2, _ = quantize(Sh, bits, axis)
            assert np.array_equal(c2, codes) and np.array_equal(s2.view(np.uint16), scales.view(np.uint16))
        # axis transposition: column groups of S are row groups of S^T
        S = rng.standard_normal((2, 9, 14)).astype(np.float32)
        cc, sc, _ = quantize(S, bits, "col")
        cr, sr, _ = quantize(np.swapaxes(S, 1, 2).copy(), bits, "row")
        assert np.array_equal(cc, np.swapaxes(cr, 1, 2))
        assert np.array_equal(sc.view(np.uint16), sr.view(np.uint16))


def check_encoder_exhaustive_scales(quantize, dequantize):
    """Every positive finite fp16 scale s and every code c round-trips: a
    group holding qmax*s (so the scale is exactly s) and c*s encodes to
    scale s and codes (qmax, c)."""
    all16 = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)   # positive finite
    s = all16.astype(np.float32)
    for bits, qmax in ((4, 7), (8, 127)):
        for c in range(-qmax, qmax + 1):
            S = np.stack([np.float32(qmax) * s, np.float32(c) * s], axis=-1)  # [n, 2]
            S = S[:, :, None]                                                  # column groups
            codes, scales, flags = quantize(S, bits, "col")
            assert flags == 0
            assert np.array_equal(scales[:, 0].view(np.uint16), all16.view(np.uint16)), (bits, c)
            assert np.all(codes[:, 0, 0] == qmax) and np.all(codes[:, 1, 0] == c), (bits, c)
            back = dequantize(codes, scales, "col")
            assert np.array_equal(back[:, 1, 0], np.float32(c) * s)


def check_encoder_special_cases(quantize, FLAG_NONFINITE, FLAG_SCALE_OVERFLOW):
    for bits, qmax in ((4, 7), (8, 127)):
        z = np.zeros((1, 4, 1), np.float32)
        codes, scales, flags = quantize(z, bits, "col")
        assert flags == 0 and np.all(codes == 0) and scales[0, 0] == 0
        tiny = np.array([1e-12, -3e-13, 0, 2e-13], np.float32).reshape(1, 4, 1)
        codes, scales, flags = quantize(tiny, bits, "col")
        assert scales[0, 0].view(np.uint16) == 1           # 2^-24 floor
        assert codes[0, 0, 0] == 0                          # 1e-12 / 2^-24 << 1/2
        huge = np.array([1e30, -1e30, 1.0, 0], np.float32).reshape(1, 4, 1)
        codes, scales, flags = quantize(huge, bits, "col")
        assert flags & FLAG_SCALE_OVERFLOW
        assert scales[0, 0] == np.float16(65504)
        assert codes[0, 0, 0] == qmax and codes[0, 1, 0] == -qmax
        bad = np.array([1.0, np.nan, 2.0, 0], np.float32).reshape(1, 4, 1)
        codes, scales, flags = quantize(bad, bits, "col")
        assert flags & FLAG_NONFINITE
        assert np.isnan(scales[0, 0]) and np.all(codes == 0)
        # a single entry always encodes to +-qmax
        for x in (3.0, -0.001, 1234.5):
            c, s, _ = quantize(np.array([[[x]]], np.float32), bits, "col")
            assert c[0, 0, 0] == (qmax if x > 0 else -qmax)


def check_rounding_primitives():
    """numpy float16 conversion, float32 division and rint match the exact
    rounding routine above (pins the encoder's arithmetic primitives)."""
    rng = np.random.default_rng(1)
    # fp16 conversion on midpoints and their fp32 neighbours, over all binades
    h = np.arange(0, 0x7BFF, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = ((h[:-1] + np.diff(h) / 2)).astype(np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                           rng.uniform(0, 70000, 3000).astype(np.float32),
                           (10.0 ** rng.uniform(-9, -4, 2000)).astype(np.float32)])
    with np.errstate(over="ignore"):
        got = vals.astype(np.float16)
    for x, g in zip(vals[::3], got[::3]):
        exp = rne_fp16(Fraction(float(x)))
        assert (np.isinf(g) and exp == float("inf")) or Fraction(float(g)) == exp, x
    # fp32 division
    for _ in range(1500):
        x = np.float32(rng.standard_normal() * 10.0 ** rng.uniform(-6, 6))
        s = np.float32(np.float16(10.0 ** rng.uniform(-6, 4)))
        if s == 0:
            continue
        q = np.float32(x) / np.float32(s)
        assert Fraction(float(q)) == rne_fp32(Fraction(float(x)) / Fraction(float(s)))
    # rint ties to even
    ties = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 6.5, 7.5, 126.5], np.float32)
    assert np.rint(ties).tolist() == [0, 2, 2, -0, -2, -2, 6, 8, 126]


def check_pack_roundtrip(pack_codes, unpack_codes, seed=0):
    rng = np.random.default_rng(seed)
    for bits, qmax in ((4, 7), (8, 127)):
        c = rng.integers(-qmax, qmax + 1, size=(3, 5, 16)).astype(np.int8)
        p = pack_codes(c, bits)
        assert p.dtype == np.uint8 and p.shape[-1] == 16 * bits // 8
        assert np.array_equal(unpack_codes(p, bits), c)
    # nibble order: even j low
    assert pack_codes(np.array([[1, -2]], np.int8), 4).tolist() == [[0xE1]]


def check_commit_ratios(commit_ratios):
    """x / sf of the period-end state, worked by hand on a 2 x 3 state
    (d_v != d_k, so a scale vector expanded on the wrong axis cannot
    broadcast) and on a 2 x 2 state with distinct scales (where it can, and
    gives other numbers).  The entry 1.25 - 2^-30 rounds to 1.25 in fp32
    ("PACE: A New 4-Bit ...", section "Channel-Aligned Encoding": the state is
    encoded from its fp32 value), so with sf = 0.5 its ratio is the tie 2.5
    exactly; in fp64 it would sit 2^-29 below the tie."""
    S = np.array([[1.5, -3.0, 0.75],
                  [1.25 - 2.0 ** -30, 0.0, -7.0]], dtype=np.float64)
    # COL: one scale per key channel j (columns)
    r = commit_ratios(S, np.array([0.5, 1.0, 0.25], np.float16), "col")
    assert r.shape == (2, 3)
    assert r.tolist() == [[3.0, -3.0, 3.0], [2.5, 0.0, -28.0]], r.tolist()
    # ROW: one scale per value channel i (rows)
    r = commit_ratios(S, np.array([0.25, 0.375], np.float16), "row")
    assert r.tolist() == [[6.0, -12.0, 3.0], [10.0 / 3.0, 0.0, -56.0 / 3.0]], r.tolist()
    # square state, scales 1 and 4: COL divides column 1 by 4, ROW row 1
    S2 = np.array([[8.0, 8.0], [-2.0, 6.0]])
    sc = np.array([1.0, 4.0], np.float16)
    assert commit_ratios(S2, sc, "col").tolist() == [[8.0, 2.0], [-2.0, 1.5]]
    assert commit_ratios(S2, sc, "row").tolist() == [[8.0, 8.0], [-0.5, 1.5]]
    # scales are read as the fp16 values stored in the record
    r = commit_ratios(np.array([[0.5]]), np.array([0.1], np.float16), "col")
    assert r.tolist() == [[0.5 / (1638.0 / 16384.0)]], r.tolist()


# --------------------------------------------------------------------------
# recurrence checks
# --------------------------------------------------------------------------

def _frac_matmul(A, B):
    return [[sum(A[i][t] * B[t][j] for t in range(len(B))) for j in range(len(B[0]))]
            for i in range(len(A))]


def check_gdn_golden(gdn_step):
    data, toks = load_gdn_example()
    S = np.array([[float(x) for x in r] for r in data["s0"]])[None]
    for idx, tok in enumerate(toks, start=1):
        S, o = gdn_step(S, np.array([[float(x) for x in tok["q"]]]),
                        np.array([[float(x) for x in tok["k"]]]),
                        np.array([[float(x) for x in tok["v"]]]),
                        np.array([float(tok["alpha"][0])]), np.array([float(tok["beta"][0])]))
        exp_S = np.array([[float(x) for x in r] for r in data["s%d" % idx]])
        exp_o = np.array([float(x) for x in data["o%d" % idx][0]])
        assert np.allclose(S[0], exp_S, rtol=0, atol=1e-14), (idx, S[0], exp_S)
        assert np.allclose(o[0], exp_o, rtol=0, atol=1e-14), (idx, o[0], exp_o)


def _dyadic(rng, shape, bits=6):
    return rng.integers(-(2 ** bits), 2 ** bits + 1, size=shape) / 2.0 ** bits


def check_gdn_bruteforce(gdn_step, seed=0):
    """Tiny inputs (d <= 4, T <= 8) against the unrolled solution of the
    linear recurrence in exact rationals:
    S_T = S_0 prod_t M_t + sum_t b_t v_t k_t^T prod_{r>t} M_r, with
    M_t = a_t (I - b_t k_t k_t^T)."""
    rng = np.random.default_rng(seed)
    for trial in range(12):
        d_v, d_k = int(rng.integers(1, 5)), int(rng.integers(1, 5))
        T = int(rng.integers(1, 9))
        S0 = _dyadic(rng, (d_v, d_k))
        toks = [dict(q=_dyadic(rng, d_k), k=_dyadic(rng, d_k), v=_dyadic(rng, d_v),
                     alpha=rng.integers(1, 9) / 8.0, beta=rng.integers(0, 9) / 8.0) for _ in range(T)]
        F = Fraction
        Ms = []
        for tk in toks:
            k = [F(x) for x in tk["k"]]
            Ms.append([[F(tk["alpha"]) * ((1 if i == j else 0) - F(tk["beta"]) * k[i] * k[j])
                        for j in range(d_k)] for i in range(d_k)])
        total = [[F(x) for x in r] for r in S0]
        for M in Ms:
            total = _frac_matmul(total, M)
        for t, tk in enumerate(toks):
            W = [[F(tk["beta"]) * F(vi) * F(kj) for kj in tk["k"]] for vi in tk["v"]]
            for M in Ms[t + 1:]:
                W = _frac_matmul(W, M)
            total = [[total[i][j] + W[i][j] for j in range(d_k)] for i in range(d_v)]
        o_exact = [sum(total[i][j] * F(toks[-1]["q"][j]) for j in range(d_k)) for i in range(d_v)]
        S = S0[None].astype(np.float64)
        for tk in toks:
            S, o = gdn_step(S, tk["q"][None], tk["k"][None], tk["v"][None],
                            np.array([tk["alpha"]]), np.array([tk["beta"]]))
        assert np.allclose(S[0], np.array(total, dtype=float), rtol=1e-12, atol=1e-12), trial
        assert np.allclose(o[0], np.array(o_exact, dtype=float), rtol=1e-12, atol=1e-12), trial


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def check_gdn_closed_forms(gdn_step, seed=0):
    rng = np.random.default_rng(seed)
    N, d_v, d_k = 3, 6, 5
    S0 = rng.standard_normal((N, d_v, d_k))
    q, k, v = _unit(rng, N, d_k), _unit(rng, N, d_k), rng.standard_normal((N, d_v))
    # (i) alpha = 1, beta = 0: nothing changes, o = S q
    S1, o = gdn_step(S0, q, k, v, np.ones(N), np.zeros(N))
    assert np.allclose(S1, S0, atol=1e-14) and np.allclose(o, np.einsum("nij,nj->ni", S0, q), atol=1e-13)
    # (ii) beta = 0: pure decay by alpha
    a = rng.uniform(0.5, 1.0, N)
    S1, _ = gdn_step(S0, q, k, v, a, np.zeros(N))
    assert np.allclose(S1, a[:, None, None] * S0, atol=1e-14)
    # (iii) beta = 1, |k| = 1: the new state maps k exactly to v (overwrite),
    #       and leaves directions orthogonal to k decayed by alpha
    S1, _ = gdn_step(S0, q, k, v, a, np.ones(N))
    assert np.allclose(np.einsum("nij,nj->ni", S1, k), v, atol=1e-13)
    x = rng.standard_normal((N, d_k))
    x -= np.sum(x * k, axis=-1, keepdims=True) * k
    assert np.allclose(np.einsum("nij,nj->ni", S1, x), a[:, None] * np.einsum("nij,nj->ni", S0, x), atol=1e-13)
    # (iv) orthonormal keys, beta = 1, S0 = 0: S_T = sum_t gamma_{T/t} v_t k_t^T
    T = 4
    Q, _ = np.linalg.qr(rng.standard_normal((d_k, d_k)))
    keys = Q[:, :T].T                                   # [T, d_k], orthonormal
    vals = rng.standard_normal((T, d_v))
    al = rng.uniform(0.6, 1.0, T)
    S = np.zeros((1, d_v, d_k))
    for t in range(T):
        S, _ = gdn_step(S, keys[t][None], keys[t][None], vals[t][None], al[t:t + 1], np.ones(1))
    exp = sum(np.prod(al[t + 1:]) * np.outer(vals[t], keys[t]) for t in range(T))
    assert np.allclose(S[0], exp, atol=1e-13)


def random_tokens(rng, N, T, d_k, d_v):
    toks = []
    for _ in range(T):
        toks.append(dict(q=_unit(rng, N, d_k), k=_unit(rng, N, d_k), v=rng.standard_normal((N, d_v)),
                         alpha=np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal(N)))),
                         beta=1.0 / (1.0 + np.exp(-rng.standard_normal(N)))))
    return toks


def check_chunk_vs_sequential(chunk_form, gdn_step, seed=0):
    rng = np.random.default_rng(seed)
    N, d_v, d_k = 4, 12, 10
    for n in (1, 2, 3, 5, 8, 16):
        S0 = rng.standard_normal((N, d_v, d_k))
        toks = random_tokens(rng, N, n, d_k, d_v)
        S = S0
        for tk in toks:
            S, o = gdn_step(S, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
        K = np.stack([t["k"] for t in toks], 1)
        V = np.stack([t["v"] for t in toks], 1)
        A = np.stack([t["alpha"] for t in toks], 1)
        Bt = np.stack([t["beta"] for t in toks], 1)
        Sn, U, on = chunk_form(S0, K, V, A, Bt, toks[-1]["q"])
        scale = np.max(np.abs(S))
        assert np.max(np.abs(Sn - S)) <= 1e-12 * scale, n
        assert np.max(np.abs(on - o)) <= 1e-12 * np.max(np.abs(o)), n


def check_step_forms_agree(gdn_step, gdn_step_delta, seed=0):
    rng = np.random.default_rng(seed)
    N, d_v, d_k = 5, 7, 9
    S = rng.standard_normal((N, d_v, d_k))
    for tk in random_tokens(rng, N, 6, d_k, d_v):
        S1, o1 = gdn_step(S, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
        S2, o2 = gdn_step_delta(S, tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
        assert np.allclose(S1, S2, rtol=1e-13, atol=1e-13) and np.allclose(o1, o2, rtol=1e-13, atol=1e-13)
        S = S1


# ---------------- adaptive period ----------------

def _random_pool_state(rng, N, d_v, d_k, bits, axis, quantize):
    S = (rng.standard_normal((N, d_v, d_k)) * 0.5).astype(np.float32)
    codes, scales = [], []
    for i in range(N):
        c, s, _ = quantize(S[i:i + 1], bits[i], axis)
        codes.append(c[0])
        scales.append(s[0])
    return codes, scales


def check_update_norm_closed_forms(update_norm2, gdn_step, seed=0):
    """||S_n - gamma_n S0||_F^2 against what the recurrence fixes: zero without
    writes, the rank-1 norm after one token, and the one-token recursion
    N_n = a^2 N_{n-1} + 2 a u.(Delta_{n-1} k) + |u|^2 |k|^2 with
    u = b (v - a S_{n-1} k), which follows from S_n = a S_{n-1} + u k^T."""
    rng = np.random.default_rng(seed)
    N, d_v, d_k = 5, 9, 7
    S0 = rng.standard_normal((N, d_v, d_k))
    # no writes (beta = 0): the state only decays
    S, g = S0, np.ones(N)
    for tk in random_tokens(rng, N, 4, d_k, d_v):
        S, _ = gdn_step(S, tk["q"], tk["k"], tk["v"], tk["alpha"], np.zeros(N))
        g = g * tk["alpha"]
        assert np.all(update_norm2(S, S0, g) <= 1e-26 * np.sum(S0 * S0, axis=(1, 2)))
    # one token: Delta_1 = b (v - a S0 k) k^T, a rank-1 matrix
    tk = random_tokens(rng, N, 1, d_k, d_v)[0]
    k = tk["k"] * rng.uniform(0.5, 2.0, (N, 1))
    S1, _ = gdn_step(S0, tk["q"], k, tk["v"], tk["alpha"], tk["beta"])
    err = tk["v"] - tk["alpha"][:, None] * np.einsum("nij,nj->ni", S0, k)
    ref = tk["beta"] ** 2 * np.sum(err * err, axis=1) * np.sum(k * k, axis=1)
    got = update_norm2(S1, S0, tk["alpha"])
    assert np.allclose(got, ref, rtol=1e-12, atol=0), (got, ref)
    # the recursion over several tokens
    S, g, prev = S0, np.ones(N), np.zeros(N)
    for tk in random_tokens(rng, N, 6, d_k, d_v):
        a, b = tk["alpha"], tk["beta"]
        Sk = np.einsum("nij,nj->ni", S, tk["k"])
        delta_k = Sk - g[:, None] * np.einsum("nij,nj->ni", S0, tk["k"])
        u = b[:, None] * (tk["v"] - a[:, None] * Sk)
        rec = a * a * prev + 2 * a * np.sum(u * delta_k, 1) + np.sum(u * u, 1) * np.sum(tk["k"] ** 2, 1)
        S, _ = gdn_step(S, tk["q"], tk["k"], tk["v"], a, b)
        g = g * a
        got = update_norm2(S, S0, g)
        assert np.allclose(got, rec, rtol=1e-10, atol=0), (got, rec)
        prev = got


def check_adaptive_limits(pace_run_adaptive, pace_run, per_token_rounding, PoolState, quantize,
                          seed=0):
    """tau = inf is the fixed period P; tau = 0 rounds after every token."""
    rng = np.random.default_rng(seed)
    N, d_v, d_k, P = 6, 8, 8, 4
    bits = [4, 8, 4, 4, 8, 4]
    for axis in ("col", "row"):
        codes, scales = _random_pool_state(rng, N, d_v, d_k, bits, axis, quantize)
        st = PoolState(codes, scales, bits, axis)
        toks = random_tokens(rng, N, 11, d_k, d_v)
        o_a, fin_a, rounded, _, _ = pace_run_adaptive(st, toks, P, float("inf"))
        o_f, fin_f, _, _, _ = pace_run(st, toks, P)
        for x, y in zip(o_a, o_f):
            assert np.array_equal(x, y)
        assert all(np.array_equal(a, b) for a, b in zip(fin_a.codes, fin_f.codes))
        assert [bool(r.all()) for r in rounded] == [(t + 1) % P == 0 for t in range(len(toks))]
        o_a, fin_a, rounded, _, _ = pace_run_adaptive(st, toks, P, 0.0)
        o_p, fin_p = per_token_rounding(st, toks)
        for x, y in zip(o_a, o_p):
            assert np.array_equal(x, y)
        assert all(np.array_equal(a, b) for a, b in zip(fin_a.codes, fin_p.codes))
        assert all(r.all() for r in rounded)
        # a pure decay has a zero update, which still reaches tau = 0
        still = [dict(tk, beta=np.zeros(N)) for tk in toks]
        _, _, rounded, norms, _ = pace_run_adaptive(st, still, P, 0.0)
        assert all(r.all() for r in rounded) and all(np.all(x == 0.0) for x in norms)


def check_adaptive_driver_per_head(pace_run_adaptive, chunk_form, PoolState, quantize, dequantize,
                                   seed=0):
    """A finite threshold, replayed head by head in chunk form: each head keeps
    its own buffer, its state after n tokens and the accumulated update
    sum_s gamma_{n/s} u_s k_s^T both come from chunk_form, and it is rounded
    when the update's squared norm reaches tau^2 or the buffer holds P."""
    rng = np.random.default_rng(seed)
    N, d_v, d_k, P, T, tau = 6, 8, 8, 5, 24, 2.0
    bits = [4, 4, 8, 4, 8, 4]
    axis = "col"
    codes, scales = _random_pool_state(rng, N, d_v, d_k, bits, axis, quantize)
    st = PoolState(codes, scales, bits, axis)
    toks = random_tokens(rng, N, T, d_k, d_v)
    o_a, fin_a, rounded, norms, _ = pace_run_adaptive(st, toks, P, tau)
    n_rounded = 0
    for i in range(N):
        c, s = codes[i], scales[i]
        buf = []
        for t, tk in enumerate(toks):
            buf.append({key: np.asarray(val)[i:i + 1] for key, val in tk.items()})
            S0 = dequantize(c, s, axis).astype(np.float64)[None]
            K = np.stack([b["k"] for b in buf], 1)
            V = np.stack([b["v"] for b in buf], 1)
            A = np.stack([b["alpha"] for b in buf], 1)
            B = np.stack([b["beta"] for b in buf], 1)
            S_n, U, o = chunk_form(S0, K, V, A, B, buf[-1]["q"])
            n = len(buf)
            g = np.array([np.prod(A[0, s + 1:]) for s in range(n)])   # gamma_{n/s}
            delta = np.einsum("s,si,sj->ij", g, U[0], K[0])
            norm2 = float(np.sum(delta * delta))
            assert abs(norm2 - tau * tau) > 1e-9 * tau * tau, "tie: choose another seed"
            assert np.allclose(norms[t][i], norm2, rtol=1e-9), (i, t)
            assert np.allclose(o_a[t][i], o[0], rtol=1e-10, atol=1e-12), (i, t)
            due = n == P or norm2 >= tau * tau
            assert bool(rounded[t][i]) == due, (i, t)
            if due:
                n_rounded += 1
                c2, s2, _ = quantize(S_n.astype(np.float32), bits[i], axis)
                c, s = c2[0], s2[0]
                buf = []
        assert np.array_equal(fin_a.codes[i], c) and np.array_equal(
            fin_a.scales[i].view(np.uint16), np.asarray(s).view(np.uint16)), i
    # the threshold, not the buffer, must end most periods here
    full = sum(bool(r[i]) for r in rounded for i in range(N))
    assert n_rounded == full and full > N * T // P


# ---------------- pure-write window ----------------

def e4m3_code_values():
    """Every E4M3 bit pattern decoded from its fields: sign, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent 0 is subnormal (m 2^-9); S.1111.111 is
    NaN.  Returns the finite values, one per code."""
    vals = []
    for c in range(256):
        s, E, m = c >> 7, (c >> 3) & 15, c & 7
        if E == 15 and m == 7:
            continue
        v = m * 2.0 ** -9 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7)
        vals.append(-v if s else v)
    return np.array(vals)


def check_e4m3(e4m3, seed=0):
    vals = e4m3_code_values()
    assert vals.max() == 448.0 and np.min(np.abs(vals[vals != 0])) == 2.0 ** -9
    # representable values are fixed points
    assert np.array_equal(e4m3(vals), vals)
    # brute force: the nearest finite value, ties to the even mantissa, over
    # random values and every midpoint between neighbours
    pos = np.unique(np.abs(vals))
    codes = {float(v): i for i, v in enumerate(pos)}    # mantissa parity follows the index
    rng = np.random.default_rng(seed)
    xs = np.concatenate([rng.standard_normal(2000) * 4.0, rng.uniform(-460, 460, 500),
                         rng.standard_normal(500) * 0.01, (pos[1:] + pos[:-1]) / 2,
                         -(pos[1:] + pos[:-1]) / 2])
    for x in xs:
        a = abs(x)
        if a >= 448.0:
            want = 448.0
        else:
            d = np.abs(pos - a)
            best = np.nonzero(d == d.min())[0]
            want = pos[best[0]] if len(best) == 1 else pos[[b for b in best if codes[float(pos[b])] % 2 == 0][0]]
        got = e4m3(np.array([x]))[0]
        assert got == np.copysign(want, x), (x, got, want)
    # saturation, signed zero, NaN
    assert e4m3(np.array([1e6, -500.0]))[0] == 448.0 and e4m3(np.array([-500.0]))[0] == -448.0
    assert np.signbit(e4m3(np.array([-0.0]))[0]) and np.isnan(e4m3(np.array([np.nan]))[0])


def check_pw_limits(pw_run, per_token_rounding, sequential, e4m3, PoolState, quantize, seed=0):
    """A window of one step is per-token rounding of the E4M3-rounded writes;
    a window longer than the stream never merges, so it is the exact
    recurrence from the stored state over those writes."""
    rng = np.random.default_rng(seed)
    N, d_v, d_k = 5, 8, 8
    bits = [4, 8, 4, 8, 4]
    for axis in ("col", "row"):
        codes, scales = _random_pool_state(rng, N, d_v, d_k, bits, axis, quantize)
        st = PoolState(codes, scales, bits, axis)
        toks = random_tokens(rng, N, 9, d_k, d_v)
        for tk in toks:
            tk["v"] = tk["v"] * 3.0
        rounded = [dict(tk, k=e4m3(tk["k"]), v=e4m3(tk["v"])) for tk in toks]
        o_w, fin_w, window, _ = pw_run(st, toks, 1)
        o_p, fin_p = per_token_rounding(st, rounded)
        assert not window
        for x, y in zip(o_w, o_p):
            assert np.array_equal(x, y)
        assert all(np.array_equal(a, b) for a, b in zip(fin_w.codes, fin_p.codes))
        o_w, fin_w, window, _ = pw_run(st, toks, len(toks) + 1)
        _, o_s = sequential(st.dequantized(), rounded)
        assert len(window) == len(toks)
        for x, y in zip(o_w, o_s):
            assert np.allclose(x, y, rtol=1e-12, atol=1e-12)
        assert all(np.array_equal(a, b) for a, b in zip(fin_w.codes, st.codes))


def check_pw_replay(pw_run, chunk_form, e4m3, PoolState, quantize, dequantize, seed=0):
    """A window of S = 3 replayed in chunk form: the output of every token is
    the chunk-form readout of the history through the window's pairs, and
    the history after a merge is the encoding of one step of its oldest pair."""
    rng = np.random.default_rng(seed)
    N, d_v, d_k, S, T = 4, 8, 8, 3, 10
    bits = [4, 8, 4, 4]
    axis = "col"
    codes, scales = _random_pool_state(rng, N, d_v, d_k, bits, axis, quantize)
    st = PoolState(codes, scales, bits, axis)
    toks = random_tokens(rng, N, T, d_k, d_v)
    o_w, fin, window, _ = pw_run(st, toks, S)
    H = st.dequantized()
    hc, hs = list(codes), list(scales)
    win = []
    for t, tk in enumerate(toks):
        win.append(dict(tk, k=e4m3(tk["k"]), v=e4m3(tk["v"])))
        K = np.stack([w["k"] for w in win], 1)
        V = np.stack([w["v"] for w in win], 1)
        A = np.stack([w["alpha"] for w in win], 1)
        B = np.stack([w["beta"] for w in win], 1)
        _, _, o = chunk_form(H, K, V, A, B, tk["q"])
        assert np.allclose(o_w[t], o, rtol=1e-10, atol=1e-12), t
        if len(win) == S:
            old = win.pop(0)
            Sh, _, _ = chunk_form(H, old["k"][:, None], old["v"][:, None], old["alpha"][:, None],
                                  old["beta"][:, None])
            for i in range(N):
                c, s, _ = quantize(Sh[i:i + 1].astype(np.float32), bits[i], axis)
                hc[i], hs[i] = c[0], s[0]
            H = np.stack([dequantize(c, s, axis) for c, s in zip(hc, hs)]).astype(np.float64)
    assert len(window) == S - 1
    assert all(np.array_equal(a, b) for a, b in zip(fin.codes, hc))
