"""fp64 CPU oracle for PACE periodic low-bit recurrent-state decode.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package.  The product (``bit_recurrent_state_pace_b200``)
never does, and this package imports nothing from it: the two share no code.

What is computed, and where it comes from
-----------------------------------------
Pages cited (by title and section):

* [P1] "PACE：四比特循环状态量化新方法，让线性注意力模型更省内存"
* [P2] "PACE: A New 4-Bit Recurrent State Quantization Method That Makes Linear
  Attention Models More Memory-Efficient"
* [P3] "低比特量化新突破：GGA+PW让线性注意力长文本生成更准更短"
* [P4] "PACE: four-bit recurrent state by rounding less often"

1. The recurrence.  [P3], section "为什么低比特状态量化会“越写越错”" (the
   paragraph on linear attention and GDN) describes Gated DeltaNet as a gate
   that sets how fast history is forgotten plus a delta rule that makes each
   write an online-learning step.  The pages print no equation; the reading
   taken is the standard gated delta rule with state ``S`` in R^{d_v x d_k}:
   ``S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T`` and
   ``o_t = S_t q_t`` (no extra output scale).  ``gdn_step`` writes this out
   literally; ``gdn_step_delta`` writes the same rule as the online-learning
   correction ``S <- a S + b (v - a S k) k^T`` that [P3] describes.
2. Periodic rounding.  [P2] "Periodic Rounding: Reducing Error Accumulation",
   [P4] TL;DR (1) and the flowchart under "Fewer roundings, less compounded
   error": the state stays in high precision for a period of P tokens that
   sit in a small buffer, and is rounded once per period.  ``pace_run``
   applies P exact steps from the dequantised state, then quantises.
3. Chunked update.  [P2] (the chunked-kernel paragraph of "Periodic
   Rounding") and the flowchart's "State update, chunked, high precision":
   ``chunk_form`` is the UT/WY chunk form of P steps (decays, Gram matrix,
   forward substitution), checked against P sequential steps.
4. Channel-aligned scales.  [P2] "Channel-Aligned Encoding: Exploiting State
   Column Structure", [P4] TL;DR (2): one scale per column.  Reading: a column
   is a key channel j of S (all d_v entries S[:, j]); a row-axis variant (one
   scale per value channel i) is also provided.  ``quantize`` is symmetric
   absmax with an FP16 scale, codes rounded half-to-even and clamped to
   [-7, 7] (INT4) or [-127, 127] (INT8), emulating fp32 arithmetic exactly.
5. Mixed heads.  [P2] "Additionally, PACE uses 8-bit precision ..." paragraph,
   [P4] TL;DR (3) and the flowchart's "long-memory heads -> 8-bit heads":
   per-head bit widths, handled by calling ``quantize`` with bits 4 or 8.
   ``decay_rates`` / ``select_head_bits`` choose the 8-bit heads from the
   gates (mean -ln alpha per head, the slowest-decaying heads first).
6. Adaptive period.  [P4] "Research angle": round when the accumulated
   update norm crosses a threshold rather than every k tokens.  Reading: the
   accumulated update after n buffered tokens is what the writes added to
   the decayed stored state, ``Delta_n = S_n - gamma_n S~0`` (a pure decay is
   a rescaling that needs no re-encoding), in the Frobenius norm; a head is
   rounded after token n when ``||Delta_n||_F >= tau`` and in any case when
   its buffer of P tokens is full.  ``update_norm2`` writes the definition
   out; ``pace_run_adaptive`` is the per-head driver.
7. Pure-write window.  [P3], section "PW：让近期写入走“纯净通道”": the
   most recent writes are kept apart from the low-bit history as FP8 vector
   pairs (k, v) that take full part in the state transition, and a pair is
   merged into the low-bit history only when it leaves the window of S
   steps.  ``e4m3`` is the FP8 format (E4M3: 4 exponent bits, bias 7, 3
   mantissa bits, largest finite 448), rounding to nearest with ties to even
   and saturating at +-448; ``pw_run`` is the windowed driver.

Everything here is fp64 except the quantiser, which takes the fp32 state and
reproduces the fp32/fp16 operations of the encoding one by one with numpy's
IEEE float32/float16 types.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

QMAX = {4: 7, 8: 127}

# Flags the quantiser raises (same meaning as the library's status bits, but
# defined independently here).
FLAG_NONFINITE = 1
FLAG_SCALE_OVERFLOW = 2

FP16_MIN_SUBNORMAL = np.float16(2.0 ** -24)
FP16_MAX = np.float16(65504.0)


# --------------------------------------------------------------------------
# Quantiser (channel-aligned absmax encoding), [P2] "Channel-Aligned
# Encoding", [P4] TL;DR (2) and flowchart "4-bit encode, per-column scales".
# --------------------------------------------------------------------------

def _group_axis(axis: str) -> int:
    if axis == "col":
        return -2      # a group is a column S[:, j]; reduce over rows i
    if axis == "row":
        return -1      # a group is a row S[i, :]; reduce over columns j
    raise ValueError(axis)


def quantize(S, bits: int, axis: str = "col") -> Tuple[np.ndarray, np.ndarray, int]:
    """Encode fp32 matrices ``S[..., d_v, d_k]`` with one FP16 scale per group.

    Steps, per group g with ``qmax`` = 7 (INT4) or 127 (INT8):

    Q1  amax = max |x| over the group (exact in fp32);
    Q2  s32 = amax / qmax, one fp32 division rounded to nearest;
    Q3  s16 = fp16(s32) rounded to nearest even; a nonzero amax whose scale
        rounds to zero gets the smallest fp16 subnormal 2^-24; a scale that
        overflows fp16 is clamped to 65504 and flagged;
    Q4  sf = float(s16); codes c = clamp(rint_half_even(x / sf), -qmax, qmax)
        with fp32 division; all codes 0 when sf == 0;
    --  a group holding a non-finite entry gets scale NaN, codes 0, and a flag.

    Returns ``codes`` (int8, same shape as S), ``scales`` (float16,
    ``[..., d_k]`` for col or ``[..., d_v]`` for row) and the flag bits.
    """
    S = np.asarray(S, dtype=np.float32)
    qmax = QMAX[bits]
    red = _group_axis(axis)
    finite = np.isfinite(S).all(axis=red, keepdims=True)
    absS = np.where(np.isfinite(S), np.abs(S), np.float32(0))
    amax = absS.max(axis=red, keepdims=True).astype(np.float32)          # Q1
    s32 = (amax / np.float32(qmax)).astype(np.float32)                    # Q2
    with np.errstate(over="ignore"):
        s16 = s32.astype(np.float16)                                      # Q3
    s16 = np.where((amax > 0) & (s16 == 0), FP16_MIN_SUBNORMAL, s16)
    overflow = np.isinf(s16) & finite
    s16 = np.where(np.isinf(s16), FP16_MAX, s16)
    sf = s16.astype(np.float32)                                           # Q4
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (S / np.where(sf == 0, np.float32(1), sf)).astype(np.float32)
    codes = np.clip(np.rint(ratio), -qmax, qmax)
    codes = np.where(sf == 0, 0, codes)
    codes = np.where(finite, codes, 0).astype(np.int8)
    s16 = np.where(finite, s16, np.float16(np.nan)).astype(np.float16)
    flags = 0
    if not finite.all():
        flags |= FLAG_NONFINITE
    if overflow.any():
        flags |= FLAG_SCALE_OVERFLOW
    return codes, np.squeeze(s16, axis=red), flags


def dequantize(codes, scales, axis: str = "col") -> np.ndarray:
    """x_hat = float(c) * float(s16): exact in fp32 (<= 7-bit by 11-bit significands)."""
    codes = np.asarray(codes)
    sf = np.asarray(scales, dtype=np.float16).astype(np.float32)
    sf = np.expand_dims(sf, _group_axis(axis))
    return (codes.astype(np.float32) * sf).astype(np.float32)


def pack_codes(codes, bits: int) -> np.ndarray:
    """Byte image of the codes along d_k: INT8 one byte per code (two's
    complement); INT4 two codes per byte, the even index j in the low nibble,
    each nibble the 4-bit two's complement of its code."""
    codes = np.asarray(codes, dtype=np.int8)
    if bits == 8:
        return codes.view(np.uint8).copy()
    lo = codes[..., 0::2].astype(np.int16) & 0xF
    hi = codes[..., 1::2].astype(np.int16) & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_codes(packed, bits: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    if bits == 8:
        return packed.view(np.int8).copy()
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# --------------------------------------------------------------------------
# Gated delta rule, [P3] paragraph on linear attention / GDN.
# --------------------------------------------------------------------------

def gdn_step(S, q, k, v, alpha, beta):
    """One token, written as the definition (batched over leading head axis N).

    S [N, d_v, d_k]; q, k [N, d_k]; v [N, d_v]; alpha, beta [N] (fp64).
    S_t = alpha S_{t-1} (I - beta k k^T) + beta v k^T ;  o_t = S_t q_t.
    """
    S = np.asarray(S, dtype=np.float64)
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    a = np.asarray(alpha, dtype=np.float64)[:, None, None]
    b = np.asarray(beta, dtype=np.float64)[:, None, None]
    d_k = S.shape[-1]
    transition = np.eye(d_k)[None] - b * (k[:, :, None] * k[:, None, :])
    S_new = a * np.matmul(S, transition) + b * (v[:, :, None] * k[:, None, :])
    o = np.matmul(S_new, q[:, :, None])[:, :, 0]
    return S_new, o


def gdn_step_delta(S, q, k, v, alpha, beta):
    """The same token as an online-learning correction of the decayed state:
    S_t = alpha S + beta (v - alpha S k) k^T (the delta rule of [P3])."""
    S = np.asarray(S, dtype=np.float64)
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    a = np.asarray(alpha, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    decayed = a[:, None, None] * S
    err = v - np.matmul(decayed, k[:, :, None])[:, :, 0]
    S_new = decayed + b[:, None, None] * (err[:, :, None] * k[:, None, :])
    o = np.matmul(S_new, q[:, :, None])[:, :, 0]
    return S_new, o


def sequential(S0, tokens: Sequence[Dict[str, np.ndarray]], step=gdn_step):
    """Unquantised trajectory: apply ``step`` token by token in fp64."""
    S = np.asarray(S0, dtype=np.float64)
    outs = []
    for tok in tokens:
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        outs.append(o)
    return S, outs


# --------------------------------------------------------------------------
# Chunk (UT / WY) form of n buffered tokens, [P2] chunked-kernel paragraph of
# "Periodic Rounding"; [P4] flowchart "State update, chunked, high precision".
# --------------------------------------------------------------------------

def chunk_form(S0, K, V, alpha, beta, q=None):
    """n tokens applied to S0 at once.

    S0 [N, d_v, d_k]; K [N, n, d_k]; V [N, n, d_v]; alpha, beta [N, n];
    q [N, d_k] (the query of the last token, optional).

    gamma_t = prod_{r<=t} alpha_r, gamma_{t/s} = prod_{s<r<=t} alpha_r;
    A[t, s] = beta_t gamma_{t/s} k_t.k_s for s < t;
    U = (I + A)^{-1} diag(beta) (V - diag(gamma) X^T) with X = S0 K^T,
    solved by forward substitution (rows u_t);
    S_n = gamma_n S0 + sum_s gamma_{n/s} u_s k_s^T;
    o_n = gamma_n S0 q + sum_s gamma_{n/s} (k_s.q) u_s.
    Returns (S_n, U, o_n or None).
    """
    S0 = np.asarray(S0, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    al = np.asarray(alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    N, n, _ = K.shape
    # decay products gamma_{t/s} (t, s in 0..n; index 0 = before the first token)
    gam = np.ones((N, n + 1, n + 1))
    for t in range(1, n + 1):
        for s in range(0, t):
            gam[:, t, s] = np.prod(al[:, s:t], axis=1)
    gamma = gam[:, 1:, 0]                                   # gamma_t, t = 1..n
    X = np.matmul(S0, np.swapaxes(K, 1, 2))                 # [N, d_v, n]
    gram = np.matmul(K, np.swapaxes(K, 1, 2))               # [N, n, n]
    rhs = be[:, :, None] * (V - gamma[:, :, None] * np.swapaxes(X, 1, 2))
    U = np.zeros_like(rhs)
    for t in range(n):                                      # forward substitution
        acc = rhs[:, t, :].copy()
        for s in range(t):
            a_ts = be[:, t] * gam[:, t + 1, s + 1] * gram[:, t, s]
            acc -= a_ts[:, None] * U[:, s, :]
        U[:, t, :] = acc
    g_last = gam[:, n, 1:]                                  # gamma_{n/s}, s = 1..n
    S_n = gam[:, n, 0][:, None, None] * S0 + np.matmul(
        np.swapaxes(g_last[:, :, None] * U, 1, 2), K)
    o = None
    if q is not None:
        q = np.asarray(q, dtype=np.float64)
        kq = np.matmul(K, q[:, :, None])[:, :, 0]           # k_s . q
        o = gam[:, n, 0][:, None] * np.matmul(S0, q[:, :, None])[:, :, 0] \
            + np.sum((g_last * kq)[:, :, None] * U, axis=1)
    return S_n, U, o


# --------------------------------------------------------------------------
# Periodic driver: buffer P tokens, round once per period ([P2] "Periodic
# Rounding", [P4] TL;DR (1), flowchart "every k tokens").
# --------------------------------------------------------------------------

class PoolState:
    """Stored state of a set of heads: codes + FP16 scales, per-head bits."""

    def __init__(self, codes: List[np.ndarray], scales: List[np.ndarray],
                 bits: Sequence[int], axis: str):
        self.codes = [np.asarray(c, dtype=np.int8) for c in codes]
        self.scales = [np.asarray(s, dtype=np.float16) for s in scales]
        self.bits = list(bits)
        self.axis = axis

    @classmethod
    def from_fp32(cls, S32, bits: Sequence[int], axis: str) -> Tuple["PoolState", int]:
        S32 = np.asarray(S32, dtype=np.float32)
        codes, scales, flags = [], [], 0
        for i, b in enumerate(bits):
            c, s, f = quantize(S32[i:i + 1], b, axis)
            codes.append(c[0])
            scales.append(s[0])
            flags |= f
        return cls(codes, scales, bits, axis), flags

    def dequantized(self) -> np.ndarray:
        return np.stack([dequantize(c, s, self.axis)
                         for c, s in zip(self.codes, self.scales)]).astype(np.float64)


def commit(S_fp64, bits: Sequence[int], axis: str) -> Tuple[PoolState, int]:
    """End of period: round the fp64 state to fp32 (the encoder's input type),
    then encode each head with its own bit width."""
    return PoolState.from_fp32(np.asarray(S_fp64).astype(np.float32), bits, axis)


def pace_run(state: PoolState, tokens: Sequence[Dict[str, np.ndarray]], P: int,
             fill: int = 0, quantize_state: bool = True, step=gdn_step):
    """Decode ``tokens`` with periodic rounding, starting at a period boundary.

    The working state starts from the dequantised stored state and is
    advanced exactly (fp64) through every token of the period; after the
    P-th token the state is rounded (``commit``) and the next period restarts
    from the newly stored state.  With ``quantize_state=False``, ``state`` is
    an fp64 array and period ends keep it unrounded (the periodic path must
    then equal ``sequential``).

    Returns (outputs per token [N, d_v], final PoolState or fp64 state,
    list of (token index, post-commit PoolState) for every commit, flags,
    tokens buffered in the unfinished last period).
    """
    assert fill == 0, "the oracle starts at a period boundary"
    if quantize_state:
        S = state.dequantized()
    else:
        S = np.asarray(state, dtype=np.float64)
    outs, commits, flags = [], [], 0
    n = 0
    for t, tok in enumerate(tokens):
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        outs.append(o)
        n += 1
        if n == P:
            n = 0
            if quantize_state:
                st, f = commit(S, state.bits, state.axis)
                flags |= f
                commits.append((t, st))
                state = st
                S = st.dequantized()
    final = state if quantize_state else S
    return outs, final, commits, flags, n


def per_token_rounding(state: PoolState, tokens: Sequence[Dict[str, np.ndarray]],
                       step=gdn_step):
    """Round after every generated token (what prior quantisers do, [P2] "Why
    Do We Need Low-Precision Recurrent States?"): written on its own so that
    ``pace_run`` with P = 1 can be checked against it."""
    outs = []
    for tok in tokens:
        S = np.stack([dequantize(c, s, state.axis)
                      for c, s in zip(state.codes, state.scales)]).astype(np.float64)
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        outs.append(o)
        S32 = S.astype(np.float32)
        codes, scales = [], []
        for i, b in enumerate(state.bits):
            c, s, _ = quantize(S32[i:i + 1], b, state.axis)
            codes.append(c[0])
            scales.append(s[0])
        state = PoolState(codes, scales, state.bits, state.axis)
    return outs, state


def commit_ratios(S_fp64, scales, axis: str) -> np.ndarray:
    """fp64 x / sf of every entry of the period-end state against the oracle's
    own scales: how far each entry sits from a rounding tie (test checker)."""
    S32 = np.asarray(S_fp64).astype(np.float32).astype(np.float64)
    sf = np.asarray(scales, dtype=np.float16).astype(np.float64)
    sf = np.expand_dims(sf, _group_axis(axis))
    with np.errstate(divide="ignore", invalid="ignore"):
        return S32 / sf


def period_reference(state: PoolState, tokens: Sequence[Dict[str, np.ndarray]], P: int):
    """One period from a stored state: outputs of each token and, if the
    period completes, the fp64 period-end state and the committed state."""
    S = state.dequantized()
    outs = []
    for tok in tokens:
        S, o = gdn_step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        outs.append(o)
    committed, flags = (None, 0)
    if len(tokens) == P:
        committed, flags = commit(S, state.bits, state.axis)
    return outs, S, committed, flags


def relative_error(o_test, o_ref) -> np.ndarray:
    """Per head: ||o_test - o_ref||_inf / max(||o_ref||_inf, 1e-6)."""
    o_test = np.asarray(o_test, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    num = np.max(np.abs(o_test - o_ref), axis=-1)
    den = np.maximum(np.max(np.abs(o_ref), axis=-1), 1e-6)
    return num / den


# --------------------------------------------------------------------------
# Which heads keep 8 bits.  [P2] (paragraph on 8-bit precision for selected
# heads) and [P4] TL;DR (3): heads whose errors persist -- long-memory heads
# -- are stored at 8 bits.  Reading: a head's memory is set by its gate, a
# write decaying by alpha per token, so heads are ranked by their mean decay
# rate -ln(alpha) over a calibration stream (smaller = longer memory).
# --------------------------------------------------------------------------

def decay_rates(alpha) -> np.ndarray:
    """Mean of -ln(alpha) over the leading axes, per head (last axis), fp64."""
    a = np.asarray(alpha, dtype=np.float64)
    a = a.reshape(-1, a.shape[-1])
    return np.mean(-np.log(a), axis=0)


def select_head_bits(rates, num_int8: int) -> List[int]:
    """8 bits for the num_int8 heads with the smallest rate (NaN last, ties to
    the lower head index), 4 bits for the rest."""
    r = [float(x) for x in rates]
    order = sorted(range(len(r)), key=lambda h: (np.isnan(r[h]), 0.0 if np.isnan(r[h]) else r[h], h))
    bits = [4] * len(r)
    for h in order[:num_int8]:
        bits[h] = 8
    return bits


# --------------------------------------------------------------------------
# Adaptive period, [P4] "Research angle": a head is rounded when its
# accumulated update crosses a threshold instead of after a fixed number of
# tokens; the buffer's capacity P still bounds the period.
# --------------------------------------------------------------------------

def update_norm2(S_n, S0, gamma_n) -> np.ndarray:
    """||S_n - gamma_n S0||_F^2 per head (fp64): the squared Frobenius norm of
    what the writes since the last rounding added to the decayed state.
    S_n, S0 [N, d_v, d_k]; gamma_n [N] (product of the period's alphas)."""
    S_n = np.asarray(S_n, dtype=np.float64)
    S0 = np.asarray(S0, dtype=np.float64)
    g = np.asarray(gamma_n, dtype=np.float64)[:, None, None]
    delta = S_n - g * S0
    return np.sum(delta * delta, axis=(1, 2))


def pace_run_adaptive(state: PoolState, tokens: Sequence[Dict[str, np.ndarray]], P: int,
                      tau: float, step=gdn_step):
    """Decode ``tokens`` with a per-head adaptive period, every head starting
    at a period boundary.

    After each token every head advances its fp64 working state exactly from
    its dequantised stored state; head h is rounded (fp32, then its own bit
    width) when it holds P tokens or when update_norm2 >= tau^2, and restarts
    from its newly stored state.  tau = inf gives the fixed period P; tau = 0
    rounds after every token.

    Returns (outputs per token [N, d_v], final PoolState, rounded [T][N] bool,
    norm2 [T][N] (before any rounding of that token), flags).
    """
    S0 = state.dequantized()
    S = S0.copy()
    N = S.shape[0]
    codes = list(state.codes)
    scales = list(state.scales)
    gamma = np.ones(N)
    n = np.zeros(N, dtype=np.int64)
    tau2 = float(tau) * float(tau)
    outs, rounded, norms, flags = [], [], [], 0
    for tok in tokens:
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        outs.append(o)
        gamma = gamma * np.asarray(tok["alpha"], dtype=np.float64)
        n += 1
        norm2 = update_norm2(S, S0, gamma)
        due = (n == P) | (norm2 >= tau2)
        for i in np.nonzero(due)[0]:
            c, sc, f = quantize(S[i:i + 1].astype(np.float32), state.bits[i], state.axis)
            flags |= f
            codes[i], scales[i] = c[0], sc[0]
            S0[i] = dequantize(c[0], sc[0], state.axis)
            S[i] = S0[i]
            gamma[i] = 1.0
            n[i] = 0
        rounded.append(due)
        norms.append(norm2)
    final = PoolState(codes, scales, state.bits, state.axis)
    return outs, final, rounded, norms, flags


# --------------------------------------------------------------------------
# Pure-write window, [P3] section "PW：让近期写入走“纯净通道”": the last S
# writes stay outside the low-bit history as FP8 (k, v) pairs that take full
# part in the state transition; the oldest pair is merged into the history
# (which is then rounded) when it leaves the window.
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3(x) -> np.ndarray:
    """Round to FP8 E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits,
    no infinities; subnormal quantum 2^-9): the nearest representable value,
    ties to the even mantissa, saturating at +-448; NaN stays NaN; the sign of
    zero is kept.  Returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, E = np.frexp(a)                      # a = m 2^E, m in [0.5, 1)
    e = np.maximum(E - 1, -6)               # binade exponent, normals from 2^-6
    q = np.ldexp(1.0, e - 3)                # quantum: 3 mantissa bits
    with np.errstate(invalid="ignore"):
        r = np.round(a / q) * q             # a / q is exact; round() ties to even
    r = np.minimum(r, E4M3_MAX)
    r = np.where(np.isnan(x), np.nan, r)
    return np.copysign(r, x)


def pw_run(state: PoolState, tokens: Sequence[Dict[str, np.ndarray]], S: int, step=gdn_step):
    """Decode ``tokens`` with a pure-write window of S steps, every head in step.

    Each token's k and v are rounded to E4M3 and join the window; the output
    is S_t q_t with S_t the dequantised history advanced exactly (fp64)
    through every pair of the window.  When the window then holds S pairs,
    its oldest pair is applied to the history alone, the history is rounded
    (fp32, then each head's bit width) and the pair leaves the window.

    Returns (outputs per token [N, d_v], final history PoolState, the tokens
    still in the window, flags).
    """
    window: List[Dict[str, np.ndarray]] = []
    outs, flags = [], 0
    for tok in tokens:
        window.append(dict(tok, k=e4m3(tok["k"]), v=e4m3(tok["v"])))
        S_t = state.dequantized()
        for w in window:
            S_t, o = step(S_t, tok["q"], w["k"], w["v"], w["alpha"], w["beta"])
        outs.append(o)
        if len(window) == S:
            old = window.pop(0)
            S_h, _ = step(state.dequantized(), tok["q"], old["k"], old["v"], old["alpha"], old["beta"])
            state, f = commit(S_h, state.bits, state.axis)
            flags |= f
    return outs, state, window, flags
