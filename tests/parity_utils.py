"""Helpers for the GPU parity tests: write oracle states into a pool's
records (the documented layout of include/pace.h), read records back, and
judge outputs and commits against the oracle.

The oracle is the reference: a GPU period always starts from a state the
oracle produced (written into the pool), never the other way round.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np
import torch

import oracle as orc

O_TOL = 2e-3                 # max relative error of o_t (teacher-forced periods)
TIE_WINDOW = 2.0 ** -12      # |x/sf - (k + 1/2)| at which a +-1 code flip is a tie
CODE_DIFF_FRACTION = 1e-3    # at most 0.1% of codes may differ after a commit


def write_head(pool, b: int, h: int, codes: np.ndarray, scales: np.ndarray) -> None:
    """Store oracle codes [d_v, d_k] and fp16 scales into head (b, h)'s record."""
    bits = pool.head_bits[h]
    packed = orc.pack_codes(codes, bits).reshape(-1)
    sc = np.asarray(scales, dtype=np.float16).view(np.uint8).reshape(-1)
    rec = pool.record(b, h)
    img = np.zeros(rec.numel(), dtype=np.uint8)
    img[:packed.size] = packed
    img[packed.size:packed.size + sc.size] = sc
    rec.copy_(torch.from_numpy(img).to(rec.device))


def read_head(pool, b: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    bits = pool.head_bits[h]
    rec = pool.record(b, h).cpu().numpy()
    ncode = pool.d_v * pool.d_k * bits // 8
    codes = orc.unpack_codes(rec[:ncode].reshape(pool.d_v, pool.d_k * bits // 8), bits)
    ng = pool.d_k if pool.axis == 0 else pool.d_v
    scales = rec[ncode:ncode + 2 * ng].copy().view(np.float16)
    return codes, scales


def load_state(pool, heads: Sequence[Tuple[int, int]], state: "orc.PoolState") -> None:
    for idx, (b, h) in enumerate(heads):
        write_head(pool, b, h, state.codes[idx], state.scales[idx])
    fill = pool.fill()
    for b, h in heads:
        fill[b, h] = 0


def read_state(pool, heads: Sequence[Tuple[int, int]]) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    cs, ss = [], []
    for b, h in heads:
        c, s = read_head(pool, b, h)
        cs.append(c)
        ss.append(s)
    return cs, ss


def judge_commit(gpu_codes: Sequence[np.ndarray], gpu_scales: Sequence[np.ndarray],
                 ref: "orc.PoolState", S_end: np.ndarray, axis: str) -> Dict[str, float]:
    """Scales equal or one fp16 ulp apart (an amax at a rounding boundary,
    whole group excused); codes equal, or +-1 where the oracle's fp64 x/sf lies
    within TIE_WINDOW of a half-integer; at most 0.1% of codes differ."""
    red = -2 if axis == "col" else -1
    n_diff, n_total, n_scale_ulp = 0, 0, 0
    bad = []
    for i in range(len(ref.codes)):
        sg = gpu_scales[i].view(np.uint16).astype(np.int64)
        so = ref.scales[i].view(np.uint16).astype(np.int64)
        sd = np.abs(sg - so)
        both_nan = np.isnan(gpu_scales[i]) & np.isnan(ref.scales[i])
        sd = np.where(both_nan, 0, sd)
        if np.any(sd > 1):
            bad.append(("scale", i, int(np.max(sd))))
        n_scale_ulp += int(np.sum(sd == 1))
        group_excused = np.expand_dims(sd == 1, red)
        diff = gpu_codes[i].astype(np.int64) - ref.codes[i].astype(np.int64)
        ratios = orc.commit_ratios(S_end[i], ref.scales[i], axis)
        dist = np.abs(np.abs(ratios) % 1.0 - 0.5)
        tie = (np.abs(diff) == 1) & (dist <= TIE_WINDOW)
        wrong = (diff != 0) & ~tie & ~np.broadcast_to(group_excused, diff.shape)
        if np.any(wrong):
            ii = np.argwhere(wrong)[0]
            bad.append(("code", i, tuple(int(x) for x in ii), int(diff[tuple(ii)]),
                        float(ratios[tuple(ii)])))
        n_diff += int(np.sum(diff != 0))
        n_total += diff.size
    frac = n_diff / max(n_total, 1)
    assert not bad, bad[:5]
    assert frac <= CODE_DIFF_FRACTION, (n_diff, n_total)
    return {"codes_differing": n_diff, "codes_total": n_total, "fraction": frac,
            "scales_one_ulp": n_scale_ulp}


def host_tokens(inputs: Dict[str, torch.Tensor], heads: Sequence[Tuple[int, int]]) -> Dict[str, np.ndarray]:
    bs = torch.tensor([b for b, _ in heads])
    hs = torch.tensor([h for _, h in heads])
    out = {}
    for name, x in inputs.items():
        out[name] = x[bs.to(x.device), hs.to(x.device)].to("cpu", torch.float64).numpy()
    return out


def oracle_warm_state(w, heads: Sequence[Tuple[int, int]], bits: Sequence[int], seed: int = 0,
                      tokens: int = None, device="cpu") -> "orc.PoolState":
    """The workload's unquantised fp32 warm-up prefill from a zero state,
    computed by the oracle (fp64, rounded to fp32) for the listed heads, then
    encoded by the oracle."""
    import pace_synth
    T = w.warmup if tokens is None else tokens
    S = np.zeros((len(heads), w.d_v, w.d_k))
    for t in range(T):
        inp = pace_synth.token_inputs(w, t, seed=seed, device=device, phase="warmup")
        tok = host_tokens(inp, heads)
        S, _ = orc.gdn_step_delta(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
    st, flags = orc.PoolState.from_fp32(S.astype(np.float32), bits, w.axis)
    assert flags == 0
    return st
