"""Choosing the 8-bit heads from the gates (long-memory heads keep 8 bits).

CPU: the oracle's rate is pinned to closed forms and its selection to hand
cases; the library's host selection must equal the oracle's exactly.
GPU: the fp64 decay-rate kernel against the oracle, and on the mixed 4/8
workload the selection must recover exactly the heads the generator gave the
long-memory gate.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth


def test_oracle_rates_closed_forms():
    alpha = np.array([[0.5, 1.0, math.exp(-0.25), 0.9]] * 7)
    r = orc.decay_rates(alpha)
    assert r[0] == pytest.approx(math.log(2.0), rel=1e-15)
    assert r[1] == 0.0
    assert r[2] == pytest.approx(0.25, rel=1e-15)
    # mean over rows: two gate values alternate
    alt = np.array([[0.5], [0.25]] * 3)
    assert orc.decay_rates(alt)[0] == pytest.approx(1.5 * math.log(2.0), rel=1e-15)


def test_oracle_selection_hand_cases():
    assert orc.select_head_bits([0.3, 0.1, 0.2], 1) == [4, 8, 4]
    assert orc.select_head_bits([0.1, 0.1, 0.1], 2) == [8, 8, 4]          # ties: lower index
    assert orc.select_head_bits([float("nan"), 0.5, 0.7], 2) == [4, 8, 8]  # NaN last
    assert orc.select_head_bits([0.5, 0.2], 0) == [4, 4]
    assert orc.select_head_bits([0.5, 0.2], 2) == [8, 8]


@pytest.mark.parametrize("seed", range(6))
def test_library_selection_matches_oracle(seed):
    import bit_recurrent_state_pace_b200 as pace
    rng = np.random.RandomState(seed)
    H = int(rng.randint(1, 257))
    rates = rng.rand(H)
    rates[rng.rand(H) < 0.2] = 0.5          # ties
    if H > 3:
        rates[rng.randint(H)] = float("nan")
    n8 = int(rng.randint(0, H + 1))
    assert pace.pace_select_head_bits(rates, n8) == orc.select_head_bits(rates, n8)


def test_library_selection_rejects_bad_arguments():
    import bit_recurrent_state_pace_b200 as pace
    with pytest.raises(pace.PaceError):
        pace.pace_select_head_bits([0.1, 0.2], 3)
    with pytest.raises(pace.PaceError):
        pace.pace_select_head_bits([0.1] * 257, 1)


@pytest.mark.gpu
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decay_rates_kernel_and_long_memory_recovery(io):
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("mixed_4_8", B=64, io_dtype=io)
    seed = 3   # the generator's long-memory heads depend on the seed
    gates = torch.stack([pace_synth.token_inputs(w, t, seed=seed, device="cuda", phase="warmup")["alpha"]
                         for t in range(48)])                     # [T][B][H]
    rates = pace.pace_decay_rates(gates.contiguous(), w.H, pace.PACE_IO_BF16 if io == "bf16"
                                  else pace.PACE_IO_F32)
    ref = orc.decay_rates(gates.float().cpu().numpy())
    np.testing.assert_allclose(rates.cpu().numpy(), ref, rtol=1e-12, atol=0.0)
    n8 = len(pace_synth.int8_heads(w, seed))
    bits = pace.pace_select_head_bits(rates.cpu().tolist(), n8)
    assert bits == orc.select_head_bits(ref, n8)
    chosen = sorted(h for h in range(w.H) if bits[h] == 8)
    assert chosen == sorted(pace_synth.long_memory_heads(w, seed))
