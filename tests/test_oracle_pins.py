"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle as orc
from tests import oracle_checks as ck


def test_rounding_primitives():
    ck.check_rounding_primitives()


def test_encoder_golden_worked_example():
    ck.check_encoder_golden(orc.quantize, orc.pack_codes)


def test_encoder_bruteforce_exact_rationals():
    ck.check_encoder_bruteforce(orc.quantize)


def test_encoder_invariants():
    ck.check_encoder_invariants(orc.quantize, orc.dequantize)


def test_encoder_exhaustive_fp16_scales():
    ck.check_encoder_exhaustive_scales(orc.quantize, orc.dequantize)


def test_encoder_special_cases():
    ck.check_encoder_special_cases(orc.quantize, orc.FLAG_NONFINITE, orc.FLAG_SCALE_OVERFLOW)


def test_pack_roundtrip_and_nibble_order():
    ck.check_pack_roundtrip(orc.pack_codes, orc.unpack_codes)


def test_commit_ratios_hand_worked():
    ck.check_commit_ratios(orc.commit_ratios)


def test_gdn_golden_two_tokens():
    ck.check_gdn_golden(orc.gdn_step)


def test_gdn_bruteforce_exact_rationals():
    ck.check_gdn_bruteforce(orc.gdn_step)


def test_gdn_closed_forms():
    ck.check_gdn_closed_forms(orc.gdn_step)


def test_gdn_delta_form_agrees():
    ck.check_step_forms_agree(orc.gdn_step, orc.gdn_step_delta)
    ck.check_gdn_golden(orc.gdn_step_delta)


def test_chunk_form_equals_sequential():
    ck.check_chunk_vs_sequential(orc.chunk_form, orc.gdn_step)


def _state(rng, N, d_v, d_k, bits, axis):
    S = rng.standard_normal((N, d_v, d_k)).astype(np.float32)
    st, flags = orc.PoolState.from_fp32(S, bits, axis)
    assert flags == 0
    return st


@pytest.mark.parametrize("axis", ["col", "row"])
def test_periodic_without_rounding_is_sequential(axis):
    rng = np.random.default_rng(3)
    N, d_v, d_k, T = 3, 10, 8, 13
    S0 = rng.standard_normal((N, d_v, d_k))
    toks = ck.random_tokens(rng, N, T, d_k, d_v)
    _, ref = orc.sequential(S0, toks)
    for P in (1, 4, 5):
        outs, final, commits, flags, n = orc.pace_run(S0, toks, P, quantize_state=False)
        assert not commits
        for a, b in zip(outs, ref):
            assert np.array_equal(a, b)


@pytest.mark.parametrize("axis", ["col", "row"])
def test_period_one_is_per_token_rounding(axis):
    rng = np.random.default_rng(4)
    N, d_v, d_k, T = 3, 8, 8, 9
    st = _state(rng, N, d_v, d_k, [4, 8, 4], axis)
    toks = ck.random_tokens(rng, N, T, d_k, d_v)
    outs, final, commits, flags, n = orc.pace_run(st, toks, 1)
    ref_outs, ref_state = orc.per_token_rounding(st, toks)
    assert len(commits) == T and n == 0
    for a, b in zip(outs, ref_outs):
        assert np.array_equal(a, b)
    for a, b in zip(final.codes, ref_state.codes):
        assert np.array_equal(a, b)


def test_outputs_inside_a_period_follow_the_dequantised_state():
    """Before the first commit, the periodic path is the exact recurrence from
    the dequantised stored state; after a commit it restarts from the newly
    stored state (rounding happens once per period, nowhere else)."""
    rng = np.random.default_rng(5)
    N, d_v, d_k, P = 2, 8, 6, 4
    st = _state(rng, N, d_v, d_k, [4, 8], "col")
    toks = ck.random_tokens(rng, N, 2 * P, d_k, d_v)
    outs, final, commits, flags, n = orc.pace_run(st, toks, P)
    _, ref1 = orc.sequential(st.dequantized(), toks[:P])
    for a, b in zip(outs[:P], ref1):
        assert np.array_equal(a, b)
    t0, st1 = commits[0]
    assert t0 == P - 1
    _, ref2 = orc.sequential(st1.dequantized(), toks[P:])
    for a, b in zip(outs[P:], ref2):
        assert np.array_equal(a, b)
    # the committed state is the encoding of the fp32-rounded period-end state
    S_end, _ = orc.sequential(st.dequantized(), toks[:P])
    for i, bits in enumerate([4, 8]):
        c, s, _ = orc.quantize(S_end[i:i + 1].astype(np.float32), bits, "col")
        assert np.array_equal(c[0], st1.codes[i])


def test_period_reference_matches_run():
    rng = np.random.default_rng(6)
    st = _state(rng, 2, 8, 8, [4, 4], "row")
    toks = ck.random_tokens(rng, 2, 4, 8, 8)
    outs, S_end, committed, flags = orc.period_reference(st, toks, 4)
    outs2, final, commits, _, _ = orc.pace_run(st, toks, 4)
    for a, b in zip(outs, outs2):
        assert np.array_equal(a, b)
    assert np.array_equal(committed.codes[0], final.codes[0])


def test_relative_error_metric():
    ref = np.array([[1.0, -2.0, 0.5]])
    assert orc.relative_error(ref, ref)[0] == 0
    assert orc.relative_error(ref + np.array([[0, 0.004, 0]]), ref)[0] == pytest.approx(0.002)
    assert orc.relative_error(np.zeros((1, 3)), np.zeros((1, 3)))[0] == 0


def test_update_norm_closed_forms():
    ck.check_update_norm_closed_forms(orc.update_norm2, orc.gdn_step)


def test_adaptive_period_limits():
    ck.check_adaptive_limits(orc.pace_run_adaptive, orc.pace_run, orc.per_token_rounding,
                             orc.PoolState, orc.quantize)


def test_adaptive_period_replayed_per_head_in_chunk_form():
    ck.check_adaptive_driver_per_head(orc.pace_run_adaptive, orc.chunk_form, orc.PoolState,
                                      orc.quantize, orc.dequantize)


def test_e4m3_against_its_code_table():
    ck.check_e4m3(orc.e4m3)


def test_pure_write_window_limits():
    ck.check_pw_limits(orc.pw_run, orc.per_token_rounding, orc.sequential, orc.e4m3, orc.PoolState,
                       orc.quantize)


def test_pure_write_window_replayed_in_chunk_form():
    ck.check_pw_replay(orc.pw_run, orc.chunk_form, orc.e4m3, orc.PoolState, orc.quantize,
                       orc.dequantize)
