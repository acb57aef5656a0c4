"""pace_quantize / pace_dequantize through the C ABI against the oracle:
codes, scales and flags bit-exact on identical fp32 input."""
import numpy as np
import pytest
import torch

import oracle as orc
import pace_synth

pytestmark = pytest.mark.gpu


def _pace():
    import bit_recurrent_state_pace_b200 as pace
    return pace


def _special_mats(d_v, d_k, qmax, rng):
    """Matrices with the encoder's corner cases in some of their groups."""
    mats = []
    z = np.zeros((d_v, d_k), np.float32)
    mats.append(z)                                        # all-zero groups
    t = rng.standard_normal((d_v, d_k)).astype(np.float32)
    t[:, 0] *= 1e-12                                       # tiny group (subnormal scale floor)
    t[0, :] *= 1e-12
    t[:, 1 % d_k] = 0
    mats.append(t)
    hgs = rng.standard_normal((d_v, d_k)).astype(np.float32)
    hgs[:, -1] *= 1e36                                     # scale overflow -> 65504
    hgs[-1, :] *= 1e36
    mats.append(hgs)
    nf = rng.standard_normal((d_v, d_k)).astype(np.float32)
    nf[0, 0] = np.nan                                      # non-finite groups
    nf[-1, -1] = np.inf
    mats.append(nf)
    ties = np.zeros((d_v, d_k), np.float32)               # exact half-integer ratios
    s = np.float32(np.float16(0.013))
    for j in range(d_k):
        ties[0, j] = np.float32(qmax) * s
        for i in range(1, d_v):
            ties[i, j] = np.float32(((i * 7 + j) % (2 * qmax)) - qmax + 0.5) * s
    for i in range(d_v):
        ties[i, 0] = np.float32(qmax) * s
    mats.append(ties)
    return mats


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("axis", ["col", "row"])
@pytest.mark.parametrize("shape", [(128, 128), (32, 32), (18, 30), (64, 2), (3, 128)])
def test_quantize_bit_exact(bits, axis, shape):
    pace = _pace()
    d_v, d_k = shape
    qmax = orc.QMAX[bits]
    rng = np.random.default_rng(bits * 1000 + d_v * 7 + d_k + (axis == "row"))
    S = pace_synth.random_state(29, d_v, d_k, seed=bits * 7 + d_k,
                                column_outliers=[d_k // 3], row_outliers=[d_v // 2]).numpy()
    S[3] *= 1e-3
    S[4] *= 300.0
    S = np.concatenate([S, np.stack(_special_mats(d_v, d_k, qmax, rng))], axis=0)
    n = S.shape[0]
    ng = d_k if axis == "col" else d_v
    ax = pace.PACE_SCALE_COL if axis == "col" else pace.PACE_SCALE_ROW
    Sd = torch.from_numpy(S).cuda()
    codes = torch.empty(n, d_v * d_k * bits // 8, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, ng, dtype=torch.int16, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pace.pace_quantize(Sd, n, d_k, d_v, bits, ax, codes, scales, flags)
    torch.cuda.synchronize()
    c_ref, s_ref, f_ref = orc.quantize(S, bits, axis)
    packed = orc.pack_codes(c_ref, bits).reshape(n, -1)
    got_codes = codes.cpu().numpy()
    assert np.array_equal(got_codes, packed), np.argwhere(got_codes != packed)[:5]
    got_s = scales.cpu().numpy().view(np.uint16)
    ref_s = s_ref.view(np.uint16)
    assert np.array_equal(got_s, ref_s), np.argwhere(got_s != ref_s)[:5]
    assert int(flags.item()) == f_ref

    # dequantize of the oracle's codes is the oracle's dequantisation, bit for bit
    out = torch.empty(n, d_v, d_k, dtype=torch.float32, device="cuda")
    pace.pace_dequantize(torch.from_numpy(packed.copy()).cuda(),
                         torch.from_numpy(s_ref.view(np.int16).copy()).cuda(), n, d_k, d_v, bits, ax, out)
    torch.cuda.synchronize()
    ref = orc.dequantize(c_ref, s_ref, axis)
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got, ref)


def test_quantize_rejects_bad_arguments():
    pace = _pace()
    S = torch.zeros(1, 4, 4, device="cuda")
    codes = torch.empty(16, dtype=torch.uint8, device="cuda")
    scales = torch.empty(4, dtype=torch.int16, device="cuda")
    for args in [(S, 1, 4, 4, 5, 0), (S, 1, 3, 4, 4, 0), (S, 1, 4, 4, 4, 2), (S, -1, 4, 4, 4, 0),
                 (S, 1, 512, 4, 4, 0)]:
        with pytest.raises(pace.PaceError):
            pace.pace_quantize(*args, codes, scales)
    pace.pace_quantize(S, 0, 4, 4, 4, 0, codes, scales)   # empty input is a no-op
