"""The C-ABI library loads and exports every call include/pace.h declares;
host-only logic (descriptor validation, pool byte accounting) on the CPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:[A-Za-z_][\w ]*\*?\s+)\*?(pace_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pace_init_pool", "pace_decode_step", "pace_commit_period", "pace_quantize",
                     "pace_dequantize", "pace_pool_bytes", "pace_pool_status"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import bit_recurrent_state_pace_b200 as pace
    lib = ctypes.CDLL(pace.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_pool_byte_accounting():
    import bit_recurrent_state_pace_b200 as pace
    # one head, d = 128: INT4 record 8192 codes + 256 scale bytes, INT8 16384 + 256
    s4, _, _ = pace.pace_pool_bytes(1, 1, 128, 128, 8, 0, 0, [4])
    s8, _, _ = pace.pace_pool_bytes(1, 1, 128, 128, 8, 0, 0, [8])
    assert (s4, s8) == (8448, 16640)
    # concurrency-stress pool: 4096 x 48 heads, 12 of them INT8
    bits = [8] * 12 + [4] * 36
    st, buf, aux = pace.pace_pool_bytes(4096, 48, 128, 128, 8, 0, 0, bits)
    assert st == 4096 * (12 * 16640 + 36 * 8448) == 2063597568
    # k,v rows; alpha,beta rows (32 B per head); Gram cache (256 B per head)
    assert buf == 4096 * 48 * 8 * 512 + 4096 * 48 * 32 + 4096 * 48 * 304
    # mixed 4/8 pool against an all-INT8 pool: 0.631 (the pages' "about two
    # thirds" of 8-bit memory, "PACE: four-bit recurrent state by rounding less
    # often", TL;DR; there the 8-bit baseline also keeps FP16 channels)
    st8, _, _ = pace.pace_pool_bytes(4096, 48, 128, 128, 8, 0, 0, [8] * 48)
    assert round(st / st8, 3) == 0.631
    # INT4 against a bf16 state of the same shape: 8448 / 32768
    assert round(s4 / (128 * 128 * 2), 3) == 0.258
    # tiny workload: 32 x 32 INT4 -> 512 code bytes + 64 scale bytes
    st, _, _ = pace.pace_pool_bytes(2, 2, 32, 32, 4, 0, 1, [4, 4])
    assert st == 2 * 2 * 576


@pytest.mark.parametrize("kw,status", [
    (dict(H=0), 1), (dict(H=257), 1), (dict(P=0), 1), (dict(P=17), 1), (dict(axis=2), 1),
    (dict(io=3), 1), (dict(bits=5), 1), (dict(d_v=64), 2), (dict(d_k=48, d_v=48), 2), (dict(B=0), 1),
])
def test_descriptor_validation(kw, status):
    import bit_recurrent_state_pace_b200 as pace
    a = dict(B=2, H=4, d_k=128, d_v=128, P=8, axis=0, io=0, bits=4)
    a.update(kw)
    bits = [a["bits"]] * max(a["H"], 1)
    with pytest.raises(pace.PaceError) as e:
        pace.pace_pool_bytes(a["B"], a["H"], a["d_k"], a["d_v"], a["P"], a["axis"], a["io"], bits)
    assert e.value.status == status


def test_e4m3_buffer_layout():
    import bit_recurrent_state_pace_b200 as pace
    bits = [8] * 12 + [4] * 36
    st, buf, _ = pace.pace_pool_bytes(4096, 48, 128, 128, 8, 0, 0, bits, 1)
    st0, buf0, _ = pace.pace_pool_bytes(4096, 48, 128, 128, 8, 0, 0, bits, 0)
    # k, v rows at one byte per element; gates and Gram cache unchanged
    assert st == st0 and buf0 - buf == 4096 * 48 * 8 * 256
    with pytest.raises(pace.PaceError) as e:
        pace.pace_pool_bytes(2, 4, 128, 128, 8, 0, 0, [4] * 4, 2)
    assert e.value.status == 1


def test_status_strings():
    import bit_recurrent_state_pace_b200 as pace
    assert pace.pace_status_string(0) == "PACE_OK"
    assert pace.pace_status_string(3) == "PACE_ERR_CUDA"
    assert pace.pace_version()


def test_binding_constants_match_the_header():
    """Every #define and enum value of include/pace.h that the binding
    mirrors has the same value there."""
    import bit_recurrent_state_pace_b200 as pace
    text = open(os.path.join(ROOT, "include", "pace.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    values = {m.group(1): int(m.group(2), 0)
              for m in re.finditer(r"#define\s+(PACE_\w+)\s+(0x[0-9a-fA-F]+|\d+)u?", text)}
    for m in re.finditer(r"(PACE_[A-Z0-9_]+)\s*=\s*(\d+)", text):
        values[m.group(1)] = int(m.group(2))
    mirrored = [n for n in values if hasattr(pace, n)]
    assert len(mirrored) >= 10, mirrored
    for n in mirrored:
        assert getattr(pace, n) == values[n], (n, getattr(pace, n), values[n])
