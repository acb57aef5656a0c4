"""Decode from host memory (pace_decode_host).

The host-buffer entry point only moves bytes and orders streams around the
same kernels as the device path (decode step, then the commit of full heads),
so its outputs and the pool it leaves must equal, bit for bit, those of the
device-path calls on the same inputs -- for a token count that is not a
multiple of the period, across two calls that reuse the staging buffer, and
with the output copy left out.
"""
import pytest
import torch

import pace_synth

pytestmark = pytest.mark.gpu


def _pool(w, bits, S):
    import bit_recurrent_state_pace_b200 as pace
    pool = pace.PacePool(w.B, w.H, w.d_k, w.d_v, w.P, bits, axis=w.axis, io=w.io_dtype)
    pool.load(S)
    return pool


def _host_tokens(w, t0, T):
    xs = [pace_synth.token_inputs(w, t, seed=21, device="cpu") for t in range(t0, t0 + T)]
    return {k: torch.stack([x[k] for x in xs]).contiguous().pin_memory() for k in xs[0]}


def _device_run(pool, w, h, o):
    for t in range(h["q"].shape[0]):
        x = {k: v[t].cuda() for k, v in h.items()}
        pool.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], o[t])
        pool.commit_period()


@pytest.mark.parametrize("name,axis", [("mixed_4_8", "col"), ("gdn_layer_4b", "row")])
def test_host_path_matches_device_calls_bit_for_bit(name, axis):
    w = pace_synth.workload(name, B=24, axis=axis)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=5, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    dev, host = _pool(w, bits, S), _pool(w, bits, S)
    for t0, T in ((0, 2 * w.P + 3), (2 * w.P + 3, w.P + 1)):   # ragged, then a second call
        h = _host_tokens(w, t0, T)
        o_dev = torch.empty(T, w.B, w.H, w.d_v, device="cuda")
        _device_run(dev, w, h, o_dev)
        o_host = torch.full((T, w.B, w.H, w.d_v), float("nan")).pin_memory()
        host.decode_host(h["q"], h["k"], h["v"], h["alpha"], h["beta"], o_host)
        torch.cuda.synchronize()
        assert torch.equal(o_dev.cpu(), o_host), (t0, T)
    assert dev.status() == 0 and host.status() == 0
    assert torch.equal(dev.state, host.state)
    assert torch.equal(dev.buffer, host.buffer)
    assert torch.equal(dev.fill(), host.fill())


def test_host_path_with_a_commit_threshold():
    """With a commit threshold the host path commits the heads each step marks,
    exactly as the device-path calls do."""
    w = pace_synth.workload("mixed_4_8", B=6)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=8, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    dev, host = _pool(w, bits, S), _pool(w, bits, S)
    for pool in (dev, host):
        pool.set_commit_threshold(4.0)
    T = 2 * w.P + 1
    h = _host_tokens(w, 0, T)
    o_dev = torch.empty(T, w.B, w.H, w.d_v, device="cuda")
    _device_run(dev, w, h, o_dev)
    o_host = torch.empty(T, w.B, w.H, w.d_v).pin_memory()
    host.decode_host(h["q"], h["k"], h["v"], h["alpha"], h["beta"], o_host)
    torch.cuda.synchronize()
    assert torch.equal(o_dev.cpu(), o_host)
    assert torch.equal(dev.state, host.state)
    assert torch.equal(dev.fill(), host.fill())
    assert dev.status() == 0 and host.status() == 0


def test_host_path_without_outputs_still_advances_the_pool():
    w = pace_synth.workload("mixed_4_8", B=8)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=6, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    dev, host = _pool(w, bits, S), _pool(w, bits, S)
    h = _host_tokens(w, 0, w.P + 2)
    _device_run(dev, w, h, torch.empty(w.P + 2, w.B, w.H, w.d_v, device="cuda"))
    host.decode_host(h["q"], h["k"], h["v"], h["alpha"], h["beta"], None)
    torch.cuda.synchronize()
    assert torch.equal(dev.state, host.state)
    assert torch.equal(dev.buffer, host.buffer)
    assert torch.equal(dev.fill(), host.fill())


def test_host_path_rejects_shared_streams_and_device_tensors():
    import bit_recurrent_state_pace_b200 as pace
    w = pace_synth.workload("mixed_4_8", B=2)
    bits = pace_synth.head_bits(w, 0)
    S = pace_synth.random_state(w.B * w.H, w.d_v, w.d_k, seed=7, device="cuda").view(
        w.B, w.H, w.d_v, w.d_k)
    pool = _pool(w, bits, S)
    h = _host_tokens(w, 0, 1)
    staging = torch.empty(pace.pace_host_staging_bytes(pool.handle), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    with pytest.raises(RuntimeError):
        pace.pace_decode_host(pool.handle, 1, h["q"], h["k"], h["v"], h["alpha"], h["beta"], None,
                              staging, s, s, torch.cuda.Stream())
    with pytest.raises(ValueError):
        pace.pace_decode_host(pool.handle, 1, h["q"].cuda(), h["k"], h["v"], h["alpha"], h["beta"],
                              None, staging, s, torch.cuda.Stream(), torch.cuda.Stream())
