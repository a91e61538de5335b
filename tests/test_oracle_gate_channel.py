"""Pins of the oracle's per-channel gated compressor (the variant with one
gate per channel: g_id = x_id * w_d + b_id, softmax over the block's tokens
for every channel separately; the pages give no compressor formula, this is
the per-channel counterpart of the scalar-gate reading).

Pinned against: the block mean (zero gates), single-token selection by a
large bias per channel, the scalar-gate pooling when the gate does not
depend on the channel, independence of the channels, m = 1, and a second
transcription (oracle/twin.py)."""
import numpy as np
import pytest

import oracle
from oracle import twin


def _blk(seed, m, width):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((m, width)), rng.standard_normal(width) / 8, rng.standard_normal((m, width))


@pytest.mark.parametrize("m", [4, 128])
def test_zero_gates_give_the_block_mean(m):
    xs, _, _ = _blk(1, m, 64)
    out = oracle.gate_pool_channel(xs, np.zeros(64), np.zeros((m, 64)))
    assert np.allclose(out, xs.mean(axis=0), rtol=0, atol=1e-13)


def test_a_large_bias_selects_one_token_per_channel():
    xs, w, _ = _blk(2, 4, 32)
    b = np.zeros((4, 32))
    pick = np.arange(32) % 4
    b[pick, np.arange(32)] = 1e3
    out = oracle.gate_pool_channel(xs, w, b)
    assert np.allclose(out, xs[pick, np.arange(32)], rtol=0, atol=1e-12)


def test_channel_independent_gate_equals_scalar_gate_pooling():
    xs, _, _ = _blk(3, 4, 48)
    beta = np.array([0.3, -1.2, 2.0, 0.1])
    out = oracle.gate_pool_channel(xs, np.zeros(48), np.repeat(beta[:, None], 48, axis=1))
    ref, _ = oracle.gate_pool(xs, np.zeros(48), beta)
    assert np.allclose(out, ref, rtol=0, atol=1e-13)


def test_channels_are_independent_and_m1_is_the_identity():
    xs, w, b = _blk(4, 4, 16)
    out = oracle.gate_pool_channel(xs, w, b)
    xs2 = xs.copy()
    xs2[:, 5] += 7.0
    out2 = oracle.gate_pool_channel(xs2, w, b)
    keep = np.arange(16) != 5
    assert np.array_equal(out[keep], out2[keep])
    one = oracle.gate_pool_channel(xs[:1], w, b[:1])
    assert np.array_equal(one, xs[0])


@pytest.mark.parametrize("m,width", [(4, 512), (128, 512), (4, 128)])
def test_twin_agreement(m, width):
    for seed in range(3):
        xs, w, b = _blk(10 + seed, m, width)
        assert np.allclose(oracle.gate_pool_channel(xs, w, b), twin.pool_channel(xs, w, b), rtol=0, atol=1e-12)
