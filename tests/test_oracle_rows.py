"""Pins for the oracle's per-row steps: RMSNorm, partial RoPE, the mixed
fp8/bf16 row quantiser, the gated block compressor and the index key."""
import math

import numpy as np
import pytest

from conftest import read_table

RNG = np.random.default_rng(7)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_unit_mean_square(oracle_lib):
    for D in (128, 512):
        x = RNG.standard_normal(D) * 3.0
        y = oracle_lib.rmsnorm(x, np.ones(D), eps=1e-6)
        ms = np.mean(x * x)
        # closed form: mean(y^2) = ms / (ms + eps)
        assert abs(np.mean(y * y) - ms / (ms + 1e-6)) < 1e-14
        assert np.all(np.sign(y) == np.sign(x))


def test_rmsnorm_gamma_and_scale_invariance(oracle_lib):
    D = 64
    x = RNG.standard_normal(D)
    g = RNG.standard_normal(D)
    y1 = oracle_lib.rmsnorm(x, g, eps=0.0)
    y2 = oracle_lib.rmsnorm(7.5 * x, g, eps=0.0)
    assert np.allclose(y1, y2, rtol=0, atol=1e-14)
    assert np.allclose(y1, oracle_lib.rmsnorm(x, None, eps=0.0) * g, atol=1e-14)
    # constant vector -> all ones (times gamma)
    assert np.allclose(oracle_lib.rmsnorm(np.full(D, -2.0), None, eps=0.0), -1.0)


# ---------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity(oracle_lib):
    y = RNG.standard_normal(512)
    assert np.array_equal(oracle_lib.rope(y, 0), y)


def test_rope_touches_only_last_64_dims_and_keeps_norm(oracle_lib):
    y = RNG.standard_normal(512)
    r = oracle_lib.rope(y, 12345)
    assert np.array_equal(r[:448], y[:448])
    assert not np.allclose(r[448:], y[448:])
    assert abs(np.linalg.norm(r[448:]) - np.linalg.norm(y[448:])) < 1e-12
    # every pair keeps its own norm
    pr = r[448:].reshape(32, 2)
    py = y[448:].reshape(32, 2)
    assert np.allclose(np.hypot(pr[:, 0], pr[:, 1]), np.hypot(py[:, 0], py[:, 1]), atol=1e-13)


def test_rope_pair_zero_closed_form(oracle_lib):
    """Pair 0 has frequency theta^0 = 1: position pi/2 rad rotates (1,0) to (0,1)
    by the angle `pos` itself; pair i rotates by pos*theta^(-2i/64)."""
    D = 128
    for i in (0, 5, 31):
        y = np.zeros(D)
        y[64 + 2 * i] = 1.0
        pos = 3
        r = oracle_lib.rope(y, pos, theta=10000.0)
        ang = pos * 10000.0 ** (-2.0 * i / 64)
        assert abs(r[64 + 2 * i] - math.cos(ang)) < 1e-15
        assert abs(r[64 + 2 * i + 1] - math.sin(ang)) < 1e-15
        assert np.count_nonzero(r) <= 2


def test_rope_relative_position_invariance(oracle_lib):
    q = RNG.standard_normal(512)
    k = RNG.standard_normal(512)
    for (pq, pk, delta) in [(100, 37, 1000), (5, 5, 131071), (1048575, 0, -1000)]:
        a = oracle_lib.rope(q, pq) @ oracle_lib.rope(k, pk)
        b = oracle_lib.rope(q, pq + delta) @ oracle_lib.rope(k, pk + delta)
        assert abs(a - b) < 1e-9 * (1 + abs(a))


# ---------------------------------------------------------------- quantiser
def test_quantize_layout_and_bounds(oracle_lib):
    D = 512
    y = RNG.standard_normal(D) * 2.0
    row, scale = oracle_lib.quantize(y)
    assert row.shape == (576,)
    amax = np.float32(np.max(np.abs(np.float32(y[:448]))))
    assert scale == np.float32(amax / np.float32(448.0))
    deq = oracle_lib.dequantize(row, scale, D)
    # the largest fp8 dim maps exactly to +-448 * scale
    j = int(np.argmax(np.abs(y[:448])))
    assert abs(deq[j]) == 448.0 * float(scale)
    # E4M3 RNE: relative error <= 2^-4 for normals, absolute <= 2^-10*scale below 2^-6*scale
    err = np.abs(deq[:448] - y[:448])
    bound = np.maximum(np.abs(y[:448]) * 2.0 ** -4, 2.0 ** -10 * float(scale)) * (1 + 1e-6)
    assert np.all(err <= bound)
    # bf16 RoPE dims: relative error <= 2^-8
    assert np.all(np.abs(deq[448:] - y[448:]) <= np.abs(y[448:]) * 2.0 ** -8 + 1e-30)
    # little-endian bf16 at bytes 448..575
    h = int(row[448]) | (int(row[449]) << 8)
    assert oracle_lib.bf16_value(h) == deq[448]


def test_quantize_zero_row_has_unit_scale(oracle_lib):
    y = np.zeros(128)
    y[64:] = 1.5
    row, scale = oracle_lib.quantize(y)
    assert scale == 1.0 and np.all(row[:64] == 0)


def test_quantize_exact_values_roundtrip(oracle_lib):
    """Values that are exactly E4M3 codes times a power-of-two scale survive."""
    codes = np.array([0x7E, 0x38, 0x01, 0x40, 0xB8, 0x0F] * 11, np.uint8)[:64]
    vals = np.array([oracle_lib.e4m3_value(c) for c in codes]) * 2.0 ** -3
    y = np.concatenate([vals, np.ones(64)])
    row, scale = oracle_lib.quantize(y)
    assert scale == 2.0 ** -3
    assert np.array_equal(row[:64], codes)


# ---------------------------------------------------------------- compressor
def test_gate_pool_zero_gate_is_block_mean(oracle_lib):
    xs = RNG.standard_normal((4, 96))
    out, alpha = oracle_lib.gate_pool(xs, np.zeros(96), np.zeros(4))
    assert np.allclose(alpha, 0.25, atol=0)
    assert np.allclose(out, xs.mean(axis=0), atol=1e-15)


def test_gate_pool_large_bias_selects_token(oracle_lib):
    xs = RNG.standard_normal((128, 32))
    for i in (0, 77, 127):
        gb = np.zeros(128)
        gb[i] = 1e3
        out, alpha = oracle_lib.gate_pool(xs, RNG.standard_normal(32) * 0.01, gb)
        assert abs(alpha[i] - 1.0) < 1e-12
        assert np.allclose(out, xs[i], atol=1e-12)


def test_gate_pool_weights_are_softmax_of_gate(oracle_lib):
    xs = RNG.standard_normal((4, 16))
    wg = RNG.standard_normal(16)
    gb = RNG.standard_normal(4)
    out, alpha = oracle_lib.gate_pool(xs, wg, gb)
    assert abs(alpha.sum() - 1.0) < 1e-15
    g = xs @ wg + gb
    # ratio of weights = exp of gate difference
    assert abs(alpha[1] / alpha[0] - math.exp(g[1] - g[0])) < 1e-12
    # a shift of every bias by c changes nothing
    out2, alpha2 = oracle_lib.gate_pool(xs, wg, gb + 123.0)
    assert np.allclose(alpha, alpha2, atol=1e-15)


def test_compressed_row_with_m1_is_window_row(oracle_lib):
    """m = 1: the block is one token, softmax weight 1, RoPE at b*1 = the token's
    own position: the compressed entry must equal the window row."""
    D = 512
    x = RNG.standard_normal((1, D))
    gamma = 1 + 0.1 * RNG.standard_normal(D)
    for b in (0, 9, 70000):
        r1, s1 = oracle_lib.compressed_row(x, RNG.standard_normal(D), RNG.standard_normal(1), gamma, b)
        r2, s2 = oracle_lib.window_row(x[0], gamma, b)
        assert np.array_equal(r1, r2) and s1 == s2


def test_compressed_row_rope_at_block_start(oracle_lib):
    """Identical block content in two blocks differs only through RoPE at b*m."""
    D, m = 128, 4
    xs = RNG.standard_normal((m, D))
    wg, gb, gamma = RNG.standard_normal(D) * 0.05, RNG.standard_normal(m), np.ones(D)
    r0, s0 = oracle_lib.compressed_row(xs, wg, gb, gamma, 0)
    r5, s5 = oracle_lib.compressed_row(xs, wg, gb, gamma, 5)
    assert np.array_equal(r0[:64], r5[:64]) and s0 == s5
    c, _ = oracle_lib.gate_pool(xs, wg, gb)
    y = oracle_lib.rope(oracle_lib.rmsnorm(c, gamma), 20)
    ref_row, _ = oracle_lib.quantize(y)
    assert np.array_equal(ref_row, r5)


def test_index_key_is_bf16_of_pooled_keys(oracle_lib):
    xis = RNG.standard_normal((4, 64))
    key = oracle_lib.index_key(xis, np.zeros(64), np.zeros(4))
    mean = xis.mean(axis=0)
    for e in range(64):
        assert key[e] == oracle_lib.bf16_from_f32(np.float32(mean[e]))


# ---------------------------------------------------------------- page constants
def test_page_constants_consistent():
    t = {k: int(v) for k, v, _ in read_table("page_constants.txt")}
    import oracle
    assert math.lcm(t["csa_m"], t["hca_m"]) == t["page_tokens"] == oracle.PAGE_TOKENS
    assert t["page_tokens"] // t["csa_m"] == t["csa_entries_page"]
    assert t["page_tokens"] // t["hca_m"] == t["hca_entries_page"]
    assert t["d_rope"] < t["head_dim"]
    # the tail (< m tokens) always fits inside the window: no token is ever
    # invisible to the current query
    assert t["hca_m"] - 1 < t["n_win"] and t["csa_m"] - 1 < t["n_win"]


def test_visibility_rule(oracle_lib):
    # block b visible at context L iff (b+1)*m <= L
    for m in (4, 128):
        for L in range(0, 3 * m + 2):
            assert oracle_lib.n_visible(L, m) == sum(1 for b in range(L) if (b + 1) * m <= L)
