"""Seeded synthetic inputs shared by the tests, the oracle runs and the bench.

This module holds random-number generation and array shaping only: no step
of the attention method (no norm, rotation, pooling, quantisation, scoring,
selection or softmax) is computed here.

Generator: splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based stream.  Every named
tensor gets a 64-bit stream key (a hash of seed and name); element i of that
tensor is mix(key + (i + 1) * 0x9E3779B97F4A7C15), with mix the splitmix64
finaliser.  Normals come from the Box-Muller transform of two such uniform
streams.  Everything is vectorised uint64 arithmetic, so the same
(seed, name, shape) always yields the same bytes.
"""
import hashlib

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z):
    z = z.copy()
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def _key(seed, name):
    h = hashlib.sha256(("%d/%s" % (seed, name)).encode()).digest()
    return np.uint64(int.from_bytes(h[:8], "little"))


def u64(seed, name, n, start=0):
    """Raw 64-bit outputs start..start+n-1 of the (seed, name) stream."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _key(seed, name) + i * _GOLDEN
    return _mix(z)


def uniform(seed, name, shape, start=0):
    """U(0,1) with 53-bit resolution, never exactly 0 (elements start.. of the stream)."""
    n = int(np.prod(shape)) if len(shape) else 1
    u = (u64(seed, name, n, start) >> np.uint64(11)).astype(np.float64)
    return ((u + 0.5) * (1.0 / 9007199254740992.0)).reshape(shape)


def normal(seed, name, shape, std=1.0, mean=0.0, start=0):
    """N(mean, std^2) by Box-Muller on two independent sub-streams; element
    i of the result is element start+i of the stream."""
    n = int(np.prod(shape)) if len(shape) else 1
    u1 = uniform(seed, name + "#a", (n,), start)
    u2 = uniform(seed, name + "#b", (n,), start)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return (mean + std * z).reshape(shape)


def integers(seed, name, shape, lo, hi):
    """Uniform integers in [lo, hi)."""
    n = int(np.prod(shape)) if len(shape) else 1
    r = u64(seed, name, n) % np.uint64(hi - lo)
    return (r.astype(np.int64) + lo).reshape(shape)


def permutation(seed, name, n):
    """A seeded permutation of range(n) (argsort of a uniform stream)."""
    return np.argsort(uniform(seed, name, (n,)), kind="stable")


def to_bf16_bits(x):
    """Round float64 values to bfloat16 (nearest even) and return the uint16
    bit patterns: used to make activations that are exact bf16 inputs."""
    f = np.asarray(x, np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f64(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32) \
        .astype(np.float64)
