"""The csla_synth streams evaluated with torch on any device (used to make
the large synthetic token streams directly in GPU memory).

Same definition as csla_synth.normal: element i of stream (seed, name) is
splitmix64's finaliser applied to key + (i+1)*0x9E3779B97F4A7C15, two such
streams feed Box-Muller.  uint64 arithmetic is emulated on int64 tensors
(wrapping multiply, masked right shifts).  Bits agree with the numpy version
except where float64 log/cos of the two libraries differ in the last ulp.
"""
import numpy as np
import torch

from . import _key

_MASK = {k: (1 << (64 - k)) - 1 for k in (11, 27, 30, 31)}


def _s64(u):
    """uint64 constant -> the int64 with the same bits."""
    u = int(u)
    return u - (1 << 64) if u >= (1 << 63) else u


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_M1 = _s64(0xBF58476D1CE4E5B9)
_M2 = _s64(0x94D049BB133111EB)


def _srl(z, k):
    return (z >> k) & _MASK[k]


def _mix(z):
    z = (z ^ _srl(z, 30)) * _M1
    z = (z ^ _srl(z, 27)) * _M2
    return z ^ _srl(z, 31)


def uniform(seed, name, n, start=0, device="cuda"):
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = _mix(_s64(_key(seed, name)) + i * _GOLDEN)
    u = _srl(z, 11).to(torch.float64)
    return (u + 0.5) * (1.0 / 9007199254740992.0)


def normal(seed, name, shape, start=0, device="cuda", std=1.0):
    n = int(np.prod(shape)) if len(shape) else 1
    u1 = uniform(seed, name + "#a", n, start, device)
    u2 = uniform(seed, name + "#b", n, start, device)
    z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * np.pi * u2)
    return (std * z).reshape(shape)
