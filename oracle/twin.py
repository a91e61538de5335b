"""Second, separately written fp64 transcription of the hot path in numpy.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  It exists so that one
author's slip in csla_oracle.c shows up as a disagreement between two
independent writings of the same definitions; it is used on tiny inputs only.
The codecs here use ml_dtypes' float8_e4m3fn / bfloat16 conversions (a
library routine), not the C oracle's own rounding code.

Definitions as in oracle/csla_oracle.c: haiqwa.github.io "DeepSeek-V4" blog
§RMSNorm归一化, §Partial RoPE位置编码, §让注意力学会"忽略"; 硅星人 article
§两大压缩注意力 (CSA/HCA data flow).
"""
import ml_dtypes
import numpy as np


def e4m3_values():
    """All 256 E4M3 codes as float64 (ml_dtypes view of the bytes)."""
    return np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def quantize(y, d_rope=64):
    y32 = np.asarray(y, np.float64).astype(np.float32)
    dn = y32.shape[-1] - d_rope
    amax = np.float32(np.max(np.abs(y32[:dn]))) if dn else np.float32(0)
    scale = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    v = (y32[:dn] / scale).astype(np.float32)
    v = np.clip(v, -448.0, 448.0)
    codes = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    rope = y32[dn:].astype(ml_dtypes.bfloat16).view(np.uint16)
    row = np.concatenate([codes, rope.view(np.uint8)])
    return row, scale


def dequantize(row, scale, D, d_rope=64):
    row = np.asarray(row, np.uint8)
    dn = D - d_rope
    nope = row[:dn].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * np.float64(scale)
    rope = row[dn:dn + 2 * d_rope].copy().view(ml_dtypes.bfloat16).astype(np.float64)
    return np.concatenate([nope, rope])


def rms(x, gamma, eps=1e-6):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def rotate(y, pos, theta=10000.0, d_rope=64):
    y = np.array(y, np.float64)
    D = y.shape[-1]
    half = d_rope // 2
    ang = np.float64(pos) * theta ** (-np.arange(half) * 2.0 / d_rope)
    ev = y[..., D - d_rope::2].copy()
    od = y[..., D - d_rope + 1::2].copy()
    y[..., D - d_rope::2] = ev * np.cos(ang) - od * np.sin(ang)
    y[..., D - d_rope + 1::2] = ev * np.sin(ang) + od * np.cos(ang)
    return y


def pool(xs, wg, gb):
    xs = np.asarray(xs, np.float64)
    g = xs @ np.asarray(wg, np.float64) + np.asarray(gb, np.float64)
    a = np.exp(g - g.max())
    a /= a.sum()
    return a @ xs


def pool_channel(xs, w, b):
    """Per-channel gates: a separate softmax over the block's tokens for every channel."""
    xs = np.asarray(xs, np.float64)
    g = xs * np.asarray(w, np.float64)[None, :] + np.broadcast_to(np.asarray(b, np.float64), xs.shape)
    a = np.exp(g - g.max(axis=0, keepdims=True))
    a /= a.sum(axis=0, keepdims=True)
    return (a * xs).sum(axis=0)


def window_row(x, gamma, pos, eps=1e-6, theta=10000.0, d_rope=64):
    return quantize(rotate(rms(x, gamma, eps), pos, theta, d_rope), d_rope)


def compressed_row(xs, wg, gb, gamma, bk, eps=1e-6, theta=10000.0, d_rope=64):
    m = np.asarray(xs).shape[0]
    return quantize(rotate(rms(pool(xs, wg, gb), gamma, eps), bk * m, theta, d_rope), d_rope)


def index_key(xis, wgi, gbi):
    c = pool(xis, wgi, gbi).astype(np.float32)
    return c.astype(ml_dtypes.bfloat16).view(np.uint16)


def key_scale_e4m3(amax):
    """2^ceil(log2(amax / 448)), exponent clamped to [-126, 127] (by frexp)."""
    if amax <= 0:
        return 2.0 ** -126
    mant, ex = np.frexp(np.float64(amax) / 448.0)   # amax/448 = mant * 2^ex, mant in [0.5, 1)
    e = ex - 1 if mant == 0.5 else ex
    return 2.0 ** int(min(max(e, -126), 127))


def index_key_e4m3(xis, wgi, gbi):
    c = pool(xis, wgi, gbi).astype(np.float32)
    s = key_scale_e4m3(float(np.max(np.abs(c))))
    v = np.clip((c.astype(np.float64) / s).astype(np.float32), -448.0, 448.0)
    return v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8), s


def scores(cq, W, w, keys, HI, dI):
    qI = (np.asarray(W, np.float64) @ np.asarray(cq, np.float64)).reshape(HI, dI)
    dots = np.asarray(keys, np.float64) @ qI.T          # [N, HI]
    return np.maximum(dots, 0.0) @ np.asarray(w, np.float64)


def topk(sc, k):
    sc = np.asarray(sc, np.float64)
    order = np.lexsort((np.arange(len(sc)), -sc))      # score desc, then index asc
    sel = np.sort(order[:k])
    out = -np.ones(k, np.int32)
    out[:len(sel)] = sel
    return out


def attend(q, gamma_q, t, rows, sink, eps=1e-6, theta=10000.0, d_rope=64):
    q = np.asarray(q, np.float64)
    H, D = q.shape
    qh = rotate(rms(q, gamma_q, eps), t, theta, d_rope)          # [H, D]
    rows = np.asarray(rows, np.float64).reshape(-1, D)
    logits = np.concatenate([np.asarray(sink, np.float64)[:, None], qh @ rows.T / np.sqrt(D)], axis=1)
    logits -= logits.max(axis=1, keepdims=True)
    e = np.exp(logits)
    p = e / e.sum(axis=1, keepdims=True)
    return p[:, 1:] @ rows, p[:, 0]
