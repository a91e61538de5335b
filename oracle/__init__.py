"""fp64 CPU oracle for the CSA/HCA compressed-attention hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library: the arithmetic lives in
``csla_oracle.c`` (plain C, fp64) and a second, separately written numpy
transcription lives in ``twin.py``; the cache byte format is decoded here from
its written definition.

Sources: haiqwa.github.io "DeepSeek-V4" blog (§CSA, §HCA, §RMSNorm归一化,
§Partial RoPE位置编码, §让注意力学会"忽略", §索引可见性处理) and the 硅星人 article
"DeepSeek V4 ... 让token大降价", §两大压缩注意力 (CSA/HCA data flow, window of
128, sink logit, RoPE on the last 64 dims, bf16/fp8 cache, state cache and
classical cache).  Every function is pinned by tests/test_oracle_*.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

PAGE_TOKENS = 128  # a classical-cache block covers lcm(4, 128) raw tokens

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        fp = ctypes.POINTER(ctypes.c_float)
        ll = ctypes.c_longlong
        I = ctypes.c_int
        D_ = ctypes.c_double
        sig = {
            "csla_orc_e4m3_value": (D_, [ctypes.c_uint]),
            "csla_orc_e4m3_from_f32": (ctypes.c_uint, [ctypes.c_float]),
            "csla_orc_bf16_value": (D_, [ctypes.c_uint]),
            "csla_orc_bf16_from_f32": (ctypes.c_uint, [ctypes.c_float]),
            "csla_orc_rmsnorm": (None, [dp, dp, I, D_, dp]),
            "csla_orc_rope": (None, [dp, I, I, ll, D_]),
            "csla_orc_quantize": (None, [dp, I, I, u8p, fp]),
            "csla_orc_dequantize": (None, [u8p, ctypes.c_float, I, I, dp]),
            "csla_orc_gate_pool": (None, [dp, I, I, dp, dp, dp, dp]),
            "csla_orc_window_row": (None, [dp, dp, I, I, D_, D_, ll, u8p, fp]),
            "csla_orc_compressed_row": (None, [dp, I, dp, dp, dp, I, I, D_, D_, ll, u8p, fp]),
            "csla_orc_index_key": (None, [dp, I, dp, dp, I, u16p]),
            "csla_orc_key_scale_e4m3": (D_, [D_]),
            "csla_orc_gate_pool_channel": (None, [dp, I, I, dp, dp, dp]),
            "csla_orc_key_bf16": (None, [dp, I, u16p]),
            "csla_orc_key_e4m3": (None, [dp, I, u8p, fp]),
            "csla_orc_index_key_e4m3": (None, [dp, I, dp, dp, I, u8p, fp]),
            "csla_orc_index_query": (None, [dp, dp, I, I, I, dp]),
            "csla_orc_index_scores": (None, [dp, dp, I, I, dp, ll, dp]),
            "csla_orc_topk": (None, [dp, I, I, i32p]),
            "csla_orc_attend": (None, [dp, dp, ll, dp, I, dp, I, I, I, D_, D_, dp, dp]),
            "csla_orc_n_visible": (ll, [ll, I]),
            "csla_orc_gather_set": (I, [u8p, fp, i32p, I, u8p, fp, I, I, ll, I, I, I, i32p, I, dp]),
            "csla_orc_gather_keys": (None, [ctypes.c_void_p, fp, i32p, I, I, ll, I, I, dp]),
            "csla_orc_csa_decode": (None, [u8p, fp, ctypes.c_void_p, fp, i32p, I, u8p, fp, I, i32p, i32p, I, I, I,
                                           I, I, I, I, I, I, D_, D_, dp, dp, dp, dp, dp, dp, i32p,
                                           dp]),
            "csla_orc_hca_decode": (None, [u8p, fp, i32p, I, u8p, fp, I, i32p, i32p, I, I, I, I, I,
                                           D_, D_, dp, dp, dp, dp]),
            "csla_orc_num_threads": (I, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ---------------------------------------------------------------- codecs
def e4m3_value(code):
    return lib().csla_orc_e4m3_value(int(code))


def e4m3_from_f32(v):
    return lib().csla_orc_e4m3_from_f32(float(np.float32(v)))


def bf16_value(h):
    return lib().csla_orc_bf16_value(int(h))


def bf16_from_f32(v):
    return lib().csla_orc_bf16_from_f32(float(np.float32(v)))


# ---------------------------------------------------------------- rows
def rmsnorm(x, gamma=None, eps=1e-6):
    x = _d(x)
    y = np.empty_like(x)
    g = None if gamma is None else _d(gamma)
    lib().csla_orc_rmsnorm(_p(x, ctypes.c_double), None if g is None else _p(g, ctypes.c_double),
                           x.shape[-1], eps, _p(y, ctypes.c_double))
    return y


def rope(y, pos, theta=10000.0, d_rope=64):
    y = _d(y).copy()
    lib().csla_orc_rope(_p(y, ctypes.c_double), y.shape[-1], d_rope, int(pos), theta)
    return y


def row_bytes(D, d_rope=64):
    return (D - d_rope) + 2 * d_rope


def quantize(y, d_rope=64):
    y = _d(y)
    D = y.shape[-1]
    row = np.zeros(row_bytes(D, d_rope), np.uint8)
    sc = np.zeros(1, np.float32)
    lib().csla_orc_quantize(_p(y, ctypes.c_double), D, d_rope, _p(row, ctypes.c_uint8),
                            _p(sc, ctypes.c_float))
    return row, sc[0]


def dequantize(row, scale, D, d_rope=64):
    row = np.ascontiguousarray(row, np.uint8)
    x = np.zeros(D, np.float64)
    lib().csla_orc_dequantize(_p(row, ctypes.c_uint8), float(scale), D, d_rope, _p(x, ctypes.c_double))
    return x


def dequantize_rows(rows, scales, D, d_rope=64):
    rows = np.asarray(rows, np.uint8).reshape(-1, row_bytes(D, d_rope))
    scales = np.asarray(scales, np.float32).reshape(-1)
    return np.stack([dequantize(rows[i], scales[i], D, d_rope) for i in range(rows.shape[0])]) \
        if rows.shape[0] else np.zeros((0, D))


def gate_pool(xs, wg, gb=None):
    xs = _d(xs)
    m, width = xs.shape
    wg = _d(wg)
    out = np.zeros(width)
    alpha = np.zeros(m)
    g = None if gb is None else _d(gb)
    lib().csla_orc_gate_pool(_p(xs, ctypes.c_double), m, width, _p(wg, ctypes.c_double),
                             None if g is None else _p(g, ctypes.c_double), _p(out, ctypes.c_double),
                             _p(alpha, ctypes.c_double))
    return out, alpha


def gate_pool_channel(xs, w, b):
    """Per-channel gated pooling: out_d = sum_i softmax_i(x_id w_d + b_id) x_id."""
    xs = _d(xs)
    m, width = xs.shape
    w, b = _d(w), _d(np.broadcast_to(b, (m, width)))
    out = np.zeros(width)
    lib().csla_orc_gate_pool_channel(_p(xs, ctypes.c_double), m, width, _p(w, ctypes.c_double),
                                     _p(b, ctypes.c_double), _p(out, ctypes.c_double))
    return out


def key_bf16(c):
    c = _d(c)
    key = np.zeros(c.shape[-1], np.uint16)
    lib().csla_orc_key_bf16(_p(c, ctypes.c_double), c.shape[-1], _p(key, ctypes.c_uint16))
    return key


def key_e4m3(c):
    c = _d(c)
    codes = np.zeros(c.shape[-1], np.uint8)
    sc = np.zeros(1, np.float32)
    lib().csla_orc_key_e4m3(_p(c, ctypes.c_double), c.shape[-1], _p(codes, ctypes.c_uint8), _p(sc, ctypes.c_float))
    return codes, float(sc[0])


def compressed_row_channel(xs, w, b, gamma, bk, eps=1e-6, theta=10000.0, d_rope=64):
    """Compressed entry of block bk with the per-channel gate: pool, then
    RMSNorm * gamma, RoPE at position bk * m, quantise (as compressed_row)."""
    m = np.asarray(xs).shape[0]
    y = rope(rmsnorm(gate_pool_channel(xs, w, b), gamma, eps), bk * m, theta, d_rope)
    return quantize(y, d_rope)


def window_row(x, gamma, pos, eps=1e-6, theta=10000.0, d_rope=64):
    x = _d(x)
    g = _d(gamma)
    D = x.shape[-1]
    row = np.zeros(row_bytes(D, d_rope), np.uint8)
    sc = np.zeros(1, np.float32)
    lib().csla_orc_window_row(_p(x, ctypes.c_double), _p(g, ctypes.c_double), D, d_rope, eps, theta,
                              int(pos), _p(row, ctypes.c_uint8), _p(sc, ctypes.c_float))
    return row, sc[0]


def compressed_row(xs, wg, gb, gamma, bk, eps=1e-6, theta=10000.0, d_rope=64):
    xs = _d(xs)
    m, D = xs.shape
    wg, gb, g = _d(wg), _d(gb), _d(gamma)
    row = np.zeros(row_bytes(D, d_rope), np.uint8)
    sc = np.zeros(1, np.float32)
    lib().csla_orc_compressed_row(_p(xs, ctypes.c_double), m, _p(wg, ctypes.c_double),
                                  _p(gb, ctypes.c_double), _p(g, ctypes.c_double), D, d_rope, eps,
                                  theta, int(bk), _p(row, ctypes.c_uint8), _p(sc, ctypes.c_float))
    return row, sc[0]


def index_key(xis, wgi, gbi):
    xis = _d(xis)
    m, dI = xis.shape
    wgi, gbi = _d(wgi), _d(gbi)
    key = np.zeros(dI, np.uint16)
    lib().csla_orc_index_key(_p(xis, ctypes.c_double), m, _p(wgi, ctypes.c_double),
                             _p(gbi, ctypes.c_double), dI, _p(key, ctypes.c_uint16))
    return key


def key_scale_e4m3(amax):
    """Smallest 2^e (-126 <= e <= 127) with 448 * 2^e >= amax."""
    return float(lib().csla_orc_key_scale_e4m3(float(amax)))


def index_key_e4m3(xis, wgi, gbi):
    """E4M3 storage of a CSA block's index key: (codes uint8 [dI], scale)."""
    xis = _d(xis)
    m, dI = xis.shape
    wgi, gbi = _d(wgi), _d(gbi)
    codes = np.zeros(dI, np.uint8)
    sc = np.zeros(1, np.float32)
    lib().csla_orc_index_key_e4m3(_p(xis, ctypes.c_double), m, _p(wgi, ctypes.c_double),
                                  _p(gbi, ctypes.c_double), dI, _p(codes, ctypes.c_uint8), _p(sc, ctypes.c_float))
    return codes, float(sc[0])


# ---------------------------------------------------------------- indexer / top-k / attention
def index_query(cq, W, HI, dI):
    cq, W = _d(cq), _d(W)
    dc = cq.shape[-1]
    assert W.shape == (HI * dI, dc)
    qI = np.zeros(HI * dI)
    lib().csla_orc_index_query(_p(cq, ctypes.c_double), _p(W, ctypes.c_double), HI, dI, dc,
                               _p(qI, ctypes.c_double))
    return qI.reshape(HI, dI)


def index_scores(qI, w, keys):
    qI, w, keys = _d(qI), _d(w), _d(keys)
    HI, dI = qI.shape
    N = keys.shape[0]
    sc = np.zeros(max(N, 1))
    lib().csla_orc_index_scores(_p(qI, ctypes.c_double), _p(w, ctypes.c_double), HI, dI,
                                _p(keys, ctypes.c_double), N, _p(sc, ctypes.c_double))
    return sc[:N]


def topk(scores, k):
    scores = _d(scores)
    idx = np.zeros(k, np.int32)
    lib().csla_orc_topk(_p(scores, ctypes.c_double), scores.shape[0], k, _p(idx, ctypes.c_int32))
    return idx


def attend(q, gamma_q, t, rows, sink, eps=1e-6, theta=10000.0, d_rope=64):
    """q: [H, D] raw query heads; rows: [n, D] values; returns (out [H, D], sink_share [H])."""
    q, g, rows, sink = _d(q), _d(gamma_q), _d(rows), _d(sink)
    H, D = q.shape
    n = rows.shape[0]
    out = np.zeros((H, D))
    share = np.zeros(H)
    lib().csla_orc_attend(_p(q, ctypes.c_double), _p(g, ctypes.c_double), int(t),
                          _p(rows, ctypes.c_double) if n else None, n, _p(sink, ctypes.c_double), H, D,
                          d_rope, eps, theta, _p(out, ctypes.c_double), _p(share, ctypes.c_double))
    return out, share


def n_visible(L, m):
    return int(lib().csla_orc_n_visible(int(L), int(m)))


# ---------------------------------------------------------------- cache views
class CacheView:
    """Host copies of one layer's classical cache and state cache, in the
    byte layout the library defines (see include/csla.h):

      rows   [n_pages, 128//m, row_bytes] uint8      scales [n_pages, 128//m] f32
      kidx   [n_pages, 128//m, dI] uint16 (bf16)     block_table [n_slots, bt_stride] int32
             or uint8 E4M3 codes with kscale [n_pages, 128//m] f32
      win_rows [n_slots, n_win, row_bytes] uint8     win_scales [n_slots, n_win] f32
    """

    def __init__(self, m, D, rows, scales, block_table, win_rows, win_scales, kidx=None, dI=0,
                 d_rope=64, kscale=None):
        self.m, self.D, self.d_rope, self.dI = m, D, d_rope, dI
        self.rows = np.ascontiguousarray(rows, np.uint8)
        self.scales = np.ascontiguousarray(scales, np.float32)
        self.block_table = np.ascontiguousarray(block_table, np.int32)
        self.win_rows = np.ascontiguousarray(win_rows, np.uint8)
        self.win_scales = np.ascontiguousarray(win_scales, np.float32)
        self.kscale = None if kscale is None else np.ascontiguousarray(kscale, np.float32)
        kdt = np.uint8 if kscale is not None else np.uint16
        self.kidx = None if kidx is None else np.ascontiguousarray(kidx, kdt)
        self.n_win = self.win_scales.shape[-1]
        self.bt_stride = self.block_table.shape[-1]

    def gather_set(self, slot, L, sel=None):
        """Decoded attention set (selected or all visible entries, then window)."""
        nv = n_visible(L, self.m)
        cap = (len(sel) if sel is not None else nv) + self.n_win
        out = np.zeros((max(cap, 1), self.D))
        s = None if sel is None else np.ascontiguousarray(sel, np.int32)
        n = lib().csla_orc_gather_set(
            _p(self.rows, ctypes.c_uint8), _p(self.scales, ctypes.c_float),
            _p(self.block_table, ctypes.c_int32), self.bt_stride, _p(self.win_rows, ctypes.c_uint8),
            _p(self.win_scales, ctypes.c_float), self.n_win, int(slot), int(L), self.m, self.D,
            self.d_rope, None if s is None else _p(s, ctypes.c_int32), 0 if s is None else len(s),
            _p(out, ctypes.c_double))
        return out[:n]

    def gather_keys(self, slot, N):
        keys = np.zeros((max(N, 1), self.dI))
        lib().csla_orc_gather_keys(self.kidx.ctypes.data, self._kscale_p(), _p(self.block_table, ctypes.c_int32),
                                   self.bt_stride, int(slot), int(N), self.m, self.dI,
                                   _p(keys, ctypes.c_double))
        return keys[:N]

    def _kscale_p(self):
        return None if self.kscale is None else _p(self.kscale, ctypes.c_float)


def csa_decode(cv: CacheView, slots, lens, q, gamma_q, cq, W, head_w, sink, HI, k, eps=1e-6,
               theta=10000.0):
    """Whole CSA decode step for B requests (fp64).  Returns (idx [B,k], out [B,H,D])."""
    slots = np.ascontiguousarray(slots, np.int32)
    lens = np.ascontiguousarray(lens, np.int32)
    q, g, cq, W, hw, sink = _d(q), _d(gamma_q), _d(cq), _d(W), _d(head_w), _d(sink)
    B, H, D = q.shape
    dc = cq.shape[-1]
    idx = np.zeros((B, k), np.int32)
    out = np.zeros((B, H, D))
    lib().csla_orc_csa_decode(
        _p(cv.rows, ctypes.c_uint8), _p(cv.scales, ctypes.c_float), cv.kidx.ctypes.data, cv._kscale_p(),
        _p(cv.block_table, ctypes.c_int32), cv.bt_stride, _p(cv.win_rows, ctypes.c_uint8),
        _p(cv.win_scales, ctypes.c_float), cv.n_win, _p(slots, ctypes.c_int32),
        _p(lens, ctypes.c_int32), B, cv.m, H, D, cv.d_rope, HI, cv.dI, dc, k, eps, theta,
        _p(q, ctypes.c_double), _p(g, ctypes.c_double), _p(cq, ctypes.c_double),
        _p(W, ctypes.c_double), _p(hw, ctypes.c_double), _p(sink, ctypes.c_double),
        _p(idx, ctypes.c_int32), _p(out, ctypes.c_double))
    return idx, out


def hca_decode(cv: CacheView, slots, lens, q, gamma_q, sink, eps=1e-6, theta=10000.0):
    slots = np.ascontiguousarray(slots, np.int32)
    lens = np.ascontiguousarray(lens, np.int32)
    q, g, sink = _d(q), _d(gamma_q), _d(sink)
    B, H, D = q.shape
    out = np.zeros((B, H, D))
    lib().csla_orc_hca_decode(
        _p(cv.rows, ctypes.c_uint8), _p(cv.scales, ctypes.c_float), _p(cv.block_table, ctypes.c_int32),
        cv.bt_stride, _p(cv.win_rows, ctypes.c_uint8), _p(cv.win_scales, ctypes.c_float), cv.n_win,
        _p(slots, ctypes.c_int32), _p(lens, ctypes.c_int32), B, cv.m, H, D, cv.d_rope, eps, theta,
        _p(q, ctypes.c_double), _p(g, ctypes.c_double), _p(sink, ctypes.c_double),
        _p(out, ctypes.c_double))
    return out


def num_threads():
    return int(lib().csla_orc_num_threads())


# ---------------------------------------------------------------- expected state after appends
_encode_key_e4m3 = key_e4m3   # the flag argument below shadows the name


def expected_append(raw_kv, raw_idx, L0, L1, m, gamma_kv, wg, gb, wgi=None, gbi=None, eps=1e-6,
                    theta=10000.0, d_rope=64, window_from=0, key_e4m3=False, per_channel=False):
    """Rows the state and classical caches must hold after tokens L0..L1-1 of a
    request are appended (raw_kv/raw_idx hold the whole token history 0..L1-1).

    Returns dict: window {pos: (row, scale)}, entries {b: (row, scale)},
    keys {b: bf16 key, or (E4M3 codes, scale) with key_e4m3} for every block
    completed by these tokens.  Window rows are produced for positions >=
    window_from only.  per_channel: the per-channel gate (gb, gbi are
    [m][width] biases).
    """
    out = {"window": {}, "entries": {}, "keys": {}}
    for p in range(max(L0, window_from), L1):
        out["window"][p] = window_row(raw_kv[p], gamma_kv, p, eps, theta, d_rope)
    for b in range(L0 // m, L1 // m):
        if (b + 1) * m <= L0:
            continue
        xs = raw_kv[b * m:(b + 1) * m]
        if per_channel:
            out["entries"][b] = compressed_row_channel(xs, wg, gb, gamma_kv, b, eps, theta, d_rope)
        else:
            out["entries"][b] = compressed_row(xs, wg, gb, gamma_kv, b, eps, theta, d_rope)
        if raw_idx is not None and wgi is not None:
            xi = raw_idx[b * m:(b + 1) * m]
            if per_channel:
                c = gate_pool_channel(xi, wgi, gbi)
                out["keys"][b] = _encode_key_e4m3(c) if key_e4m3 else key_bf16(c)
            else:
                out["keys"][b] = index_key_e4m3(xi, wgi, gbi) if key_e4m3 else index_key(xi, wgi, gbi)
    return out
