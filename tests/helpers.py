"""Test-side assembly: expected cache contents built by the oracle from the
seeded token streams, in the library's byte layout (include/csla.h)."""
import numpy as np

import oracle
from csla_synth import permutation
from csla_synth.workloads import Workload, layer_params, token_stream

PAGE = oracle.PAGE_TOKENS


def block_table(w: Workload, lens, n_slots, seed_name="bt"):
    """A scattered page assignment: every slot gets enough pages for its
    length; physical page ids are a seeded permutation (never contiguous)."""
    need = [-(-int(L) // PAGE) for L in lens]
    bt_stride = max(max(need), 1)
    total = sum(need)
    perm = permutation(w.seed, seed_name, max(total, 1))
    bt = -np.ones((n_slots, bt_stride), np.int32)
    k = 0
    for s, n in enumerate(need):
        bt[s, :n] = perm[k:k + n]
        k += n
    return bt, max(total, 1)


def oracle_cache(w: Workload, lens, params=None, with_raw=False, stream_ids=None, bt=None):
    """Expected cache of len(lens) requests (slot i = request i, whose token
    stream is stream_ids[i], default i) after their whole token streams
    0..L_i-1 were appended, computed by the oracle.  bt: a given block table
    (pages 0..max id), else a seeded one of the layer's own."""
    p = params or layer_params(w)
    n_slots = len(lens)
    if bt is None:
        bt, n_pages = block_table(w, lens, n_slots)
    else:
        n_pages = int(bt.max()) + 1
    epp = PAGE // w.m
    rb = oracle.row_bytes(w.D, w.d_rope)
    rows = np.zeros((n_pages, epp, rb), np.uint8)
    scales = np.zeros((n_pages, epp), np.float32)
    e4m3 = w.is_csa and w.key_fmt == 1
    kidx = np.zeros((n_pages, epp, max(w.dI, 1)), np.uint8 if e4m3 else np.uint16) if w.is_csa else None
    kscale = np.zeros((n_pages, epp), np.float32) if e4m3 else None
    win_rows = np.zeros((n_slots, w.n_win, rb), np.uint8)
    win_scales = np.zeros((n_slots, w.n_win), np.float32)
    raws = []
    for s, L in enumerate(lens):
        ts = token_stream(w, s if stream_ids is None else stream_ids[s], 0, L)
        raws.append(ts)
        exp = oracle.expected_append(ts["kv"], ts.get("idx"), 0, L, w.m, p["gamma_kv"], p["wg"],
                                     p["gb"], p.get("wgi"), p.get("gbi"), w.eps, w.theta, w.d_rope,
                                     window_from=L - w.n_win, key_e4m3=e4m3,
                                     per_channel=w.gate == 1)
        for pos, (r, sc) in exp["window"].items():
            if pos >= L - w.n_win:
                win_rows[s, pos % w.n_win] = r
                win_scales[s, pos % w.n_win] = sc
        for b, (r, sc) in exp["entries"].items():
            pg = bt[s, b // epp]
            rows[pg, b % epp] = r
            scales[pg, b % epp] = sc
            if e4m3:
                kidx[pg, b % epp], kscale[pg, b % epp] = exp["keys"][b]
            elif w.is_csa:
                kidx[pg, b % epp] = exp["keys"][b]
    cv = oracle.CacheView(w.m, w.D, rows, scales, bt, win_rows, win_scales, kidx, w.dI, w.d_rope, kscale=kscale)
    return (cv, raws, p) if with_raw else (cv, p)
