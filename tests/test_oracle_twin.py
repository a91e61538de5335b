"""Two-oracle agreement: the C oracle against the separately written numpy
transcription (oracle/twin.py, codecs from ml_dtypes), on a tiny CSA and a
tiny HCA layer with a scattered page table."""
import dataclasses

import numpy as np

import oracle
from oracle import twin
from csla_synth.workloads import CSA_TINY, layer_params, step_inputs, token_stream
from helpers import oracle_cache

W_CSA = dataclasses.replace(CSA_TINY, L=300, B=2, name="twin_csa")
W_HCA = dataclasses.replace(CSA_TINY, L=300, B=3, m=128, HI=0, dI=0, dc=0, k=0, name="twin_hca")


def test_rows_bytes_agree():
    w = W_CSA
    p = layer_params(w)
    ts = token_stream(w, 0, 0, 40)
    for pos in range(0, 40, 3):
        r1, s1 = oracle.window_row(ts["kv"][pos], p["gamma_kv"], pos)
        r2, s2 = twin.window_row(ts["kv"][pos], p["gamma_kv"], pos)
        assert s1 == s2 and np.array_equal(r1, r2)
    for b in range(10):
        xs = ts["kv"][b * 4:(b + 1) * 4]
        r1, s1 = oracle.compressed_row(xs, p["wg"], p["gb"], p["gamma_kv"], b)
        r2, s2 = twin.compressed_row(xs, p["wg"], p["gb"], p["gamma_kv"], b)
        assert s1 == s2 and np.array_equal(r1, r2)
        k1 = oracle.index_key(ts["idx"][b * 4:(b + 1) * 4], p["wgi"], p["gbi"])
        k2 = twin.index_key(ts["idx"][b * 4:(b + 1) * 4], p["wgi"], p["gbi"])
        assert np.array_equal(k1, k2)


def _twin_set(cv, slot, L, sel):
    """Twin decoding of the attention set straight from the page table."""
    epp = 128 // cv.m
    out = []
    ids = [b for b in sel if b >= 0] if sel is not None else range(L // cv.m)
    for b in ids:
        pg = cv.block_table[slot, b // epp]
        out.append(twin.dequantize(cv.rows[pg, b % epp], cv.scales[pg, b % epp], cv.D))
    for pos in range(max(0, L - cv.n_win), L):
        out.append(twin.dequantize(cv.win_rows[slot, pos % cv.n_win], cv.win_scales[slot, pos % cv.n_win],
                                   cv.D))
    return np.stack(out)


def test_csa_decode_step_agrees():
    w = W_CSA
    lens = [300, 37]
    cv, p = oracle_cache(w, lens)
    si = step_inputs(w, 0)
    idx, out = oracle.csa_decode(cv, [0, 1], lens, si["q"], p["gamma_q"], si["cq"], p["W_iq"],
                                 si["head_w"], p["sink"], w.HI, w.k)
    for s, L in enumerate(lens):
        nv = L // w.m
        epp = 128 // w.m
        keys = np.stack([cv.kidx[cv.block_table[s, b // epp], b % epp] for b in range(nv)]) \
            .astype(np.uint32) << 16
        keys = keys.view(np.float32).astype(np.float64)
        sc = twin.scores(si["cq"][s], p["W_iq"], si["head_w"][s], keys, w.HI, w.dI)
        tk = twin.topk(sc, w.k)
        assert np.array_equal(tk, idx[s])
        rows = _twin_set(cv, s, L, tk)
        o, _ = twin.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"])
        assert np.allclose(o, out[s], rtol=0, atol=1e-12)


def test_hca_decode_step_agrees_and_equals_csa_with_full_topk():
    w = W_HCA
    lens = [300, 129, 5]
    cv, p = oracle_cache(w, lens)
    si = step_inputs(w, 1)
    out = oracle.hca_decode(cv, [0, 1, 2], lens, si["q"], p["gamma_q"], p["sink"])
    for s, L in enumerate(lens):
        rows = _twin_set(cv, s, L, None)
        o, _ = twin.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"])
        assert np.allclose(o, out[s], rtol=0, atol=1e-12)
        # HCA == attention over "top-k covering every visible entry"
        allsel = np.arange(L // w.m, dtype=np.int32)
        o2, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, cv.gather_set(s, L, allsel), p["sink"])
        assert np.allclose(o2, out[s], atol=1e-13)
