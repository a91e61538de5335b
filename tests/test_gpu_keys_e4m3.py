"""GPU parity of the E4M3 index-key storage (haiqwa "DeepSeek-V4"
§FP4精度加速: the indexer's key path in low precision; csla_cfg.key_fmt =
CSLA_KEY_E4M3): the compressor's codes and power-of-two scales against the
oracle's quantiser, the indexer's scores on E4M3 keys (decode rows and the
query rows of one request) against the oracle's scores on the same decoded
keys, and a whole CSA decode step (indexer, top-k, attention) against the
oracle's step."""
import dataclasses

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from csla_synth.workloads import CSA_DECODE, CSA_TINY, step_inputs, token_stream
from gpu_helpers import (DEV, act_tensor, assert_no_device_error, build_layer, check_out, check_scores,
                         near_midpoint, upload_layer)
from helpers import oracle_cache

pytestmark = pytest.mark.gpu

E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
FINITE = np.sort(np.unique(np.abs(E4M3[np.isfinite(E4M3)])))
MIDS = 0.5 * (FINITE[1:] + FINITE[:-1])


def compare_key_e4m3(codes, scale, key32):
    """GPU codes/scale of one entry against the oracle's fp32 key: the scale
    must be the oracle's (unless max |key| sits within 1e-6 of a boundary
    448*2^e, where the two fp32 poolings may fall on either side), and each
    code must be the oracle's except where key/scale lies within 1e-5 of an
    E4M3 rounding midpoint (then one step either way)."""
    amax = float(np.max(np.abs(key32)))
    s_ref = oracle.key_scale_e4m3(amax)
    if scale != s_ref:
        b = 448.0 * min(scale, s_ref)
        assert abs(amax - b) <= 1e-6 * b and max(scale, s_ref) == 2 * min(scale, s_ref), (scale, s_ref, amax)
        return 0
    v = key32.astype(np.float64) / scale
    ref = np.array([oracle.e4m3_from_f32(x) for x in v.astype(np.float32)], np.uint8)
    diff = np.nonzero(codes != ref)[0]
    for d in diff:
        a = abs(v[d])
        i = np.clip(np.searchsorted(MIDS, a), 1, len(MIDS) - 1)
        near = min(abs(a - MIDS[i - 1]), abs(a - MIDS[i])) <= 1e-5 * max(a, 2.0 ** -9)
        assert near, (d, codes[d], ref[d], v[d])
    return len(diff)


KEYS = dataclasses.replace(CSA_DECODE, L=900, key_fmt=1, name="keys_e4m3")
# E4M3 keys are scored by kind::f8f6f4 MMAs at dI = 128 (the tiny shape with 128-dim keys)
KEYS_TINY = dataclasses.replace(CSA_TINY, L=700, dI=128, key_fmt=1, name="keys_e4m3_tiny")


@pytest.mark.parametrize("w,lens,chunk", [(KEYS, [900, 133], 64), (KEYS_TINY, [700, 9], None), (KEYS, [90], 1)])
def test_compressor_writes_oracle_codes_and_scales(w, lens, chunk):
    lb, cp, p = build_layer(w, lens, chunk=chunk)
    assert_no_device_error()
    h = lb.host_view()
    epp = 128 // w.m
    flips = checked = 0
    for s, L in enumerate(lens):
        ts = token_stream(w, s, 0, L)
        for b in range(L // w.m):
            xi = ts["idx"][b * w.m:(b + 1) * w.m]
            c, _ = oracle.gate_pool(xi, p["wgi"], p["gbi"])
            pg = h["block_table"][s, b // epp]
            flips += compare_key_e4m3(h["kidx"][pg, b % epp], float(h["kscale"][pg, b % epp]),
                                      c.astype(np.float32))
            checked += w.dI
    assert flips <= max(2, checked // 2000), (flips, checked)


def _scores(w, lb, si, p, slots, max_len, qs=None):
    B = len(slots)
    cfg = lb.cfg()
    stride = max_len // w.m
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, max_len)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    C.csla_indexer_scores(cfg, lb.state(), lb.cache(), torch.as_tensor(slots, dtype=torch.int32, device=DEV), B,
                          max_len, act_tensor(w, si["cq"][:B]), dt, act_tensor(w, p["W_iq"]), dt,
                          torch.as_tensor(si["head_w"][:B], dtype=torch.float32, device=DEV), scores, stride, ws, wsb,
                          qs=qs)
    return scores.cpu().numpy()


@pytest.mark.parametrize("w,lens", [
    (dataclasses.replace(CSA_TINY, B=3, L=2048, dI=128, key_fmt=1, name="idx8_tiny"), [2048, 515, 3]),
    (dataclasses.replace(CSA_TINY, B=2, L=2048, dI=128, HI=8, key_fmt=1, name="idx8_hi8"), [2048, 700]),
    (dataclasses.replace(CSA_DECODE, B=2, L=5000, key_fmt=1, name="idx8_big"), [5000, 1113]),
])
def test_indexer_on_e4m3_keys_matches_oracle(w, lens):
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 41)
    got = _scores(w, lb, si, p, list(range(len(lens))), max(lens))
    assert_no_device_error()
    for s, L in enumerate(lens):
        nv = L // w.m
        if nv:
            qI = oracle.index_query(si["cq"][s], p["W_iq"], w.HI, w.dI)
            ref = oracle.index_scores(qI, si["head_w"][s], cv.gather_keys(s, nv))
            check_scores(got[s, :nv].astype(np.float64), ref)
        assert np.all(np.isnan(got[s, nv:]))


@pytest.mark.parametrize("HI", [16, 4])
def test_indexer_query_rows_of_one_request_on_e4m3_keys(HI):
    """Query rows of one request with their own visible lengths: several rows
    share each key tile (the prefill path: 4 rows at 16 index heads, 16 at 4)."""
    w = dataclasses.replace(CSA_DECODE, B=7, L=3000, HI=HI, key_fmt=1, name="idx8_rows%d" % HI)
    L = 3000
    cv, p = oracle_cache(w, [L])
    lb = upload_layer(w, cv, [L])
    q_len = np.array([1, 4, 777, 1500, 2999, 3000, 2000], np.int32)
    si = step_inputs(w, 42)
    qs = C.queries(torch.as_tensor(q_len, device=DEV), one_request=True)
    got = _scores(w, lb, si, p, [0] * len(q_len), L, qs=qs)
    assert_no_device_error()
    for i, Lq in enumerate(q_len):
        nv = int(Lq) // w.m
        if nv:
            qI = oracle.index_query(si["cq"][i], p["W_iq"], w.HI, w.dI)
            ref = oracle.index_scores(qI, si["head_w"][i], cv.gather_keys(0, nv))
            check_scores(got[i, :nv].astype(np.float64), ref)
        assert np.all(np.isnan(got[i, nv:]))


def test_decode_step_on_e4m3_keys_matches_oracle():
    """Indexer -> top-k -> attention on E4M3 keys against the oracle's whole
    step; the top-k set equal except inside the 1e-4 band."""
    w = dataclasses.replace(CSA_DECODE, B=3, L=4000, key_fmt=1, name="step8")
    lens = [4000, 2222, 700]
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 43)
    B, ml = len(lens), max(lens)
    got = _scores(w, lb, si, p, list(range(B)), ml)
    cfg = lb.cfg()
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    sc = torch.as_tensor(got, device=DEV).contiguous()
    idx = torch.zeros((B, w.k), dtype=torch.int32, device=DEV)
    C.csla_topk_select(cfg, lb.state(), slots, B, ml, sc, sc.shape[1], w.k, idx)
    out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)
    wsa = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, w.k)
    wa = torch.zeros(wsa, dtype=torch.uint8, device=DEV)
    C.csla_csa_attend(cfg, lb.state(), lb.cache(), slots, B, act_tensor(w, si["q"][:B]), C.CSLA_BF16, idx, w.k,
                      torch.as_tensor(p["sink"], dtype=torch.float32, device=DEV),
                      torch.as_tensor(p["gamma_q"], dtype=torch.float32, device=DEV), out, C.CSLA_F32,
                      C.CSLA_VARIANT_AUTO, wa, wsa)
    assert_no_device_error()
    oidx, oout = oracle.csa_decode(cv, np.arange(B), lens, si["q"][:B], p["gamma_q"], si["cq"][:B], p["W_iq"],
                                   si["head_w"][:B], p["sink"], w.HI, w.k)
    gi = idx.cpu().numpy()
    gout = out.cpu().numpy().astype(np.float64)
    for s, L in enumerate(lens):
        nv = L // w.m
        qI = oracle.index_query(si["cq"][s], p["W_iq"], w.HI, w.dI)
        ref = oracle.index_scores(qI, si["head_w"][s], cv.gather_keys(s, nv))
        kth = np.sort(ref)[::-1][min(w.k, nv) - 1]
        sel = set(int(x) for x in gi[s] if x >= 0)
        assert set(np.nonzero(ref > kth + 1e-4)[0].tolist()) <= sel
        assert not (sel & set(np.nonzero(ref < kth - 1e-4)[0].tolist()))
        if set(oidx[s][oidx[s] >= 0].tolist()) == sel:
            check_out(gout[s], oout[s])
        else:   # a tie inside the band: attention over the GPU's set
            rows = cv.gather_set(s, L, gi[s])
            r2, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
            check_out(gout[s], r2)
