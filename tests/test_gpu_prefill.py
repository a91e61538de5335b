"""GPU parity of query rows other than each request's latest token (a
prefill chunk's queries): per-row visible lengths in the indexer, top-k and
attention; window rows read from a chunk buffer; the compressor's token-row
output and the ring snapshot that fill that buffer.

A prefill query at position t sees what a decode step at t would see
(causal visibility of blocks and of the window), so every expected value is
the decode oracle evaluated at that query's own position."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import CompressParams, LayerBuffers
from csla_synth import normal, permutation
from csla_synth.workloads import CSA_PREFILL, HCA_DECODE, layer_params, prefill_inputs, token_stream
from gpu_helpers import (DEV, act_tensor, append, assert_no_device_error, check_out, check_scores,
                         compare_rows, shape_of, upload_layer)
from helpers import block_table, oracle_cache

pytestmark = pytest.mark.gpu

SMALL = dataclasses.replace(CSA_PREFILL, B=1, L=1500, H=16, k=64, name="prefill_small")
HCA_P = dataclasses.replace(HCA_DECODE, B=1, L=3000, H=16, name="prefill_hca")
NW = 127   # window rows from before the chunk that its first query needs


def _i32(x):
    return torch.as_tensor(np.asarray(x, np.int32), device=DEV)


def _f32(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


def prefix_layer(w, L0, L1):
    """Layer whose block table covers L1 tokens, with tokens 0..L0-1 appended."""
    p = layer_params(w)
    bt, n_pages = block_table(w, [L1], 1)
    lb = LayerBuffers(shape_of(w), 1, n_pages, bt.shape[1], DEV)
    lb.block_table.copy_(torch.from_numpy(bt))
    cp = CompressParams(p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"), DEV)
    ts = token_stream(w, 0, 0, L1)
    if L0:
        append(w, lb, cp, 0, ts, 0, L0)
    return lb, cp, p, ts


def window_source(w, ts, p, L0, L1):
    """The oracle's window rows of positions L0-NW .. L1-1 (zero rows before 0)."""
    rb = oracle.row_bytes(w.D, w.d_rope)
    rows = np.zeros((NW + L1 - L0, rb), np.uint8)
    sc = np.zeros(NW + L1 - L0, np.float32)
    for i in range(NW + L1 - L0):
        pos = L0 - NW + i
        if pos >= 0:
            rows[i], sc[i] = oracle.window_row(ts["kv"][pos], p["gamma_kv"], pos, w.eps, w.theta, w.d_rope)
    return rows, sc


@pytest.mark.parametrize("w,L0,T", [(SMALL, 1000, 500), (SMALL, 50, 40), (SMALL, 0, 300), (SMALL, 200, 1),
                                    (HCA_P, 2000, 700)])
def test_chunk_window_rows(w, L0, T):
    """csla_window_rows (the NW rows before the chunk) + the token-row output
    of csla_compress_append (the chunk's T rows) = the oracle's window rows of
    positions L0-NW .. L0+T-1; the ring afterwards holds the same bytes."""
    L1 = L0 + T
    lb, cp, p, ts = prefix_layer(w, L0, L1)
    rb = oracle.row_bytes(w.D, w.d_rope)
    rows = torch.full((NW + T, rb), 0xEE, dtype=torch.uint8, device=DEV)
    sc = torch.full((NW + T,), float("nan"), dtype=torch.float32, device=DEV)
    slots = _i32([0])
    C.csla_window_rows(lb.cfg(), lb.state(), slots, 1, NW, rows, sc, NW + T)
    kv = act_tensor(w, ts["kv"][L0:L1])
    ki = act_tensor(w, ts["idx"][L0:L1]) if w.is_csa else None
    C.csla_compress_append(lb.cfg(), lb.state(), lb.cache(), slots, 1, T, kv, ki,
                           C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32, cp.struct(),
                           tok=C.token_rows(rows, sc, NW + T, NW))
    assert_no_device_error()
    got, gsc = rows.cpu().numpy(), sc.cpu().numpy()
    h = lb.host_view()
    assert h["len"][0] == L1
    for i in range(NW + T):
        pos = L0 - NW + i
        if pos < 0:
            assert not got[i].any() and gsc[i] == 0.0, pos
            continue
        y = oracle.rope(oracle.rmsnorm(ts["kv"][pos], p["gamma_kv"], w.eps), pos, w.theta, w.d_rope)
        compare_rows(got[i], gsc[i], y, w.D, w.d_rope)
        if pos >= L1 - w.n_win:
            assert np.array_equal(h["win_rows"][0, pos % w.n_win], got[i]), pos
            assert h["win_scales"][0, pos % w.n_win] == gsc[i], pos


def _queries(L0, T):
    return np.arange(L0 + 1, L0 + T + 1, dtype=np.int32)


@pytest.mark.parametrize("L0,T,one", [(1000, 500, False), (1000, 503, True), (37, 44, True)])
def test_indexer_query_rows(L0, T, one):
    """one: the rows are flagged as one request's queries, so several rows
    share each key tile (a group that does not divide T included)."""
    w = SMALL
    L1 = L0 + T
    cv, p = oracle_cache(w, [L1])
    lb = upload_layer(w, cv, [L1])
    pi = prefill_inputs(w, T, tag=1)
    q_len = _queries(L0, T)
    stride = L1 // w.m
    scores = torch.full((T, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(lb.cfg(), C.CSLA_OP_INDEXER, T, L1)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    ql = _i32(q_len)
    C.csla_indexer_scores(lb.cfg(), lb.state(), lb.cache(), _i32(np.zeros(T)), T, L1, act_tensor(w, pi["cq"]), dt,
                          act_tensor(w, p["W_iq"]), dt, _f32(pi["head_w"]), scores, stride, ws, wsb,
                          qs=C.queries(ql, one_request=one))
    assert_no_device_error()
    got = scores.cpu().numpy()
    keys = cv.gather_keys(0, L1 // w.m)
    for i in range(T):
        nv = int(q_len[i]) // w.m
        qI = oracle.index_query(pi["cq"][i], p["W_iq"], w.HI, w.dI)
        check_scores(got[i, :nv].astype(np.float64), oracle.index_scores(qI, pi["head_w"][i], keys[:nv]))
        assert np.all(np.isnan(got[i, nv:])), i


@pytest.mark.parametrize("L0,T,k", [(1000, 300, 64), (150000, 40, 1024)])
def test_topk_query_rows(L0, T, k):
    """Exact on given fp32 scores: row i ranks only its first q_len[i]/m."""
    L1 = L0 + T
    stride = L1 // 4
    sc = np.stack([normal(7, "ptopk/%d/%d" % (L0, i), (stride,)) for i in range(T)]).astype(np.float32)
    lb = LayerBuffers(shape_of(SMALL), 1, 1, 1, DEV)
    lb.len.copy_(torch.tensor([L1], dtype=torch.int32))
    q_len = _queries(L0, T)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    C.csla_topk_select(lb.cfg(), lb.state(), _i32(np.zeros(T)), T, L1, _f32(sc), stride, k, idx,
                       qs=C.queries(_i32(q_len)))
    assert_no_device_error()
    got = idx.cpu().numpy()
    for i in range(T):
        n = int(q_len[i]) // 4
        assert np.array_equal(got[i], oracle.topk(sc[i, :n].astype(np.float64), k)), i


def _selection(w, q_len, tag):
    """A seeded valid top-k list per row: min(k, nv) distinct ascending
    entries below the row's visible count, padded with -1."""
    out = -np.ones((len(q_len), w.k), np.int32)
    for i, L in enumerate(q_len):
        nv = int(L) // w.m
        if nv:
            sel = np.sort(permutation(w.seed, "psel/%d/%d" % (tag, i), nv)[:min(w.k, nv)])
            out[i, :len(sel)] = sel
    return out


def _attend_rows(w, lb, qs, q, p, T, L1, idx=None, variant=C.CSLA_VARIANT_AUTO):
    cfg = lb.cfg()
    out = torch.full((T, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)
    slots = _i32(np.zeros(T))
    if idx is not None:
        wsb = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, T, w.k)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=DEV)
        C.csla_csa_attend(cfg, lb.state(), lb.cache(), slots, T, q, C.CSLA_BF16, idx, w.k, _f32(p["sink"]),
                          _f32(p["gamma_q"]), out, C.CSLA_F32, variant, ws, wsb, qs=qs)
    else:
        wsb = C.csla_workspace_size(cfg, C.CSLA_OP_HCA_ATTEND, T, L1)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=DEV)
        C.csla_hca_attend(cfg, lb.state(), lb.cache(), slots, T, L1, q, C.CSLA_BF16, _f32(p["sink"]),
                          _f32(p["gamma_q"]), out, C.CSLA_F32, variant, ws, wsb, qs=qs)
    return out


def _oracle_rows(w, cv, src_rows, src_sc, L0, L, sel):
    """Decoded set of the query at position L-1: its window rows come from
    the chunk buffer, placed in the view's ring at position % n_win."""
    for pos in range(max(0, L - w.n_win), L):
        cv.win_rows[0, pos % w.n_win] = src_rows[pos - L0 + NW]
        cv.win_scales[0, pos % w.n_win] = src_sc[pos - L0 + NW]
    return cv.gather_set(0, L, sel)


@pytest.mark.parametrize("w,L0,T", [(SMALL, 1000, 300), (SMALL, 30, 200), (HCA_P, 2000, 300)])
def test_attend_query_rows_with_window_source(w, L0, T):
    L1 = L0 + T
    cv, raws, p = oracle_cache(w, [L1], with_raw=True)
    lb = upload_layer(w, cv, [L1])
    src_rows, src_sc = window_source(w, raws[0], p, L0, L1)
    q_len = _queries(L0, T)
    base = np.full(T, NW - L0, np.int32)
    keep = [_i32(q_len), torch.from_numpy(src_rows).to(DEV), _f32(src_sc), _i32(base)]
    qs = C.queries(keep[0], keep[1], keep[2], keep[3], NW + T)
    pi = prefill_inputs(w, T, tag=2)
    q = act_tensor(w, pi["q"])
    idx_np = _selection(w, q_len, L0) if w.is_csa else None
    idx = _i32(idx_np) if w.is_csa else None
    outs = {v: _attend_rows(w, lb, qs, q, p, T, L1, idx, v)
            for v in (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED)}
    assert_no_device_error()
    assert torch.equal(outs[1], outs[2]), "variants differ"
    got = outs[1].cpu().numpy().astype(np.float64)
    for i in range(T):
        L = int(q_len[i])
        rows = _oracle_rows(w, cv, src_rows, src_sc, L0, L, idx_np[i] if w.is_csa else None)
        ref, _ = oracle.attend(pi["q"][i], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
        check_out(got[i], ref)


@pytest.mark.parametrize("L1,q_len", [(1400, [1400, 1400, 1400]), (120, [120, 60, 1, 119])])
def test_attend_query_rows_from_ring(L1, q_len):
    """Without a window source the rows read the ring: several queries at the
    latest position, or any position while the whole history fits the ring."""
    w = SMALL
    cv, p = oracle_cache(w, [L1])
    lb = upload_layer(w, cv, [L1])
    q_len = np.array(q_len, np.int32)
    T = len(q_len)
    pi = prefill_inputs(w, T, tag=3)
    idx_np = _selection(w, q_len, 99)
    out = _attend_rows(w, lb, C.queries(_i32(q_len)), act_tensor(w, pi["q"]), p, T, L1, _i32(idx_np))
    assert_no_device_error()
    got = out.cpu().numpy().astype(np.float64)
    for i in range(T):
        L = int(q_len[i])
        ref, _ = oracle.attend(pi["q"][i], p["gamma_q"], L - 1, cv.gather_set(0, L, idx_np[i]), p["sink"], w.eps,
                               w.theta, w.d_rope)
        check_out(got[i], ref)


def test_query_row_errors_are_recorded_not_trapped():
    """q_len above the request's length -> CSLA_DEVERR_LEN; a window position
    that left the ring, or one outside the window source -> CSLA_DEVERR_INDEX.
    Every access stays inside its buffer: the kernels skip such rows."""
    w = SMALL
    L1 = 1400
    cv, p = oracle_cache(w, [L1])
    lb = upload_layer(w, cv, [L1])
    pi = prefill_inputs(w, 2, tag=4)
    q = act_tensor(w, pi["q"])
    idx = _i32(_selection(w, [L1, L1], 5))
    _attend_rows(w, lb, C.queries(_i32([L1 + 1, L1])), q, p, 2, L1, idx)
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits & C.CSLA_DEVERR_LEN
    _attend_rows(w, lb, C.queries(_i32([L1 - 200, L1])), q, p, 2, L1, idx)
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits & C.CSLA_DEVERR_INDEX
    rb = oracle.row_bytes(w.D, w.d_rope)
    src = torch.zeros((128, rb), dtype=torch.uint8, device=DEV)
    ssc = torch.ones(128, dtype=torch.float32, device=DEV)
    keep = [_i32([L1, L1]), _i32([128 - L1, 0])]   # row 0: rows 0..127; row 1: past the buffer's end
    qs = C.queries(keep[0], src, ssc, keep[1], 128)
    _attend_rows(w, lb, qs, q, p, 2, L1, idx)
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits & C.CSLA_DEVERR_INDEX


def test_indexer_one_request_rows_with_another_slot():
    """A row flagged as part of one request but naming another slot is
    skipped (its scores stay untouched) and CSLA_DEVERR_INDEX is recorded;
    the other rows are scored as usual."""
    w = SMALL
    lens = [900, 900]
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    T = 6
    pi = prefill_inputs(w, T, tag=5)
    q_len = np.array([400, 500, 600, 700, 800, 900], np.int32)
    slots = np.array([0, 0, 1, 0, 0, 0], np.int32)
    stride = 900 // w.m
    scores = torch.full((T, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(lb.cfg(), C.CSLA_OP_INDEXER, T, 900)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    C.csla_indexer_scores(lb.cfg(), lb.state(), lb.cache(), _i32(slots), T, 900, act_tensor(w, pi["cq"]), dt,
                          act_tensor(w, p["W_iq"]), dt, _f32(pi["head_w"]), scores, stride, ws, wsb,
                          qs=C.queries(_i32(q_len), one_request=True))
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits == C.CSLA_DEVERR_INDEX
    got = scores.cpu().numpy()
    keys = cv.gather_keys(0, 900 // w.m)
    for i in range(T):
        if slots[i] != 0:
            assert np.all(np.isnan(got[i])), i
            continue
        nv = int(q_len[i]) // w.m
        qI = oracle.index_query(pi["cq"][i], p["W_iq"], w.HI, w.dI)
        check_scores(got[i, :nv].astype(np.float64), oracle.index_scores(qI, pi["head_w"][i], keys[:nv]))
