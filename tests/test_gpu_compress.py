"""GPU parity: csla_compress_append against the oracle (window rows,
compressed entries, index keys, tail and length), decode (one token per
call) and multi-token appends, CSA (m=4) and HCA (m=128)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from csla_synth.workloads import CSA_DECODE, CSA_TINY, HCA_DECODE, layer_params, token_stream
from gpu_helpers import assert_bf16_close, assert_no_device_error, build_layer, compare_rows

pytestmark = pytest.mark.gpu


def _check_layer(w, lb, p, lens):
    h = lb.host_view()
    epp = 128 // w.m
    tolerated = 0
    checked = 0
    for s, L in enumerate(lens):
        ts = token_stream(w, s, 0, L)
        assert h["len"][s] == L
        # window rows: the last min(L, n_win) positions
        for pos in range(max(0, L - w.n_win), L):
            y = oracle.rope(oracle.rmsnorm(ts["kv"][pos], p["gamma_kv"], w.eps), pos, w.theta, w.d_rope)
            ring = pos % w.n_win
            tolerated += compare_rows(h["win_rows"][s, ring], h["win_scales"][s, ring], y, w.D, w.d_rope)
            checked += 1
        # compressed entries
        for b in range(L // w.m):
            xs = ts["kv"][b * w.m:(b + 1) * w.m]
            if w.gate == 1:
                c = oracle.gate_pool_channel(xs, p["wg"], p["gb"])
            else:
                c, _ = oracle.gate_pool(xs, p["wg"], p["gb"])
            y = oracle.rope(oracle.rmsnorm(c, p["gamma_kv"], w.eps), b * w.m, w.theta, w.d_rope)
            pg = h["block_table"][s, b // epp]
            tolerated += compare_rows(h["rows"][pg, b % epp], h["scales"][pg, b % epp], y, w.D, w.d_rope)
            checked += 1
            if w.is_csa:
                xi = ts["idx"][b * w.m:(b + 1) * w.m]
                if w.gate == 1:
                    ref = oracle.key_bf16(oracle.gate_pool_channel(xi, p["wgi"], p["gbi"]))
                else:
                    ref = oracle.index_key(xi, p["wgi"], p["gbi"])
                got = h["kidx"][pg, b % epp]
                # fp32 gates and pooled sum: error well under 1e-5 of the largest input
                assert_bf16_close(got, ref, 1e-5 * float(np.max(np.abs(xi))))
        # tail: raw rows of the open block, exact fp32 copies
        for pos in range((L // w.m) * w.m, L):
            assert np.array_equal(h["tail_kv"][s, pos % w.m], ts["kv"][pos].astype(np.float32))
    # tolerated code flips must be rare
    assert tolerated <= max(2, checked * w.D // 2000), (tolerated, checked)


TINY = dataclasses.replace(CSA_TINY, L=700, name="compress_tiny")
HCA_SMALL = dataclasses.replace(HCA_DECODE, L=1000, name="compress_hca")
CSA_BIG = dataclasses.replace(CSA_DECODE, L=600, name="compress_csa512")


@pytest.mark.parametrize("w,lens,chunk", [
    (TINY, [700, 3, 129], None),          # one multi-token call per request
    (TINY, [263], 37),                    # ragged multi-token calls over open tails
    (CSA_BIG, [600, 77], 64),
    (HCA_SMALL, [1000, 128, 255], 200),
    (HCA_SMALL, [300], 1),                # decode: one token per call
    (dataclasses.replace(TINY, gate=1), [700, 3, 129], None),      # per-channel gate
    (dataclasses.replace(CSA_BIG, gate=1), [600, 77], 1),
    (dataclasses.replace(HCA_SMALL, gate=1), [1000, 128, 255], 200),
    (dataclasses.replace(HCA_SMALL, gate=1), [300], 1),
])
def test_compress_append_matches_oracle(w, lens, chunk):
    lb, cp, p = build_layer(w, lens, chunk=chunk)
    assert_no_device_error()
    _check_layer(w, lb, p, lens)


def test_compress_decode_path_equals_multi_token_path():
    """T=1 calls and one long call must leave bit-identical caches."""
    w = dataclasses.replace(CSA_DECODE, L=300, name="compress_paths")
    a, _, _ = build_layer(w, [300], chunk=1)
    b, _, _ = build_layer(w, [300], chunk=None)
    ha, hb = a.host_view(), b.host_view()
    for k in ("rows", "scales", "kidx", "win_rows", "win_scales", "len"):
        assert np.array_equal(ha[k], hb[k]), k
    assert np.array_equal(ha["tail_kv"][0, :300 % 4], hb["tail_kv"][0, :300 % 4])
