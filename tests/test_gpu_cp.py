"""Context-parallel prefill through the library on one GPU.  The R ranks run
one after another in one process (run_cp_prefill_local: the boundary sends
and the all-gather become tensor copies; no collective, and no kernel waits
on another rank's), each rank with its own full-size cache on its own
scattered block table.  After reassembly every rank's cache holds, byte for
byte, the entries of the same request prefilled in one piece (a one-rank
plan through the same calls), every rank's query outputs equal the one-piece
rows bit for bit, and sampled rows match the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.cp import LibRank, cp_plan, run_cp_prefill_local
from compressed_sparse_long_append_b200.layer import CompressParams, LayerBuffers
from csla_synth.workloads import CSA_DECODE, CSA_PREFILL, HCA_DECODE, layer_params, prefill_inputs, token_stream
from gpu_helpers import DEV, act_tensor, assert_no_device_error, cache_view, check_out, shape_of
from helpers import block_table

pytestmark = pytest.mark.gpu

CSA_CP = dataclasses.replace(CSA_PREFILL, B=1, L=1500, H=16, k=64, name="cp_csa")
CSA_CP8 = dataclasses.replace(CSA_DECODE, B=1, L=1500, H=16, k=64, key_fmt=1, gate=1, name="cp_csa8")
HCA_CP = dataclasses.replace(HCA_DECODE, B=1, L=1300, H=16, name="cp_hca")


def _f32(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


def _entries(w, lb, N):
    """Entry bytes of blocks 0 .. N/m-1 of slot 0, in block order."""
    h = lb.host_view()
    epp = 128 // w.m
    out = []
    for b in range(N // w.m):
        pg, e = h["block_table"][0, b // epp], b % epp
        t = (h["rows"][pg, e].tobytes(), h["scales"][pg, e].tobytes())
        if w.is_csa:
            t += (h["kidx"][pg, e].tobytes(),) + ((h["kscale"][pg, e].tobytes(),) if "kscale" in h else ())
        out.append(t)
    return out


def _run(w, plan, kv, ki, pin, p, seed_name):
    """Every rank of `plan`; returns (ranks, outputs per rank, top-k lists per rank)."""
    N = plan.N
    bt, n_pages = block_table(w, [N], 1, seed_name=seed_name)
    cp = CompressParams(p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"), DEV)
    ranks, kvs, kis = [], [], []
    for r in range(plan.R):
        lb = LayerBuffers(shape_of(w), 1, n_pages, bt.shape[1], DEV)
        # each rank its own page assignment
        lb.block_table.copy_(torch.from_numpy(np.roll(bt, r, axis=1) if r else bt))
        ranks.append(LibRank(plan, r, lb, cp, 0, DEV))
        p0, p1 = plan.rng(r)
        kvs.append(act_tensor(w, kv[p0:p1]))
        kis.append(act_tensor(w, ki[p0:p1]) if w.is_csa else None)
    run_cp_prefill_local(ranks, kvs, kis)
    outs, idxs = [], []
    for r, rk in enumerate(ranks):
        p0, p1 = plan.rng(r)
        T = p1 - p0
        out = torch.full((T, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)
        q = act_tensor(w, pin["q"][p0:p1])
        if w.is_csa:
            idx = torch.full((T, w.k), -7, dtype=torch.int32, device=DEV)
            rk.queries(q, _f32(p["sink"]), _f32(p["gamma_q"]), out, cq=act_tensor(w, pin["cq"][p0:p1]),
                       W_iq=act_tensor(w, p["W_iq"]), head_w=_f32(pin["head_w"][p0:p1]), k=w.k, q_chunk=512,
                       idx_out=idx)
            idxs.append(idx)
        else:
            rk.queries(q, _f32(p["sink"]), _f32(p["gamma_q"]), out, q_chunk=512)
            idxs.append(None)
        outs.append(out)
    torch.cuda.synchronize()
    assert_no_device_error()
    return ranks, outs, idxs


@pytest.mark.parametrize("w,R,starts", [
    (CSA_CP, 2, None),
    (CSA_CP, 3, [0, 400, 1001, 1500]),
    (CSA_CP8, 2, [0, 733, 1500]),
    (HCA_CP, 3, [0, 300, 811, 1300]),
    (dataclasses.replace(CSA_CP, L=10000, name="cp_csa10k"), 4, [0, 2501, 4999, 7777, 10000]),
    (dataclasses.replace(HCA_CP, L=6000, name="cp_hca6k"), 4, None),
])
def test_cp_prefill_equals_one_piece(w, R, starts):
    N = w.L
    p = layer_params(w)
    ts = token_stream(w, 0, 0, N)
    kv, ki = ts["kv"], ts.get("idx")
    pin = prefill_inputs(w, N, tag=9)
    one, one_out, one_idx = _run(w, cp_plan(N, 1, w.m, w.n_win), kv, ki, pin, p, "cp_bt")
    plan = cp_plan(N, R, w.m, w.n_win, starts=starts)
    ranks, outs, idxs = _run(w, plan, kv, ki, pin, p, "cp_bt")
    want = _entries(w, one[0].lb, N)
    for r, rk in enumerate(ranks):
        assert _entries(w, rk.lb, N) == want, r
        p0, p1 = plan.rng(r)
        got = outs[r]
        assert bool(torch.isfinite(got).all()), r
        assert torch.equal(got.view(torch.int32), one_out[0][p0:p1].view(torch.int32)), r
        if w.is_csa:
            assert torch.equal(idxs[r], one_idx[0][p0:p1]), r
    # the one-piece cache and sampled rows against the oracle
    cv = cache_view(w, one[0].lb)
    exp = oracle.expected_append(kv, ki, 0, N, w.m, p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"),
                                 w.eps, w.theta, w.d_rope, window_from=0, key_e4m3=w.key_fmt == 1,
                                 per_channel=w.gate == 1)
    got_all = one_out[0].cpu().numpy().astype(np.float64)
    gidx = one_idx[0].cpu().numpy() if w.is_csa else None
    for r in range(R):
        p0, p1 = plan.rng(r)
        for pos in (p0, (p0 + p1) // 2, p1 - 1):
            L = pos + 1
            for wp in range(max(0, L - w.n_win), L):
                row, sc = exp["window"][wp]
                cv.win_rows[0, wp % w.n_win] = row
                cv.win_scales[0, wp % w.n_win] = sc
            if w.is_csa:
                # the GPU's selection: every entry clearly above the oracle's
                # k-th score, none clearly below; attention over that set
                nv = L // w.m
                sel = set(int(x) for x in gidx[pos] if x >= 0)
                if nv:
                    qI = oracle.index_query(pin["cq"][pos], p["W_iq"], w.HI, w.dI)
                    ref_s = oracle.index_scores(qI, pin["head_w"][pos], cv.gather_keys(0, nv))
                    kth = np.sort(ref_s)[::-1][min(w.k, nv) - 1]
                    assert set(np.nonzero(ref_s > kth + 1e-4)[0].tolist()) <= sel, pos
                    assert not (sel & set(np.nonzero(ref_s < kth - 1e-4)[0].tolist())), pos
                    assert len(sel) == min(w.k, nv), pos
                rows = cv.gather_set(0, L, gidx[pos])
            else:
                rows = cv.gather_set(0, L)
            ref, _ = oracle.attend(pin["q"][pos], p["gamma_q"], pos, rows, p["sink"], w.eps, w.theta, w.d_rope)
            check_out(got_all[pos], ref)
